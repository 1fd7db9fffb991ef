"""Host-side pieces of bench.py and of the input builder that the benchmark relies on
(no GPU): the compact oracle sample decodes exactly like the full pool, the sample sizes
stay within their budget, and both benchmark arms describe a workload with the same
config dict."""
import argparse

import numpy as np
import torch

import bench
import oracle
from paged_kv_cache_344_b200 import workloads


def _bf16(t):
    return torch.from_numpy(np.ascontiguousarray(t)).view(torch.int16).view(torch.bfloat16)


def test_compact_sample_decodes_like_the_full_pool():
    """Gathering the first sequences' blocks into a compact pool (shared blocks once, tables
    renumbered) changes nothing in the decode: the oracle gives bit-identical rows."""
    for name, sd in (("share_fork", 8), ("gqa16", 16), ("long", 64)):
        wl = workloads.make(name, scale_down=sd)
        host = workloads.host_tensors(wl)
        kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
        oracle.copy_blocks(kc, vc, wl.cow_pairs)
        oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping)
        n = max(1, wl.B // 2)
        sample = workloads.compact_sample(wl, n, _bf16(kc), _bf16(vc))
        assert sample["k_cache"].shape[0] <= wl.num_blocks
        q = host["q"][:n]
        full = oracle.paged_decode(q, kc, vc, wl.block_tables[:n], wl.seq_lens_post[:n], wl.scale)
        comp = oracle.paged_decode(q, sample["k_cache"], sample["v_cache"], sample["block_tables"],
                                   sample["seq_lens"], wl.scale)
        assert np.array_equal(full, comp), name


def test_compact_sample_counts_shared_blocks_once():
    wl = workloads.make("share_tails", scale_down=8)
    sample = workloads.compact_sample(wl, wl.B)
    assert sample["k_cache"].shape[0] == workloads.unique_blocks_touched(wl)
    assert bench.sample_bytes(wl, sample) == workloads.decode_algorithmic_bytes(wl)


def test_oracle_sample_size_respects_the_budget():
    wl = workloads.make("mha", scale_down=4)
    rows = wl.seq_lens_post.astype(np.int64) * wl.Hq
    for budget in (1, int(rows[0]), int(rows[:3].sum()), 10 ** 12):
        n = bench.oracle_sample_size(wl, budget)
        assert 1 <= n <= wl.B
        assert n == wl.B or rows[:n].sum() >= budget
        assert n == 1 or rows[:n - 1].sum() < budget


def test_both_arms_report_the_same_config():
    args = argparse.Namespace(contiguous=False, block_size=0, decode="auto", step="fused")
    for name in bench.PER_CONFIG:
        wl = workloads.make(name, scale_down=16)
        shared = name.startswith("share")
        a = bench.config_dict(args, name, wl, True, shared, len(wl.cow_pairs) > 0, 1)
        assert a["workload"] == name and a["block_size"] == wl.bs
        assert a["bytes_per_step"] == (workloads.decode_algorithmic_bytes(wl) +
                                       workloads.write_bytes(wl) + workloads.copy_bytes(wl))


def test_pools_hold_eight_l2s_or_flush():
    """Small working sets are cycled through enough pools to hold 8 L2s; beyond
    MAX_POOLS pools the bench flushes L2 instead."""
    L2 = bench.L2_BYTES
    assert bench.pools_for(8 * L2) == 1 and bench.pools_for(20 * L2) == 1
    for ws in (158_371_328, 211_064_720, L2, 8 * L2 - 1):
        n = bench.pools_for(ws)
        assert n >= 2 and n * ws >= 8 * L2 and (n - 1) * ws < 8 * L2
    assert bench.pools_for(8 * L2 // bench.MAX_POOLS) == bench.MAX_POOLS
    assert bench.pools_for(8 * L2 // bench.MAX_POOLS - 1) == 0
    assert bench.pools_for(4096) == 0
