"""GPU parity of the shared-prefix decode against the fp64 oracle.

The shared-prefix entry point must give the same attention as the plain decode: the
oracle's definition does not know about groups.  Cases: the two shared-prefix workloads
(fork with copy-on-write, shared prefix with private tails), one-member groups (nothing
shared), random group sizes with G = 1, 4, 8, 16 (member chunks of 16 / G), partition
lengths that cut prefixes and tails into many pieces, prefix lengths that must be clamped,
empty sequences, and a table that breaks the sharing contract (flagged).
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, device_inputs, oracle_step, widen

pytestmark = pytest.mark.gpu


def _run_shared(wl, dev, partition_size=0, prefix_lens=None, offsets=None, seq_lens=None,
                max_group=None):
    offs = wl.group_offsets if offsets is None else offsets
    plen = wl.prefix_lens if prefix_lens is None else prefix_lens
    sl = dev["seq_lens"] if seq_lens is None else seq_lens
    msl = int(sl.max().item())
    n = pkv.paged_attention_decode_shared_prefix_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, msl,
                                                                wl.bs, partition_size)
    ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
    out = torch.full_like(dev["q"], float("nan"))
    mg = max_group or int(np.diff(offs).max())
    pkv.paged_attention_decode_shared_prefix(
        out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], sl, msl, wl.scale,
        torch.from_numpy(np.asarray(offs, np.int32)).cuda(),
        torch.from_numpy(np.asarray(plen, np.int32)).cuda(), mg, workspace=ws,
        partition_size=partition_size)
    return out, ws


def _step_inputs(wl, host):
    dev = device_inputs(wl, host)
    if len(wl.cow_pairs):
        pkv.copy_blocks(dev["k_cache"], dev["v_cache"], dev["cow_pairs"])
    pkv.paged_kv_write(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
                       dev["slot_mapping"])
    return dev


@pytest.fixture(autouse=True)
def _clean():
    pkv.device_errors(clear=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("P", [0, 16, 128])
@pytest.mark.parametrize("name,sd", [("share_fork", 4), ("share_tails", 4), ("share_tails", 2),
                                     ("mha", 8), ("gqa16", 8)])
def test_shared_prefix_matches_oracle(name, sd, P):
    wl = workloads.make(name, scale_down=sd)
    host = workloads.host_tensors(wl)
    dev = _step_inputs(wl, host)
    out, ws = _run_shared(wl, dev, P)
    _, _, ref = oracle_step(wl, host)
    assert_attention_close(widen(out), ref, wl.dtype, f"{name} P={P}")
    assert pkv.device_errors() == 0
    assert int(ws[:wl.B * wl.Hkv * 4].view(torch.int32).abs().sum()) == 0  # tickets reset


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (32, 4), (64, 8), (32, 2)])
def test_random_groups_and_heads(Hq, Hkv):
    """Group sizes 1..9 (more members than fit one 16-row piece when G is small or large),
    prefixes of whole blocks, private tails from 0 tokens up."""
    rng = np.random.default_rng(Hq * 100 + Hkv)
    sizes = [1, 3, 9, 2, 5, 1, 4]
    shared = [int(x) * 16 for x in rng.integers(0, 12, size=len(sizes))]
    tails = [int(x) for x in rng.integers(0, 70, size=sum(sizes))]
    wl = workloads.grouped("grp", "bf16", Hq, Hkv, 128, 16, sizes, shared, tails, seed=11)
    host = workloads.host_tensors(wl)
    dev = _step_inputs(wl, host)
    _, _, ref = oracle_step(wl, host)
    for P in (0, 32):
        out, _ = _run_shared(wl, dev, P)
        assert_attention_close(widen(out), ref, wl.dtype, f"G={Hq // Hkv} P={P}")
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("D,bs", [(64, 16), (256, 32), (128, 64)])
def test_head_dims_and_block_sizes(D, bs):
    wl = workloads.grouped("grp", "bf16", 16, 4, D, bs, [4, 2, 3], [2 * bs, bs, 3 * bs],
                           [0, 5, bs, 40, 1, 2, 3, 70, 9], seed=3)
    host = workloads.host_tensors(wl)
    dev = _step_inputs(wl, host)
    out, _ = _run_shared(wl, dev, 0)
    _, _, ref = oracle_step(wl, host)
    assert_attention_close(widen(out), ref, wl.dtype, f"D={D} bs={bs}")
    assert pkv.device_errors() == 0


def test_prefix_lengths_are_clamped_and_empty_sequences():
    """A claimed prefix that is not a multiple of 16, or longer than a member, is cut down
    to what every member holds; empty sequences give zero rows."""
    wl = workloads.grouped("grp", "bf16", 32, 8, 128, 16, [3, 4], [48, 64], [7, 0, 30, 3, 1, 2, 9],
                           seed=9)
    host = workloads.host_tensors(wl)
    dev = _step_inputs(wl, host)
    _, _, ref = oracle_step(wl, host)
    out, _ = _run_shared(wl, dev, 0, prefix_lens=[40, 10_000])
    assert_attention_close(widen(out), ref, wl.dtype, "clamped prefix")
    seq = dev["seq_lens"].clone()
    seq[1] = 0
    seq[5] = 0
    out, _ = _run_shared(wl, dev, 16, seq_lens=seq)
    lens = wl.seq_lens_post.copy()
    lens[[1, 5]] = 0
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    oracle.copy_blocks(kc, vc, wl.cow_pairs)
    oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping)
    ref2 = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, lens, wl.scale)
    got = widen(out)
    assert_attention_close(got, ref2, wl.dtype, "empty members")
    assert np.all(got[[1, 5]] == 0.0)
    assert pkv.device_errors() == 0


def test_broken_sharing_contract_is_flagged():
    wl = workloads.grouped("grp", "bf16", 32, 8, 128, 16, [4], [64], [3, 4, 5, 6], seed=4)
    host = workloads.host_tensors(wl)
    dev = _step_inputs(wl, host)
    bt = dev["block_tables"].clone()
    bt[2, 1] = bt[2, 4]  # member 2 no longer holds the group's block 1 (its own tail block)
    out = torch.empty_like(dev["q"])
    n = pkv.paged_attention_decode_shared_prefix_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D,
                                                                wl.max_seq_len, wl.bs, 0)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    pkv.paged_attention_decode_shared_prefix(
        out, dev["q"], dev["k_cache"], dev["v_cache"], bt, dev["seq_lens"], wl.max_seq_len,
        wl.scale, torch.tensor([0, 4], dtype=torch.int32, device="cuda"),
        torch.tensor([64], dtype=torch.int32, device="cuda"), 4, workspace=ws)
    assert pkv.device_errors() & pkv.DEVERR_PREFIX
    # offsets that leave a sequence uncovered are flagged too, and stay in bounds
    pkv.paged_attention_decode_shared_prefix(
        out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["seq_lens"],
        wl.max_seq_len, wl.scale, torch.tensor([0, 2], dtype=torch.int32, device="cuda"),
        torch.tensor([64], dtype=torch.int32, device="cuda"), 4, workspace=ws)
    assert pkv.device_errors() & pkv.DEVERR_PREFIX


@pytest.mark.parametrize("Hq,Hkv,mc", [(8, 8, 16), (16, 4, 4), (64, 8, 2), (32, 2, 1)])
def test_grouped_pieces(Hq, Hkv, mc):
    """Groups whose members fit one 16-row MMA run one CTA per (group, KV head): the prefix
    stages and every member's own stages in one list, own stages scored for their member's
    rows only.  Group sizes up to the limit, prefixes from 0 tokens, tails from 0 tokens,
    and empty members; the split pieces (an explicit partition length) must agree."""
    rng = np.random.default_rng(Hq * 7 + Hkv)
    sizes = [int(x) for x in rng.integers(1, mc + 1, size=7)] + [mc]
    shared = [int(x) * 16 for x in rng.integers(0, 14, size=len(sizes))]
    tails = [int(x) for x in rng.integers(0, 90, size=sum(sizes))]
    wl = workloads.grouped("grp", "bf16", Hq, Hkv, 128, 16, sizes, shared, tails, seed=21)
    host = workloads.host_tensors(wl)
    dev = _step_inputs(wl, host)
    _, _, ref = oracle_step(wl, host)
    for P in (0, 32):
        out, _ = _run_shared(wl, dev, P)
        assert_attention_close(widen(out), ref, wl.dtype, f"G={Hq // Hkv} P={P}")
    # empty members in the one-CTA-per-group path
    seq = dev["seq_lens"].clone()
    empty = [0, wl.B - 1]
    seq[empty] = 0
    out, _ = _run_shared(wl, dev, 0, seq_lens=seq)
    lens = wl.seq_lens_post.copy()
    lens[empty] = 0
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    oracle.copy_blocks(kc, vc, wl.cow_pairs)
    oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping)
    ref2 = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, lens, wl.scale)
    got = widen(out)
    assert_attention_close(got, ref2, wl.dtype, "empty members")
    assert np.all(got[empty] == 0.0)
    assert pkv.device_errors() == 0
