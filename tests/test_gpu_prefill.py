"""GPU parity of the tcgen05 multi-query (prefill / chunked append) attention against the
oracle's fp64 definition: every query row is causal attention over the tokens up to its
own position.  Covers pure prefill (no context), chunks appended to long contexts, single
queries, query tiles cut mid-sequence, G = 1..16, D = 64/128/256, block sizes 16 and 32,
and NaN-poisoned unused slots."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, to_device, widen

pytestmark = pytest.mark.gpu


def _run(Hq, Hkv, D, bs, lens, qlens, seed=3):
    wl = workloads.custom("pf", "bf16", len(lens), Hq, Hkv, D, bs, lens, seed=seed)
    host = workloads.host_tensors(wl)
    rng = np.random.default_rng(seed + 1)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    qf = rng.standard_normal((int(cu[-1]), Hq, D), dtype=np.float32)
    q = torch.from_numpy(qf).to(torch.bfloat16)
    q_bits = q.view(torch.int16).numpy().view(np.uint16)
    seq = np.asarray(lens, np.int32)
    ref = oracle.paged_prefill(q_bits, host["k_cache"], host["v_cache"], wl.block_tables, seq, cu,
                               wl.scale)
    dev_q = q.cuda()
    out = torch.full_like(dev_q, float("nan"))
    pkv.paged_attention_prefill(out, dev_q, to_device(host["k_cache"], "bf16"),
                                to_device(host["v_cache"], "bf16"),
                                torch.from_numpy(wl.block_tables).cuda(),
                                torch.from_numpy(seq).cuda(), torch.from_numpy(cu).cuda(),
                                int(max(qlens)), int(seq.max()), wl.scale)
    torch.cuda.synchronize()
    return widen(out), ref


@pytest.fixture(autouse=True)
def _clean():
    pkv.device_errors(clear=True)
    yield
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (16, 4), (32, 4), (64, 8), (32, 2)])
def test_prefill_matches_oracle(Hq, Hkv):
    lens = [40, 300, 17, 129, 1000]
    qlens = [40, 57, 1, 129, 200]   # pure prefill, chunks, one query, a long append
    got, ref = _run(Hq, Hkv, 128, 16, lens, qlens)
    assert_attention_close(got, ref, "bf16", f"G={Hq // Hkv}")


@pytest.mark.parametrize("D", [64, 256])
def test_prefill_head_dims(D):
    got, ref = _run(16, 4, D, 16, [70, 33, 400], [70, 9, 130], seed=7)
    assert_attention_close(got, ref, "bf16", f"D={D}")


def test_prefill_block_size_32_and_tile_edges():
    """Chunk lengths around the 128-row query tile and the 64-token K/V tile."""
    got, ref = _run(32, 8, 128, 32, [64, 65, 127, 128, 129, 700], [16, 17, 63, 64, 65, 300],
                    seed=9)
    assert_attention_close(got, ref, "bf16", "bs=32 edges")


def test_prefill_single_query_equals_decode():
    """With one query per sequence the prefill kernel computes the decode."""
    lens = [10, 200, 1500]
    wl = workloads.custom("pd", "bf16", 3, 32, 8, 128, 16, lens, seed=5)
    host = workloads.host_tensors(wl)
    q = to_device(host["q"], "bf16")
    kc, vc = to_device(host["k_cache"], "bf16"), to_device(host["v_cache"], "bf16")
    bt = torch.from_numpy(wl.block_tables).cuda()
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    cu = torch.arange(4, dtype=torch.int32, device="cuda")
    out_p = torch.empty_like(q)
    pkv.paged_attention_prefill(out_p, q, kc, vc, bt, seq, cu, 1, max(lens), wl.scale)
    ref = oracle.paged_decode(host["q"], host["k_cache"], host["v_cache"], wl.block_tables,
                              np.asarray(lens, np.int32), wl.scale)
    assert_attention_close(widen(out_p), ref, "bf16", "prefill Q=1")
