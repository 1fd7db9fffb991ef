"""GPU parity of the tcgen05 multi-query (prefill / chunked append) attention against the
oracle's fp64 definition: every query row is causal attention over the tokens up to its
own position.  Covers pure prefill (no context), chunks appended to long contexts, single
queries, query tiles cut mid-sequence, G = 1..16, D = 64/128/256, block sizes 16 to 256,
NaN-poisoned unused slots, positive, negative and zero scales and score ranges that move
the running maximum many times; on both kernels (two query tiles per CTA, warp-specialised,
and one tile per CTA)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, to_device, widen

pytestmark = pytest.mark.gpu


def _run(Hq, Hkv, D, bs, lens, qlens, seed=3, scale=None):
    wl = workloads.custom("pf", "bf16", len(lens), Hq, Hkv, D, bs, lens, seed=seed)
    host = workloads.host_tensors(wl)
    rng = np.random.default_rng(seed + 1)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    qf = rng.standard_normal((int(cu[-1]), Hq, D), dtype=np.float32)
    q = torch.from_numpy(qf).to(torch.bfloat16)
    q_bits = q.view(torch.int16).numpy().view(np.uint16)
    seq = np.asarray(lens, np.int32)
    scale = wl.scale if scale is None else scale
    ref = oracle.paged_prefill(q_bits, host["k_cache"], host["v_cache"], wl.block_tables, seq, cu,
                               scale)
    dev_q = q.cuda()
    out = torch.full_like(dev_q, float("nan"))
    pkv.paged_attention_prefill(out, dev_q, to_device(host["k_cache"], "bf16"),
                                to_device(host["v_cache"], "bf16"),
                                torch.from_numpy(wl.block_tables).cuda(),
                                torch.from_numpy(seq).cuda(), torch.from_numpy(cu).cuda(),
                                int(max(qlens)), int(seq.max()), scale,
                                workspace=_workspace(len(lens), Hq, Hkv, int(max(qlens))))
    torch.cuda.synchronize()
    return widen(out), ref


PATHS = ["persistent", "per_item", "single_tile"]
_path = {"name": "persistent"}


@pytest.fixture(autouse=True, params=PATHS)
def path(request):
    old = pkv.set_prefill_path(pkv.PKV_PREFILL_SINGLE_TILE if request.param == "single_tile"
                               else pkv.PKV_PREFILL_AUTO)
    _path["name"] = request.param
    pkv.device_errors(clear=True)
    yield request.param
    torch.cuda.synchronize()
    pkv.set_prefill_path(old)
    assert pkv.device_errors() == 0


_ws = {"buf": None}


def _workspace(B, Hq, Hkv, max_q):
    """Scratch for the persistent schedule: one buffer reused by every call (each call
    rebuilds its schedule), filled with garbage when it is (re)allocated, since it needs no
    initialisation; None on the per-item path."""
    if _path["name"] == "per_item":
        return None
    n = pkv.paged_attention_prefill_workspace_size(B, Hq, Hkv, max_q) // 4 + 1
    if _ws["buf"] is None or _ws["buf"].numel() < n:
        _ws["buf"] = torch.full((n,), -7, dtype=torch.int32, device="cuda")
    return _ws["buf"]


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
    pkv.paged_attention_prefill(out_p, q, kc, vc, bt, seq, cu, 1, max(lens), wl.scale,
                                workspace=_workspace(3, 32, 8, 1))
    ref = oracle.paged_decode(host["q"], host["k_cache"], host["v_cache"], wl.block_tables,
                              np.asarray(lens, np.int32), wl.scale)
    assert_attention_close(widen(out_p), ref, "bf16", "prefill Q=1")


@pytest.mark.parametrize("qlens", [[31, 32, 33, 63, 64, 65, 96, 128, 129]],
                         ids=["around-two-tiles"])
def test_prefill_two_tile_edges(qlens):
    """G = 4 (32 query tokens per 128-row tile): chunks that end inside the first tile,
    exactly on the tile pair, and one past it; contexts of 0 and 100 tokens."""
    lens = [q + (0 if i % 2 else 100) for i, q in enumerate(qlens)]
    got, ref = _run(32, 8, 128, 16, lens, qlens, seed=11)
    assert_attention_close(got, ref, "bf16", "two-tile edges")


def test_prefill_long_context_ring_wrap():
    """Chunks appended to 3000-4700 cached tokens: dozens of K/V tiles cycle the ring."""
    got, ref = _run(32, 8, 128, 16, [3000, 4700, 2100], [300, 512, 77], seed=13)
    assert_attention_close(got, ref, "bf16", "long context")


@pytest.mark.parametrize("bs", [64, 128, 256])
def test_prefill_large_blocks(bs):
    got, ref = _run(16, 2, 128, bs, [900, 260, 1], [150, 260, 1], seed=15)
    assert_attention_close(got, ref, "bf16", f"bs={bs}")


@pytest.mark.parametrize("scale", [1.0, -0.3, 0.0], ids=["wide", "negative", "zero"])
def test_prefill_scales(scale):
    """scale 1.0 spreads the scores over hundreds of log2 units (the running maximum moves
    often and O is rescaled); a negative scale flips which score is largest; zero gives
    uniform weights over the visible prefix."""
    got, ref = _run(16, 4, 128, 16, [700, 130, 64], [200, 130, 5], seed=17, scale=scale)
    assert_attention_close(got, ref, "bf16", f"scale={scale}")


def test_prefill_workspace_reuse_across_calls():
    """The shared workspace across calls with different batches in a row, with more work
    items than the persistent grid has CTAs (each CTA takes several items)."""
    if _path["name"] != "persistent":
        pytest.skip("persistent schedule only")
    for seed, lens, qlens in [(21, [500, 90, 3000, 70], [500, 90, 200, 1]),
                              (22, [1200] * 12, [300] * 12)]:
        got, ref = _run(32, 8, 128, 16, lens, qlens, seed=seed)
        assert_attention_close(got, ref, "bf16", f"seed {seed}")


def test_prefill_device_checks_flag_and_stay_in_bounds():
    """Out-of-range block ids are flagged and read as zeros (the rest of the batch is exact);
    a sequence with more queries than tokens is flagged and its rows are left as they were."""
    lens, qlens = [200, 90, 50], [40, 30, 60]  # sequence 2 has Q > L
    wl = workloads.custom("pf", "bf16", 3, 32, 8, 128, 16, lens, seed=31)
    host = workloads.host_tensors(wl)
    rng = np.random.default_rng(32)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = torch.from_numpy(rng.standard_normal((int(cu[-1]), 32, 128), dtype=np.float32))
    q = q.to(torch.bfloat16)
    bt = wl.block_tables.copy()
    bt[0, 3] = wl.num_blocks + 7  # sequence 0: one block id out of range
    seq = np.asarray(lens, np.int32)
    out = torch.full_like(q, 3.0).cuda()
    pkv.device_errors(clear=True)
    pkv.paged_attention_prefill(out, q.cuda(), to_device(host["k_cache"], "bf16"),
                                to_device(host["v_cache"], "bf16"), torch.from_numpy(bt).cuda(),
                                torch.from_numpy(seq).cuda(), torch.from_numpy(cu).cuda(),
                                max(qlens), max(lens), wl.scale,
                                workspace=_workspace(3, 32, 8, max(qlens)))
    torch.cuda.synchronize()
    bits = pkv.device_errors(clear=True)
    assert bits & pkv.DEVERR_BLOCK_ID and bits & pkv.DEVERR_SEQLEN
    got = widen(out)
    assert np.isfinite(got).all()
    # sequence 2's rows are untouched
    assert np.all(got[cu[2]:cu[3]] == 3.0)
    # sequence 1 (valid table, valid lengths) is exact
    q_bits = q.view(torch.int16).numpy().view(np.uint16)
    ref = oracle.paged_prefill(np.ascontiguousarray(q_bits[cu[1]:cu[2]]), host["k_cache"],
                               host["v_cache"], np.ascontiguousarray(wl.block_tables[1:2]),
                               seq[1:2], np.array([0, qlens[1]], np.int32), wl.scale)
    assert_attention_close(got[cu[1]:cu[2]], ref, "bf16", "valid sequence beside bad ones")
    # sequence 0 equals attention with that block read as zeros
    kz, vz = host["k_cache"].copy(), host["v_cache"].copy()
    bad = wl.block_tables[0, 3]
    kz[bad] = 0
    vz[bad] = 0
    ref0 = oracle.paged_prefill(np.ascontiguousarray(q_bits[cu[0]:cu[1]]), kz, vz,
                                np.ascontiguousarray(wl.block_tables[0:1]), seq[0:1],
                                np.array([0, qlens[0]], np.int32), wl.scale)
    assert_attention_close(got[cu[0]:cu[1]], ref0, "bf16", "bad block read as zeros")
