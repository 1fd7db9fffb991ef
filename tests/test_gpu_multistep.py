"""GPU parity of consecutive decode steps launched back to back.

Every kernel is launched with programmatic stream serialization: the next launch's CTAs
may be placed while the previous kernel finishes, and each waits for it before touching
global memory.  Here T fused steps run on one cache with no synchronisation between them.
Step t writes each sequence's token at position L + t and attends over L + t + 1 tokens,
so it reads the rows that step t - 1 has just written, and every step reuses the
workspace the previous one left behind.  The oracle runs the same steps one after the
other: each output within the bf16 tolerance, the pool at the end byte for byte.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, to_device, to_host_bits, widen

pytestmark = pytest.mark.gpu

T = 4  # steps; each sequence's tokens L .. L + T - 1 lie in one block


@pytest.fixture(autouse=True)
def _clean():
    pkv.device_errors(clear=True)
    yield
    torch.cuda.synchronize()


def _steps(wl):
    """Per step: q, k_new, v_new (host bits), slot mapping and lengths after the step."""
    L = wl.seq_lens_pre.astype(np.int64)
    assert np.all(L % wl.bs + T <= wl.bs)
    out = []
    for t in range(T):
        h = workloads.host_tensors(wl, seed_offset=100 + t)
        pos = L + t
        slots = wl.block_tables[np.arange(wl.B), pos // wl.bs].astype(np.int64) * wl.bs + pos % wl.bs
        out.append((h["q"], h["k_new"], h["v_new"], slots, (pos + 1).astype(np.int32)))
    return out


def _oracle(wl, host, steps):
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    refs = []
    for q, kn, vn, slots, lens in steps:
        assert oracle.kv_write(kn, vn, kc, vc, slots) == 0
        refs.append(oracle.paged_decode(q, kc, vc, wl.block_tables, lens, wl.scale))
    return kc, vc, refs


def _device_steps(wl, steps):
    return [tuple(to_device(a, wl.dtype) for a in (q, kn, vn)) +
            (torch.from_numpy(lens).cuda(),) for q, kn, vn, _, lens in steps]


@pytest.mark.parametrize("P", [0, 16])
def test_back_to_back_fused_steps(P):
    lens = [5, 130, 2050, 4100, 16 * 300 + 3, 7, 1000, 1024]
    wl = workloads.custom("steps", "bf16", len(lens), 32, 8, 128, 16, lens, seed=61)
    host = workloads.host_tensors(wl)
    steps = _steps(wl)
    kc, vc, refs = _oracle(wl, host, steps)
    kcache = to_device(host["k_cache"], wl.dtype)
    vcache = to_device(host["v_cache"], wl.dtype)
    bt = torch.from_numpy(wl.block_tables).cuda()
    msl = wl.max_seq_len + T
    n = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, msl, wl.bs, P)
    ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
    dsteps = _device_steps(wl, steps)
    outs = [torch.full_like(d[0], float("nan")) for d in dsteps]
    torch.cuda.synchronize()
    for o, (q, kn, vn, sl) in zip(outs, dsteps):  # no synchronisation in between
        pkv.paged_decode_step(o, q, kn, vn, kcache, vcache, bt, sl, msl, wl.scale,
                              workspace=ws, partition_size=P)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    for t, (o, ref) in enumerate(zip(outs, refs)):
        assert_attention_close(widen(o), ref, wl.dtype, f"P={P} step {t}")
    assert to_host_bits(kcache).tobytes() == kc.tobytes()
    assert to_host_bits(vcache).tobytes() == vc.tobytes()


def test_back_to_back_group_steps():
    """The shared-prefix step, one CTA per (group, KV head): each member appends to its
    own tail block, through the stages of the write."""
    sizes = [4, 4, 2, 3]
    shared = [64, 32, 80, 0]
    tails = [3, 20, 0, 40, 5, 18, 33, 12, 1, 7, 44, 28, 9]
    wl = workloads.grouped("gsteps", "bf16", 32, 8, 128, 16, sizes, shared, tails, seed=63)
    assert len(wl.cow_pairs) == 0
    host = workloads.host_tensors(wl)
    steps = _steps(wl)
    kc, vc, refs = _oracle(wl, host, steps)
    kcache = to_device(host["k_cache"], wl.dtype)
    vcache = to_device(host["v_cache"], wl.dtype)
    bt = torch.from_numpy(wl.block_tables).cuda()
    go = torch.from_numpy(wl.group_offsets).cuda()
    pl = torch.from_numpy(wl.prefix_lens).cuda()
    mg = int(np.diff(wl.group_offsets).max())
    msl = wl.max_seq_len + T
    n = pkv.paged_attention_decode_shared_prefix_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, msl,
                                                                wl.bs, 0)
    ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
    dsteps = _device_steps(wl, steps)
    outs = [torch.full_like(d[0], float("nan")) for d in dsteps]
    torch.cuda.synchronize()
    for o, (q, kn, vn, sl) in zip(outs, dsteps):
        pkv.paged_decode_step_shared_prefix(o, q, kn, vn, kcache, vcache, bt, sl, msl, wl.scale,
                                            go, pl, mg, workspace=ws)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    for t, (o, ref) in enumerate(zip(outs, refs)):
        assert_attention_close(widen(o), ref, wl.dtype, f"group step {t}")
    assert to_host_bits(kcache).tobytes() == kc.tobytes()
    assert to_host_bits(vcache).tobytes() == vc.tobytes()


def test_launch_overlap_off_gives_the_same_bits():
    """With the launch overlap switched off the kernels start in plain stream order:
    the same steps give the same bits."""
    lens = [5, 130, 2050, 4100, 7, 1000]
    wl = workloads.custom("steps_off", "bf16", len(lens), 32, 8, 128, 16, lens, seed=65)
    host = workloads.host_tensors(wl)
    steps = _steps(wl)
    bt = torch.from_numpy(wl.block_tables).cuda()
    msl = wl.max_seq_len + T
    n = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, msl, wl.bs, 0)
    results = []
    for overlap in (True, False):
        old = pkv.set_launch_overlap(overlap)
        try:
            kcache = to_device(host["k_cache"], wl.dtype)
            vcache = to_device(host["v_cache"], wl.dtype)
            ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
            outs = []
            for q, kn, vn, sl in _device_steps(wl, steps):
                o = torch.empty_like(q)
                pkv.paged_decode_step(o, q, kn, vn, kcache, vcache, bt, sl, msl, wl.scale,
                                      workspace=ws)
                outs.append(o)
            torch.cuda.synchronize()
            results.append(([to_host_bits(o).tobytes() for o in outs],
                            to_host_bits(kcache).tobytes(), to_host_bits(vcache).tobytes()))
        finally:
            pkv.set_launch_overlap(old)
    assert results[0] == results[1]
    assert pkv.device_errors() == 0
