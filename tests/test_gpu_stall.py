"""The pipelines' time limit on the GPU, without a fault.

A bounded wait that nothing satisfies (the library's own wait, in its self-test kernel)
gives up after its limit, sets DEVERR_TIMEOUT and leaves the context usable.  While that
bit is set, every CTA of every attention launch returns whole at once: the fused decode
step, the work-balanced decode, the shared-prefix decode and both prefill kernels leave
their outputs and the cache as they were.  Once the bit is cleared the same calls are
exact again.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import (assert_attention_close, device_inputs, gpu_step, oracle_step, widen,
                      workspace_for)

pytestmark = pytest.mark.gpu

SENTINEL = 5.0


def _prefill_case(seed=41):
    lens, qlens = [300, 64, 1000], [100, 64, 17]
    wl = workloads.custom("pf", "bf16", len(lens), 32, 8, 128, 16, lens, seed=seed)
    host = workloads.host_tensors(wl)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    q = torch.randn((int(cu[-1]), 32, 128), generator=g).to(torch.bfloat16).cuda()
    dev = device_inputs(wl, host)
    ws = torch.empty(pkv.paged_attention_prefill_workspace_size(3, 32, 8, max(qlens)),
                     dtype=torch.uint8, device="cuda")
    args = (q, dev["k_cache"], dev["v_cache"], dev["block_tables"],
            torch.tensor(lens, dtype=torch.int32, device="cuda"), torch.from_numpy(cu).cuda(),
            max(qlens), max(lens), wl.scale)
    return args, ws


def _stand_down_calls():
    """Every attention entry point once, on small inputs, outputs filled with SENTINEL;
    returns the outputs and the caches (with copies from before the calls)."""
    checks = []
    # fused decode step (copy-on-write + cache write + decode), fixed split
    wl = workloads.make("gqa16", scale_down=8)
    dev = device_inputs(wl, workloads.host_tensors(wl))
    before = (dev["k_cache"].clone(), dev["v_cache"].clone())
    out = torch.full_like(dev["q"], SENTINEL)
    cow = torch.from_numpy(wl.cow_src).cuda() if len(wl.cow_pairs) else None
    pkv.paged_decode_step(out, dev["q"], dev["k_new"], dev["v_new"], dev["k_cache"],
                          dev["v_cache"], dev["block_tables"], dev["seq_lens"], wl.max_seq_len,
                          wl.scale, cow_src=cow, workspace=workspace_for(wl))
    checks.append(("fused step", out, before, (dev["k_cache"], dev["v_cache"])))
    # work-balanced decode
    old = pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED)
    try:
        out = torch.full_like(dev["q"], SENTINEL)
        pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"],
                                   dev["block_tables"], dev["seq_lens"], wl.max_seq_len, wl.scale,
                                   workspace=workspace_for(wl))
        checks.append(("balanced decode", out, None, None))
    finally:
        pkv.set_decode_split(old)
    # shared-prefix decode: one CTA per group, and pieces with a partition length
    ws_ = workloads.make("share_tails", scale_down=4)
    sdev = device_inputs(ws_, workloads.host_tensors(ws_))
    offs = torch.from_numpy(ws_.group_offsets).cuda()
    plen = torch.from_numpy(ws_.prefix_lens).cuda()
    mg = int(np.diff(ws_.group_offsets).max())
    for P in (0, 64):
        n = pkv.paged_attention_decode_shared_prefix_workspace_size(
            ws_.B, ws_.Hq, ws_.Hkv, ws_.D, ws_.max_seq_len, ws_.bs, P)
        out = torch.full_like(sdev["q"], SENTINEL)
        pkv.paged_attention_decode_shared_prefix(
            out, sdev["q"], sdev["k_cache"], sdev["v_cache"], sdev["block_tables"],
            sdev["seq_lens"], ws_.max_seq_len, ws_.scale, offs, plen, mg,
            workspace=torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda"),
            partition_size=P)
        checks.append((f"shared prefix P={P}", out, None, None))
    # prefill: the persistent two-tile kernel, its per-item launch and the single-tile kernel
    args, ws = _prefill_case()
    for name, mode, w in [("prefill persistent", pkv.PKV_PREFILL_AUTO, ws),
                          ("prefill per item", pkv.PKV_PREFILL_AUTO, None),
                          ("prefill single tile", pkv.PKV_PREFILL_SINGLE_TILE, ws)]:
        old = pkv.set_prefill_path(mode)
        try:
            out = torch.full_like(args[0], SENTINEL)
            pkv.paged_attention_prefill(out, *args, workspace=w)
            checks.append((name, out, None, None))
        finally:
            pkv.set_prefill_path(old)
    return checks


def test_stalled_wait_gives_up_and_attention_stands_down():
    pkv.device_errors(clear=True)
    pkv.debug_stalled_wait()
    torch.cuda.synchronize()  # the wait ends by itself
    assert pkv.device_errors(clear=False) == pkv.DEVERR_TIMEOUT

    checks = _stand_down_calls()
    torch.cuda.synchronize()
    for name, out, before, after in checks:
        assert bool((out == SENTINEL).all()), f"{name}: output written after a timeout"
        if before is not None:
            # bitwise (unused slots hold NaN)
            same = all(torch.equal(x.view(torch.int16), y.view(torch.int16))
                       for x, y in zip(before, after))
            assert same, f"{name}: cache written after a timeout"
    # nothing else was flagged, and clearing works
    assert pkv.device_errors(clear=True) == pkv.DEVERR_TIMEOUT
    assert pkv.device_errors(clear=False) == 0

    # the context is usable and the same step is exact again
    wl = workloads.make("gqa16", scale_down=8)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, fused=True)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(wl, host)
    assert_attention_close(widen(out), ref, wl.dtype, "fused step after clearing")
    assert pkv.device_errors() == 0


def test_workspace_zero_fill_restores_it_after_a_timeout():
    """A launch stopped by a timeout can leave partition tickets non-zero in its workspace
    (its CTAs that stopped early took none).  The documented remedy is to zero-fill the
    workspace before its next use; this plants such leftover tickets, applies the remedy
    and checks that the decode is exact again."""
    pkv.device_errors(clear=True)
    wl = workloads.make("long", scale_down=16)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    P = 64
    ws = workspace_for(wl, P)
    units = wl.B * wl.Hkv
    ws[:4 * units].view(torch.int32).fill_(3)  # what a stopped launch may leave behind
    ws.zero_()  # the remedy: zero-fill before the next use
    out = gpu_step(wl, dev, partition_size=P, workspace=ws, fused=True)
    torch.cuda.synchronize()
    _, _, ref = oracle_step(wl, host)
    assert_attention_close(widen(out), ref, wl.dtype, "after zero-filling the workspace")
    assert int(ws[:4 * units].view(torch.int32).abs().sum()) == 0  # tickets back at zero
    assert pkv.device_errors() == 0
