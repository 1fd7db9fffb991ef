"""The allocation-free decode entry point.

``paged_attention_decode_noalloc`` serves callers that cannot allocate device memory (for
example a host whose device memory is entirely owned by its own pool, or a serving loop
that must not call cudaMalloc mid-step because the call may synchronise the device).  It
keeps its split-partition scratch in a fixed array inside the library.  These tests call
it through the C ABI and check that two calls in a row give what the regular entry point
gives, and what the fp64 oracle gives (with either work split), within the parity
tolerance, and that sizes needing more scratch than the array holds are rejected.  They set up everything they use, so they pass alone in a fresh
process as well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, device_inputs, widen, workspace_for

pytestmark = pytest.mark.gpu


def _noalloc_raw(out, d, wl, max_seq_len, partition_size):
    """Call the C entry point directly (ctypes), as a C caller would."""
    L = pkv.lib()
    return L.paged_attention_decode_noalloc(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(d["q"].data_ptr()),
        ctypes.c_void_p(d["k_cache"].data_ptr()), ctypes.c_void_p(d["v_cache"].data_ptr()),
        ctypes.c_void_p(d["block_tables"].data_ptr()), wl.max_blocks,
        ctypes.c_void_p(d["seq_lens"].data_ptr()), max_seq_len, wl.B, wl.Hq, wl.Hkv, wl.D, wl.bs,
        wl.num_blocks, wl.scale, pkv.PKV_BF16 if wl.dtype == "bf16" else pkv.PKV_F32,
        partition_size, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,sd,P", [("long", 16, 256), ("long", 16, 0), ("gqa16", 8, 64),
                                       ("mha", 16, 0), ("tiny", 1, 16)])
def test_noalloc_matches_regular_entry_point(name, sd, P):
    pkv.device_errors(clear=True)
    wl = workloads.make(name, scale_down=sd)
    host = workloads.host_tensors(wl)
    d = device_inputs(wl, host)
    pkv.paged_kv_write(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["slot_mapping"])
    need = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len,
                                                     wl.bs, P)
    assert need <= pkv.NOALLOC_SCRATCH_BYTES

    ref = torch.empty_like(d["q"])
    pkv.paged_attention_decode(ref, d["q"], d["k_cache"], d["v_cache"], d["block_tables"],
                               d["seq_lens"], wl.max_seq_len, wl.scale,
                               workspace=workspace_for(wl, P), partition_size=P)
    expect = widen(ref)
    for call in range(2):  # two calls in a row share the library's scratch array
        out = torch.full_like(d["q"], float("nan"))
        assert _noalloc_raw(out, d, wl, wl.max_seq_len, P) == pkv.PKV_OK
        torch.cuda.synchronize()
        assert_attention_close(widen(out), expect, wl.dtype, f"{name} P={P} call {call}")
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("split", ["fixed", "balanced"])
def test_noalloc_matches_oracle(split):
    """The allocation-free decode against the fp64 oracle directly, with the library's
    default split and with the work-balanced split (whose scratch layout differs)."""
    pkv.device_errors(clear=True)
    wl = workloads.make("long", scale_down=16)
    host = workloads.host_tensors(wl)
    d = device_inputs(wl, host)
    pkv.paged_kv_write(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"], d["slot_mapping"])
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    assert oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping) == 0
    ref = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, wl.seq_lens_post, wl.scale)
    old = pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED if split == "balanced"
                               else pkv.PKV_SPLIT_FIXED)
    try:
        for call in range(2):
            out = torch.full_like(d["q"], float("nan"))
            assert _noalloc_raw(out, d, wl, wl.max_seq_len, 0) == pkv.PKV_OK
            torch.cuda.synchronize()
            assert_attention_close(widen(out), ref, wl.dtype, f"{split} call {call}")
    finally:
        pkv.set_decode_split(old)
    assert pkv.device_errors() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    wl = workloads.custom("big", "bf16", 4, 32, 8, 128, 16, [8000] * 4, seed=5)
    d = workloads.device_tensors(wl, "cuda")
    d["block_tables"] = torch.from_numpy(wl.block_tables).cuda()
    d["seq_lens"] = torch.from_numpy(wl.seq_lens_post).cuda()
    out = torch.empty_like(d["q"])
    # partitions of 16 tokens over 8001-token sequences need far more than the fixed scratch
    need = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len,
                                                     wl.bs, 16)
    assert need > pkv.NOALLOC_SCRATCH_BYTES
    assert _noalloc_raw(out, d, wl, wl.max_seq_len, 16) == pkv.PKV_ERR_SCRATCH_LIMIT
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_decode_noalloc(out, d["q"], d["k_cache"], d["v_cache"],
                                           d["block_tables"], d["seq_lens"], wl.max_seq_len,
                                           wl.scale, partition_size=16)
    # the same sizes with the library's own partition length fit and match the regular call
    P = 0
    assert pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len,
                                                     wl.bs, P) <= pkv.NOALLOC_SCRATCH_BYTES
    pkv.paged_kv_write(d["k_new"], d["v_new"], d["k_cache"], d["v_cache"],
                       torch.from_numpy(wl.slot_mapping).cuda())
    ref = torch.empty_like(d["q"])
    pkv.paged_attention_decode(ref, d["q"], d["k_cache"], d["v_cache"], d["block_tables"],
                               d["seq_lens"], wl.max_seq_len, wl.scale,
                               workspace=workspace_for(wl, P))
    assert _noalloc_raw(out, d, wl, wl.max_seq_len, P) == pkv.PKV_OK
    torch.cuda.synchronize()
    assert_attention_close(widen(out), widen(ref), wl.dtype, "big P=auto")
