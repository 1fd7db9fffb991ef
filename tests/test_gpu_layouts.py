"""GPU parity of the two other cache layouts the decode kernel reads.

* Blocks of 8 tokens: a 16-token stage of the kernel is gathered from two blocks (two
  8-row TMA boxes).  The decode, the fused step and the cache update must match the fp64
  oracle, for both consumers and with partitions of every kind ("Paged Attention
  Explained", 2. Partial Block Waste: the block size is a trade-off the caller picks).
* The unpaged control (paged_attention_decode_contiguous): the same kernel over a
  contiguous [B, row_stride, Hkv, D] cache, with no block table at all.  On the same
  logical K/V it must give the oracle's result, and with the same partition length it
  computes exactly what the paged decode computes (same stages, same order), so the two
  outputs are equal bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import (assert_attention_close, device_inputs, gpu_step, oracle_step, raw,
                      to_host_bits, widen, workspace_for)

pytestmark = pytest.mark.gpu

PATHS = {"auto": pkv.PKV_PATH_AUTO, "cuda_cores": pkv.PKV_PATH_CUDA_CORES,
         "tensor_cores": pkv.PKV_PATH_TENSOR_CORES}


@pytest.fixture(autouse=True)
def _clean_state():
    pkv.device_errors(clear=True)
    old = pkv.set_decode_path(pkv.PKV_PATH_AUTO)
    yield
    pkv.set_decode_path(old)
    torch.cuda.synchronize()


def _bs8(name, sd):
    if name == "tiny8":
        return workloads.custom("tiny8", "f32", 4, 4, 4, 64, 8, [1, 7, 16, 33], seed=1000,
                                pool_factor=1.0, min_pool=64)
    return workloads.make(name, scale_down=sd, block_size=8)


BS8 = [("tiny8", 1), ("mha", 8), ("gqa16", 8), ("long", 16), ("share_fork", 4)]


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("P", [0, 16, 48])
@pytest.mark.parametrize("name,sd", BS8)
def test_block_size_8_decode_matches_oracle(name, sd, P, path):
    wl = _bs8(name, sd)
    assert wl.bs == 8
    if path == "tensor_cores" and wl.dtype != "bf16":
        pytest.skip("fp32 always runs on CUDA cores")
    pkv.set_decode_path(PATHS[path])
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, partition_size=P)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, f"bs=8 {name} P={P} {path}")
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("P", [0, 16])
@pytest.mark.parametrize("name,sd", BS8)
def test_block_size_8_fused_step(name, sd, P):
    wl = _bs8(name, sd)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, partition_size=P, fused=True)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, f"fused bs=8 {name} P={P}")
    assert pkv.device_errors() == 0


def test_block_size_8_balanced_request_runs_fixed_split():
    """The work-balanced split needs 16-token blocks; with 8-token blocks the fixed split
    runs and the result is still the oracle's."""
    old = pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED)
    try:
        wl = _bs8("gqa16", 8)
        host = workloads.host_tensors(wl)
        dev = device_inputs(wl, host)
        out = gpu_step(wl, dev)
        _, _, ref = oracle_step(wl, host)
        assert_attention_close(widen(out), ref, wl.dtype, "bs=8 balanced request")
    finally:
        pkv.set_decode_split(old)
    assert pkv.device_errors() == 0


def test_block_size_8_bad_block_id_is_flagged_and_read_as_zeros():
    """A table entry outside the pool, in the second half of a stage, is flagged and
    read as zeros; memory stays in bounds."""
    wl = _bs8("gqa16", 8)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    b = int(np.argmax(wl.seq_lens_post))
    bt = wl.block_tables.copy()
    bt[b, 1] = wl.num_blocks + 7  # tokens 8..15 of the sequence's first stage
    dev["block_tables"] = torch.from_numpy(bt).cuda()
    gpu_step(wl, dev)
    torch.cuda.synchronize()
    assert pkv.device_errors() & pkv.DEVERR_BLOCK_ID


def _contiguous_copy(wl, dev, stride):
    """The post-step logical K/V of every sequence laid out as [B, stride, Hkv, D], NaN in
    the rows past each sequence's length."""
    out = []
    for key in ("k_cache", "v_cache"):
        c = torch.full((wl.B, stride, wl.Hkv, wl.D), float("nan"), dtype=dev[key].dtype,
                       device="cuda")
        for b in range(wl.B):
            L = int(wl.seq_lens_post[b])
            n = -(-L // wl.bs)
            ids = torch.from_numpy(wl.block_tables[b, :n].astype(np.int64)).cuda()
            c[b, :L] = dev[key][ids].reshape(n * wl.bs, wl.Hkv, wl.D)[:L]
        out.append(c)
    return out


@pytest.mark.parametrize("P", [0, 64])
@pytest.mark.parametrize("name,sd", [("mha", 8), ("gqa16", 8), ("long", 16), ("share_tails", 4)])
def test_contiguous_control_matches_oracle_and_paged_decode(name, sd, P):
    wl = workloads.make(name, scale_down=sd)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    paged = gpu_step(wl, dev, partition_size=P)  # also applies the step's cache update
    _, _, ref = oracle_step(wl, host)
    stride = wl.max_seq_len + 5
    kc, vc = _contiguous_copy(wl, dev, stride)
    out = torch.full_like(dev["q"], float("nan"))
    n = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len, 16, P)
    ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
    pkv.paged_attention_decode_contiguous(out, dev["q"], kc, vc, dev["seq_lens"], wl.max_seq_len,
                                          wl.scale, workspace=ws, partition_size=P)
    torch.cuda.synchronize()
    assert_attention_close(widen(out), ref, wl.dtype, f"contiguous {name} P={P}")
    if wl.bs == 16:  # same stages in the same order: the same arithmetic
        assert torch.equal(raw(out), raw(paged))
    assert pkv.device_errors() == 0


def test_contiguous_control_rejects_a_short_stride():
    wl = workloads.make("gqa16", scale_down=8)
    dev = device_inputs(wl, workloads.host_tensors(wl))
    kc = torch.zeros((wl.B, wl.max_seq_len - 1, wl.Hkv, wl.D), dtype=torch.bfloat16,
                     device="cuda")
    out = torch.empty_like(dev["q"])
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_decode_contiguous(out, dev["q"], kc, kc, dev["seq_lens"],
                                              wl.max_seq_len, wl.scale,
                                              workspace=workspace_for(wl))
