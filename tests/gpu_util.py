"""Helpers for the GPU parity tests: move seeded inputs to the device, run one decode step
through the CUDA library, run the same step through the oracle, and compare.

Tolerances (from the method's statement of the target): bf16 inputs/outputs with fp32
accumulation must satisfy max|gpu - oracle| <= 1e-2 + 1e-2*|oracle| elementwise; the fp32
config 1e-5 + 1e-5*|oracle|.  Cache writes and block copies must be bit-exact.
"""
import numpy as np
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads

TOL = {"bf16": (1e-2, 1e-2), "f32": (1e-5, 1e-5)}


def to_device(a: np.ndarray, dtype: str, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.to(device)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> NumPy array of the oracle's element kind (bf16 bits or float32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def raw(t: torch.Tensor) -> torch.Tensor:
    """Bit view for exact comparisons (NaN-safe)."""
    return t.view(torch.int16) if t.element_size() == 2 else t.view(torch.int32)


def device_inputs(wl, host):
    dev = {k: to_device(v, wl.dtype) for k, v in host.items()}
    dev.update(meta_to_device(wl))
    return dev


def meta_to_device(wl, device="cuda"):
    return {
        "block_tables": torch.from_numpy(wl.block_tables).to(device),
        "seq_lens": torch.from_numpy(wl.seq_lens_post).to(device),
        "slot_mapping": torch.from_numpy(wl.slot_mapping).to(device),
        "cow_pairs": torch.from_numpy(wl.cow_pairs).to(device),
    }


def workspace_for(wl, partition_size=0, device="cuda"):
    n = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len,
                                                  wl.bs, partition_size)
    return torch.zeros(max(n, 1), dtype=torch.uint8, device=device) if n else None


def gpu_step(wl, dev, partition_size=0, workspace=None, max_seq_len=None, stream=None,
             shared=False, fused=False):
    """copy_blocks -> paged_kv_write -> paged_attention_decode (or, with ``shared``, the
    shared-prefix decode over the workload's groups; with ``fused``, paged_decode_step:
    all three in one launch) on the device; returns out."""
    if fused and shared:
        out = torch.empty_like(dev["q"])
        msl = max_seq_len or wl.max_seq_len
        n = pkv.paged_attention_decode_shared_prefix_workspace_size(
            wl.B, wl.Hq, wl.Hkv, wl.D, msl, wl.bs, partition_size)
        ws = torch.zeros(max(n, 1), dtype=torch.uint8, device=dev["q"].device)
        cow = torch.from_numpy(wl.cow_src).to(dev["q"].device) if len(wl.cow_pairs) else None
        pkv.paged_decode_step_shared_prefix(
            out, dev["q"], dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
            dev["block_tables"], dev["seq_lens"], msl, wl.scale,
            torch.from_numpy(wl.group_offsets).to(dev["q"].device),
            torch.from_numpy(wl.prefix_lens).to(dev["q"].device),
            int(np.diff(wl.group_offsets).max()), cow_src=cow, workspace=ws,
            partition_size=partition_size, stream=stream)
        return out
    if fused:
        out = torch.empty_like(dev["q"])
        if workspace is None:
            workspace = workspace_for(wl, partition_size)
        cow = torch.from_numpy(wl.cow_src).to(dev["q"].device) if len(wl.cow_pairs) else None
        pkv.paged_decode_step(out, dev["q"], dev["k_new"], dev["v_new"], dev["k_cache"],
                              dev["v_cache"], dev["block_tables"], dev["seq_lens"],
                              max_seq_len or wl.max_seq_len, wl.scale, cow_src=cow,
                              workspace=workspace, partition_size=partition_size, stream=stream)
        return out
    if len(wl.cow_pairs):
        pkv.copy_blocks(dev["k_cache"], dev["v_cache"], dev["cow_pairs"], stream=stream)
    pkv.paged_kv_write(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
                       dev["slot_mapping"], stream=stream)
    out = torch.empty_like(dev["q"])
    if shared:
        msl = max_seq_len or wl.max_seq_len
        n = pkv.paged_attention_decode_shared_prefix_workspace_size(
            wl.B, wl.Hq, wl.Hkv, wl.D, msl, wl.bs, partition_size)
        ws = torch.zeros(max(n, 1), dtype=torch.uint8, device=dev["q"].device)
        pkv.paged_attention_decode_shared_prefix(
            out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"], dev["seq_lens"],
            msl, wl.scale, torch.from_numpy(wl.group_offsets).to(dev["q"].device),
            torch.from_numpy(wl.prefix_lens).to(dev["q"].device),
            int(np.diff(wl.group_offsets).max()), workspace=ws, partition_size=partition_size,
            stream=stream)
        return out
    if workspace is None:
        workspace = workspace_for(wl, partition_size)
    pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"],
                               dev["seq_lens"], max_seq_len or wl.max_seq_len, wl.scale,
                               workspace=workspace, partition_size=partition_size, stream=stream)
    return out


def oracle_step(wl, host):
    """The same step in the oracle on host copies; returns (k_cache, v_cache, out fp64)."""
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    if len(wl.cow_pairs):
        assert oracle.copy_blocks(kc, vc, wl.cow_pairs) == 0
    assert oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping) == 0
    out = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, wl.seq_lens_post, wl.scale)
    return kc, vc, out


def widen(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_attention_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what=""):
    atol, rtol = TOL[dtype]
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} elements out of tolerance; worst at {i}: "
                             f"gpu={gpu[i]!r} oracle={ref[i]!r} err={err[i]:.3e} bound={bound[i]:.3e}")
    return float(err.max()) if err.size else 0.0
