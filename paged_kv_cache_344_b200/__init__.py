"""B200-native paged KV-cache decode attention.

A thin ctypes binding over the C ABI of ``libpagedkv.so`` (declared in
``include/pagedkv.h``).  Every function here only marshals torch tensors into pointers
and sizes; all work runs in the library's CUDA kernels on the caller's (current) stream.
There is no CPU fallback: if the library is missing, importing the binding's calls
raises.

Calls (same names as the C ABI):

* ``paged_kv_write(k, v, k_cache, v_cache, slot_mapping)``
* ``paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, max_seq_len,
  scale, workspace=None, partition_size=0)``
* ``copy_blocks(k_cache, v_cache, block_mapping)``
* ``paged_attention_decode_workspace_size(...)``, ``paged_attention_decode_partition_size(...)``
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "pagedkv.h")

PKV_OK = 0
PKV_BF16 = 0
PKV_F32 = 1
PKV_PATH_AUTO = 0
PKV_PATH_CUDA_CORES = 1
PKV_PATH_TENSOR_CORES = 2
DEVERR_SLOT = 0x1
DEVERR_SEQLEN = 0x2
DEVERR_BLOCK_ID = 0x4
DEVERR_COPY = 0x8
DEVERR_TIMEOUT = 0x10
DEVERR_PREFIX = 0x20
PKV_ERR_SCRATCH_LIMIT = -6
PKV_SPLIT_FIXED = 0
PKV_SPLIT_BALANCED = 1
PKV_PREFILL_AUTO = 0
PKV_PREFILL_SINGLE_TILE = 1
NOALLOC_SCRATCH_BYTES = 16 << 20  # PKV_NOALLOC_SCRATCH_BYTES

_lib = None


class PagedKVError(RuntimeError):
    """A library call returned a non-zero status."""

    def __init__(self, call: str, status: int):
        lib = _lib
        text = lib.pkv_status_string(status).decode() if lib is not None else str(status)
        extra = ""
        if lib is not None and status == -4:
            extra = f" (cudaError {lib.pkv_last_cuda_error()})"
        super().__init__(f"{call} failed: {text}{extra} [status {status}]")
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded ``libpagedkv.so`` with argument types set (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m paged_kv_cache_344_b200.build` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                             ctypes.c_size_t)
    L.paged_kv_write.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, i32, i64, i32, vp]
    L.paged_kv_write.restype = i32
    L.paged_attention_decode_partition_size.argtypes = [i32, i32, i32, i32, i32]
    L.paged_attention_decode_partition_size.restype = i32
    L.paged_attention_decode_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    L.paged_attention_decode_workspace_size.restype = sz
    L.paged_attention_decode.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32, i32, i32,
                                         i32, i64, f32, i32, i32, vp, sz, vp]
    L.paged_attention_decode.restype = i32
    L.paged_attention_decode_contiguous.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                    i32, f32, i32, i32, vp, sz, vp]
    L.paged_attention_decode_contiguous.restype = i32
    L.paged_attention_prefill_workspace_size.argtypes = [i32, i32, i32, i32]
    L.paged_attention_prefill_workspace_size.restype = sz
    L.paged_attention_prefill.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                          i32, i32, i32, i32, i64, f32, i32, vp, sz, vp]
    L.paged_attention_prefill.restype = i32
    L.paged_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, i32, i32,
                                    i32, i32, i64, f32, i32, i32, vp, sz, vp]
    L.paged_decode_step.restype = i32
    L.paged_decode_step_shared_prefix.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32,
                                                  vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                                  i64, f32, i32, i32, vp, sz, vp]
    L.paged_decode_step_shared_prefix.restype = i32
    L.paged_attention_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, i32,
                                                 i32, i32, i32, i64, f32, i32, i32, vp]
    L.paged_attention_decode_noalloc.restype = i32
    L.paged_attention_decode_shared_prefix.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, vp, vp,
                                                       i32, i32, i32, i32, i32, i32, i32, i64,
                                                       f32, i32, i32, vp, sz, vp]
    L.paged_attention_decode_shared_prefix.restype = i32
    L.paged_attention_decode_shared_prefix_workspace_size.argtypes = [i32] * 7
    L.paged_attention_decode_shared_prefix_workspace_size.restype = sz
    L.copy_blocks.argtypes = [vp, vp, vp, i64, i64, i64, vp]
    L.copy_blocks.restype = i32
    L.pkv_status_string.argtypes = [i32]
    L.pkv_status_string.restype = ctypes.c_char_p
    L.pkv_last_cuda_error.restype = i32
    L.pkv_device_errors.argtypes = [ctypes.POINTER(ctypes.c_uint32), i32]
    L.pkv_device_errors.restype = i32
    L.pkv_set_prefill_path.argtypes = [i32]
    L.pkv_set_prefill_path.restype = i32
    L.pkv_set_decode_path.argtypes = [i32]
    L.pkv_set_decode_path.restype = i32
    L.pkv_set_launch_overlap.argtypes = [i32]
    L.pkv_set_launch_overlap.restype = i32
    L.pkv_debug_stalled_wait.argtypes = [ctypes.c_void_p]
    L.pkv_debug_stalled_wait.restype = i32
    L.pkv_set_decode_split.argtypes = [i32]
    L.pkv_set_decode_split.restype = i32
    L.pkv_set_decode_ctas.argtypes = [i32]
    L.pkv_set_decode_ctas.restype = i32
    _lib = L
    return L


def declared_functions() -> list[str]:
    """Names of the functions ``include/pagedkv.h`` declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def _check(call: str, status: int) -> None:
    if status != PKV_OK:
        raise PagedKVError(call, status)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return PKV_BF16
    if t.dtype == torch.float32:
        return PKV_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _stream(t, stream):
    import torch
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def paged_kv_write(k, v, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Scatter ``k, v [N,Hkv,D]`` into ``k_cache, v_cache [NB,bs,Hkv,D]`` at ``slot_mapping``."""
    N, Hkv, D = k.shape
    NB, bs = k_cache.shape[0], k_cache.shape[1]
    _check("paged_kv_write", lib().paged_kv_write(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), N, Hkv, D, bs, NB,
        _dtype_code(k), _stream(k, stream)))


def paged_attention_decode_partition_size(B, Hkv, max_seq_len, block_size, partition_size=0):
    r = lib().paged_attention_decode_partition_size(B, Hkv, max_seq_len, block_size,
                                                    partition_size)
    _check("paged_attention_decode_partition_size", min(r, 0))
    return r


def paged_attention_decode_workspace_size(B, Hq, Hkv, D, max_seq_len, block_size,
                                          partition_size=0) -> int:
    return int(lib().paged_attention_decode_workspace_size(B, Hq, Hkv, D, max_seq_len,
                                                           block_size, partition_size))


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, seq_lens, max_seq_len, scale,
                           workspace=None, partition_size=0, stream=None) -> None:
    """``out[B,Hq,D] = softmax(scale * q K^T) V`` over the block-paged cache."""
    B, Hq, D = q.shape
    NB, bs, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("paged_attention_decode", lib().paged_attention_decode(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), int(max_seq_len), B, Hq, Hkv, D, bs, NB,
        float(scale), _dtype_code(q), int(partition_size), _ptr(workspace), ws_bytes,
        _stream(q, stream)))


def paged_attention_decode_contiguous(out, q, k_cache, v_cache, seq_lens, max_seq_len, scale,
                                      workspace=None, partition_size=0, stream=None) -> None:
    """The decode over an unpaged cache ``k_cache, v_cache [B, row_stride, Hkv, D]`` (the
    paging-overhead control: the same kernel without the block-table walk)."""
    B, Hq, D = q.shape
    stride, Hkv = k_cache.shape[1], k_cache.shape[2]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("paged_attention_decode_contiguous", lib().paged_attention_decode_contiguous(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), int(max_seq_len),
        stride, B, Hq, Hkv, D, float(scale), _dtype_code(q), int(partition_size),
        _ptr(workspace), ws_bytes, _stream(q, stream)))


def paged_attention_prefill_workspace_size(B, Hq, Hkv, max_q_len) -> int:
    """Bytes of the scratch that lets paged_attention_prefill schedule its work longest first."""
    return int(lib().paged_attention_prefill_workspace_size(B, Hq, Hkv, int(max_q_len)))


def paged_attention_prefill(out, q, k_cache, v_cache, block_tables, seq_lens, cu_q, max_q_len,
                            max_seq_len, scale, workspace=None, stream=None) -> None:
    """Causal multi-query attention: rows ``cu_q[b] .. cu_q[b+1]-1`` of ``q [T,Hq,D]`` are the
    last queries of sequence b (tcgen05 tensor cores).  ``workspace`` (a device tensor of at
    least ``paged_attention_prefill_workspace_size`` bytes, or None) enables the persistent,
    longest-first schedule."""
    T, Hq, D = q.shape
    NB, bs, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("paged_attention_prefill", lib().paged_attention_prefill(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), _ptr(cu_q), T, int(max_q_len), int(max_seq_len),
        seq_lens.shape[0], Hq, Hkv, D, bs, NB, float(scale), _dtype_code(q), _ptr(workspace),
        ws_bytes, _stream(q, stream)))


def paged_decode_step(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens,
                      max_seq_len, scale, cow_src=None, workspace=None, partition_size=0,
                      stream=None) -> None:
    """One decode step in one launch: optional copy-on-write of each sequence's last block
    (``cow_src[b]``), cache write of its new token (position ``seq_lens[b] - 1``), decode."""
    B, Hq, D = q.shape
    NB, bs, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("paged_decode_step", lib().paged_decode_step(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), _ptr(cow_src),
        int(max_seq_len), B, Hq, Hkv, D, bs, NB, float(scale), _dtype_code(q),
        int(partition_size), _ptr(workspace), ws_bytes, _stream(q, stream)))


def paged_decode_step_shared_prefix(out, q, k_new, v_new, k_cache, v_cache, block_tables,
                                    seq_lens, max_seq_len, scale, group_offsets, prefix_lens,
                                    max_group_size, cow_src=None, workspace=None,
                                    partition_size=0, stream=None) -> None:
    """paged_decode_step for grouped batches: copy-on-write, cache write and the
    shared-prefix decode in one launch."""
    B, Hq, D = q.shape
    NB, bs, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("paged_decode_step_shared_prefix", lib().paged_decode_step_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
        _ptr(block_tables), block_tables.shape[1], _ptr(seq_lens), _ptr(cow_src),
        int(max_seq_len), _ptr(group_offsets), _ptr(prefix_lens), prefix_lens.shape[0],
        int(max_group_size), B, Hq, Hkv, D, bs, NB, float(scale), _dtype_code(q),
        int(partition_size), _ptr(workspace), ws_bytes, _stream(q, stream)))


def paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, seq_lens, max_seq_len,
                                   scale, partition_size=0, stream=None) -> None:
    """The decode without a workspace argument, for callers that cannot allocate device
    memory: its split-partition scratch is a fixed array inside the library (see
    ``include/pagedkv.h``).  Calls that overlap on the GPU race on that array."""
    B, Hq, D = q.shape
    NB, bs, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    _check("paged_attention_decode_noalloc", lib().paged_attention_decode_noalloc(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), int(max_seq_len), B, Hq, Hkv, D, bs, NB,
        float(scale), _dtype_code(q), int(partition_size), _stream(q, stream)))


def paged_attention_decode_shared_prefix_workspace_size(B, Hq, Hkv, D, max_seq_len, block_size,
                                                        partition_size=0) -> int:
    return int(lib().paged_attention_decode_shared_prefix_workspace_size(
        B, Hq, Hkv, D, max_seq_len, block_size, partition_size))


def paged_attention_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, seq_lens,
                                         max_seq_len, scale, group_offsets, prefix_lens,
                                         max_group_size, workspace=None, partition_size=0,
                                         stream=None) -> None:
    """The decode for batches whose consecutive sequences share prefix blocks: group g is
    sequences ``group_offsets[g] .. group_offsets[g+1]-1`` sharing ``prefix_lens[g]``
    leading tokens; shared blocks are read once per group."""
    B, Hq, D = q.shape
    NB, bs, Hkv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("paged_attention_decode_shared_prefix", lib().paged_attention_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(seq_lens), int(max_seq_len), _ptr(group_offsets),
        _ptr(prefix_lens), prefix_lens.shape[0], int(max_group_size), B, Hq, Hkv, D, bs, NB,
        float(scale), _dtype_code(q), int(partition_size), _ptr(workspace), ws_bytes,
        _stream(q, stream)))


def copy_blocks(k_cache, v_cache, block_mapping, stream=None) -> None:
    """Copy whole blocks ``block_mapping[i] = (src, dst)`` in both caches."""
    P = block_mapping.shape[0]
    block_bytes = k_cache[0].numel() * k_cache.element_size()
    _check("copy_blocks", lib().copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_mapping), P,
                                            block_bytes, k_cache.shape[0],
                                            _stream(k_cache, stream)))


def device_errors(clear: bool = True) -> int:
    """The OR of device error bits since the last clear (synchronises)."""
    bits = ctypes.c_uint32(0)
    _check("pkv_device_errors", lib().pkv_device_errors(ctypes.byref(bits), int(clear)))
    return int(bits.value)


def debug_stalled_wait(stream=None) -> None:
    """Launch the time-limit self-test: one bounded wait that nothing satisfies gives up
    after about half a second and sets DEVERR_TIMEOUT (which stops later attention
    launches until device_errors(clear=True))."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    _check("pkv_debug_stalled_wait", lib().pkv_debug_stalled_wait(
        ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))))


def set_decode_path(mode: int) -> int:
    """Select CUDA-core / tensor-core decode kernels process-wide; returns the old mode."""
    r = lib().pkv_set_decode_path(int(mode))
    _check("pkv_set_decode_path", min(r, 0))
    return r


def set_launch_overlap(enabled: bool) -> bool:
    """Launch kernels with programmatic stream serialization (default) or in plain
    stream order, process-wide; returns the old setting."""
    r = lib().pkv_set_launch_overlap(1 if enabled else 0)
    _check("pkv_set_launch_overlap", min(r, 0))
    return bool(r)


def set_prefill_path(mode: int) -> int:
    """Two-tile warp-specialised (auto) or single-tile prefill kernel; returns the old mode."""
    r = lib().pkv_set_prefill_path(int(mode))
    _check("pkv_set_prefill_path", min(r, 0))
    return r


def set_decode_ctas(ctas: int) -> int:
    """CTA count of the work-balanced decode (0 = as many as are resident); returns the old."""
    r = lib().pkv_set_decode_ctas(int(ctas))
    _check("pkv_set_decode_ctas", min(r, 0))
    return r


def set_decode_split(mode: int) -> int:
    """Fixed-length partitions (default) or the work-balanced split; returns the old mode."""
    r = lib().pkv_set_decode_split(int(mode))
    _check("pkv_set_decode_split", min(r, 0))
    return r
