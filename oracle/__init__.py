"""Paged KV-cache oracle: the plain fp64 CPU definition of what the CUDA path computes.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  It
shares no code with ``paged_kv_cache_344_b200`` and never imports it.

The arithmetic lives in ``pkv_oracle.c`` (see its header for the page passages
each function follows).  This module compiles that file with gcc on first use and
wraps it with NumPy arrays:

* ``calculate_blocks(tokens, block_size)``: ceil division with the example's errors.
* ``kv_write(...)``: byte scatter of new tokens into their slots.
* ``copy_blocks(...)``: whole-block copies for copy-on-write.
* ``paged_decode(...)``: fp64 softmax attention over the block-table-resolved cache.
* ``paged_prefill(...)``: the same for several causal queries per sequence.

Element arrays are NumPy ``uint16`` (bf16 bit patterns) or ``float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_default = None

BF16 = 0
F32 = 1


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile ``src`` (default ``pkv_oracle.c``) into a shared library with gcc; return its path."""
    with _lock:
        stale = (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)
        if force or stale:
            tmp = out + f".tmp{os.getpid()}"
            cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", src, "-o", tmp, "-lm"]
            subprocess.run(cmd, check=True)
            os.replace(tmp, out)
    return out


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle element arrays are uint16 (bf16 bits) or float32, got {a.dtype}")


class Oracle:
    """One loaded build of the oracle library (the default build, or a test's variant)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i64, vp, dp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_double
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_calculate_blocks.argtypes = [i64, i64, ctypes.POINTER(i64)]
        lib.oracle_calculate_blocks.restype = ctypes.c_int
        lib.oracle_kv_write.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, ctypes.c_int]
        lib.oracle_kv_write.restype = i64
        lib.oracle_copy_blocks.argtypes = [vp, vp, vp, i64, i64, i64]
        lib.oracle_copy_blocks.restype = i64
        lib.oracle_paged_decode.argtypes = [vp, vp, vp, vp, ctypes.c_int, vp, i64, vp, i64, i64,
                                            i64, i64, i64, i64, dp, vp, vp, i64]
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_paged_prefill.argtypes = [vp, vp, vp, vp, ctypes.c_int, vp, i64, vp, vp, i64,
                                             i64, i64, i64, i64, i64, dp]
        lib.oracle_paged_prefill.restype = ctypes.c_int
        self.lib = lib

    def num_threads(self) -> int:
        """OpenMP threads the decode uses."""
        return int(self.lib.oracle_num_threads())

    def calculate_blocks(self, token_count: int, block_size: int) -> int:
        """Blocks needed for ``token_count`` cached tokens; ValueError like the page's example."""
        out = ctypes.c_int64(0)
        rc = self.lib.oracle_calculate_blocks(int(token_count), int(block_size), ctypes.byref(out))
        if rc == -1:
            raise ValueError("Token count cannot be negative.")
        if rc == -2:
            raise ValueError("Block size must be positive.")
        return int(out.value)

    def kv_write(self, k, v, k_cache, v_cache, slot_mapping) -> int:
        """Scatter ``k, v [N,Hkv,D]`` into ``k_cache, v_cache [NB,bs,Hkv,D]`` in place.

        Returns the number of out-of-range slots that were skipped.
        """
        slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        N, Hkv, D = k.shape
        NB, bs = k_cache.shape[:2]
        assert k_cache.shape == (NB, bs, Hkv, D) and v_cache.shape == k_cache.shape
        assert k.dtype == v.dtype == k_cache.dtype == v_cache.dtype
        return int(self.lib.oracle_kv_write(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                            _ptr(slot_mapping), N, Hkv, D, bs, NB, _dtype_code(k)))

    def copy_blocks(self, k_cache, v_cache, block_mapping) -> int:
        """Apply (src, dst) whole-block copies to both caches in place; returns skipped pairs."""
        mapping = np.ascontiguousarray(block_mapping, dtype=np.int64).reshape(-1, 2)
        NB = k_cache.shape[0]
        block_bytes = k_cache[0].nbytes
        return int(self.lib.oracle_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(mapping),
                                               mapping.shape[0], block_bytes, NB))

    def paged_decode(self, q, k_cache, v_cache, block_tables, seq_lens, scale, rows=None):
        """fp64 decode attention.  Returns ``[B,Hq,D]`` float64, or ``[len(rows),D]`` when
        ``rows`` (a sequence of (b, h) pairs) selects individual output rows."""
        B, Hq, D = q.shape
        NB, bs, Hkv, D2 = k_cache.shape
        assert D2 == D and v_cache.shape == k_cache.shape
        assert q.dtype == k_cache.dtype == v_cache.dtype
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
        assert bt.shape[0] == B and sl.shape == (B,)
        if rows is None:
            out = np.zeros((B, Hq, D), dtype=np.float64)
            rb = rh = None
            n = 0
        else:
            r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 2))
            rb = np.ascontiguousarray(r[:, 0])
            rh = np.ascontiguousarray(r[:, 1])
            n = r.shape[0]
            out = np.zeros((n, D), dtype=np.float64)
        rc = self.lib.oracle_paged_decode(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _dtype_code(q), _ptr(bt),
            bt.shape[1], _ptr(sl), B, Hq, Hkv, D, bs, NB, float(scale),
            None if rb is None else _ptr(rb), None if rh is None else _ptr(rh), n)
        if rc != 0:
            raise ValueError(f"oracle_paged_decode failed with status {rc}")
        return out


def _prefill(self, q, k_cache, v_cache, block_tables, seq_lens, cu_q, scale):
    """fp64 multi-query attention: ``q [T,Hq,D]`` rows ``cu_q[b] .. cu_q[b+1]-1`` are the
    last queries of sequence b, each attending causally.  Returns ``[T,Hq,D]`` float64."""
    T, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    assert D2 == D and v_cache.shape == k_cache.shape and q.dtype == k_cache.dtype
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    cq = np.ascontiguousarray(cu_q, dtype=np.int32)
    B = sl.shape[0]
    assert cq.shape == (B + 1,) and cq[-1] == T and bt.shape[0] == B
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = self.lib.oracle_paged_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       _dtype_code(q), _ptr(bt), bt.shape[1], _ptr(sl), _ptr(cq),
                                       B, Hq, Hkv, D, bs, NB, float(scale))
    if rc != 0:
        raise ValueError(f"oracle_paged_prefill failed with status {rc}")
    return out


Oracle.paged_prefill = _prefill


def default() -> Oracle:
    """The oracle built from ``pkv_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def calculate_blocks(token_count: int, block_size: int) -> int:
    return default().calculate_blocks(token_count, block_size)


def kv_write(k, v, k_cache, v_cache, slot_mapping) -> int:
    return default().kv_write(k, v, k_cache, v_cache, slot_mapping)


def copy_blocks(k_cache, v_cache, block_mapping) -> int:
    return default().copy_blocks(k_cache, v_cache, block_mapping)


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, rows=None):
    return default().paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, rows)


def paged_prefill(q, k_cache, v_cache, block_tables, seq_lens, cu_q, scale):
    return default().paged_prefill(q, k_cache, v_cache, block_tables, seq_lens, cu_q, scale)
