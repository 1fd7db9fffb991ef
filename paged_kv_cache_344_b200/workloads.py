"""Seeded synthetic decode-step workloads shared by the tests, the smoke check and the benchmark.

This module only *builds inputs*: physical block pools, block tables, slot mappings,
copy-on-write pairs and random q/K/V.  It holds none of the attention arithmetic, imports
neither the CUDA binding nor the oracle, and both sides consume what it produces.

Structure follows the pages' description of a paged cache:

* fixed-size blocks handed out from a pool in scattered order, mapped per sequence by a
  block table ("Paged Attention Explained", Steps 1-3);
* a new block is taken only when the current last block is full (the same page's Step 2,
  and "PagedAttention and KV Cache Compression", 5. Real-World Consequences);
* physical blocks shared between branches with copy-on-write of a shared block that must
  be modified ("PagedAttention: paging the KV cache like an OS pages memory", How it works).

Step semantics (a reading, stated in the design notes): ``seq_lens_pre[b]`` tokens are
cached before the step; the step copies shared blocks that are about to be written,
writes token ``seq_lens_pre[b]`` of every sequence into ``slot_mapping[b]``, and decodes
with ``seq_lens_post = seq_lens_pre + 1``.  Slots that hold no token (tails of partially
filled blocks, free blocks) are filled with NaN so that a kernel that reads them is caught.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BF16_NAN_BITS = 0x7FC0


@dataclass
class Workload:
    name: str
    dtype: str  # "bf16" or "f32"
    B: int
    Hq: int
    Hkv: int
    D: int
    bs: int
    num_blocks: int
    seq_lens_pre: np.ndarray  # int32 [B]
    block_tables_pre: np.ndarray  # int32 [B, MB], -1 padded (state before the step)
    block_tables: np.ndarray  # int32 [B, MB], -1 padded (after CoW + allocation)
    slot_mapping: np.ndarray  # int64 [B]
    cow_pairs: np.ndarray  # int64 [P, 2] (src, dst)
    seed: int
    scale: float = field(default=0.0)
    valid_pre: np.ndarray = field(default=None, repr=False)  # bool [NB, bs]: slot holds a token
    # Groups of consecutive sequences whose first prefix_lens[g] tokens sit in the same
    # physical blocks after the step (whole shared blocks; one-member groups share nothing).
    group_offsets: np.ndarray = field(default=None, repr=False)  # int32 [n_groups + 1]
    prefix_lens: np.ndarray = field(default=None, repr=False)  # int32 [n_groups]

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_blocks(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def seq_lens_post(self) -> np.ndarray:
        return (self.seq_lens_pre + 1).astype(np.int32)

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens_post.max()) if self.B else 0

    @property
    def cow_src(self) -> np.ndarray:
        """Per sequence: the block copied into its new token's block this step, else -1."""
        src = np.full(self.B, -1, dtype=np.int32)
        by_dst = {int(d): int(s_) for s_, d in self.cow_pairs}
        for b in range(self.B):
            if self.slot_mapping[b] >= 0:
                dst = int(self.slot_mapping[b]) // self.bs
                if dst in by_dst:
                    src[b] = by_dst[dst]
        return src

    @property
    def elt(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def block_bytes(self) -> int:
        """Bytes of one physical block of one cache (K or V)."""
        return self.bs * self.Hkv * self.D * self.elt


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _build(name, dtype, B, Hq, Hkv, D, bs, seq_lens_pre, seed, rng, pool_factor=1.25,
           min_pool=0, groups=None, shared_tokens=None, contiguous=False):
    """Assign physical blocks for every sequence from a shuffled pool (``contiguous``: in
    pool order, so each sequence's blocks are consecutive, as in a contiguous cache).

    ``groups`` (optional) lists, per sequence, a group id; sequences of one group share the
    physical blocks of their first ``shared_tokens[group]`` tokens (refcount = group size).
    """
    seq_lens_pre = np.asarray(seq_lens_pre, dtype=np.int32)
    post = seq_lens_pre.astype(np.int64) + 1
    need_post = np.array([_ceil_div(int(n), bs) for n in post], dtype=np.int64)

    # Blocks needed in the pool: unique shared blocks + private blocks + CoW destinations.
    if groups is None:
        groups = np.arange(B)
        shared_tokens = np.zeros(B, dtype=np.int64)
    groups = np.asarray(groups)
    shared_tokens = np.asarray(shared_tokens, dtype=np.int64)
    n_shared = np.array([_ceil_div(int(t), bs) for t in shared_tokens], dtype=np.int64)
    unique_need = int(n_shared.sum())
    for b in range(B):
        unique_need += int(need_post[b] - n_shared[groups[b]]) + 1  # +1: a possible CoW copy
    num_blocks = max(int(math.ceil(pool_factor * unique_need)), min_pool, 1)
    perm = rng.permutation(num_blocks).astype(np.int64)
    if contiguous:
        perm = np.arange(num_blocks, dtype=np.int64)
    cursor = 0

    def take(n):
        nonlocal cursor
        ids = perm[cursor:cursor + n]
        cursor += n
        assert len(ids) == n, "pool exhausted"
        return ids

    MB = int(max(need_post.max(), 1))
    bt_pre = np.full((B, MB), -1, dtype=np.int32)
    bt = np.full((B, MB), -1, dtype=np.int32)
    slot = np.zeros(B, dtype=np.int64)
    cow = []
    valid = np.zeros((num_blocks, bs), dtype=bool)

    shared_ids = {}
    for g in np.unique(groups):
        shared_ids[int(g)] = take(int(n_shared[g]))
    refcount = {}
    for b in range(B):
        for pid in shared_ids[int(groups[b])]:
            refcount[int(pid)] = refcount.get(int(pid), 0) + 1
    # Remember the holder that writes in place: the last sequence of a group keeps the block.
    last_holder = {}
    for b in range(B):
        last_holder[int(groups[b])] = b

    for b in range(B):
        L = int(seq_lens_pre[b])
        g = int(groups[b])
        have = shared_ids[g]
        n_pre = _ceil_div(L, bs)
        assert len(have) <= n_pre or L == 0 or int(shared_tokens[g]) <= L
        private = take(max(n_pre - len(have), 0))
        ids_pre = np.concatenate([have, private])[:n_pre] if n_pre else np.zeros(0, np.int64)
        bt_pre[b, :n_pre] = ids_pre
        for t in range(L):
            valid[ids_pre[t // bs], t % bs] = True
        ids = list(ids_pre)
        # The new token goes to logical block L // bs at offset L % bs.
        lb, off = L // bs, L % bs
        if lb == len(ids):  # current block full (or none yet): allocate on demand
            ids.append(int(take(1)[0]))
        else:
            pid = int(ids[lb])
            if refcount.get(pid, 1) > 1 and b != last_holder[g]:
                fresh = int(take(1)[0])
                cow.append((pid, fresh))
                refcount[pid] -= 1
                ids[lb] = fresh
        bt[b, :len(ids)] = ids
        slot[b] = int(ids[lb]) * bs + off

    # Group table: runs of equal group ids; the prefix is the whole blocks still shared
    # by every member after the step (a partially filled shared block is copied on write).
    starts = [0] + [b for b in range(1, B) if groups[b] != groups[b - 1]]
    offsets = np.array(starts + [B], dtype=np.int32)
    plens = []
    for i, b in enumerate(starts):
        g = int(groups[b])
        members = range(b, int(offsets[i + 1]))
        n_full = int(shared_tokens[g]) // bs if len(members) > 1 else 0
        while n_full > 0 and len({int(bt[m, n_full - 1]) for m in members}) != 1:
            n_full -= 1
        plens.append(n_full * bs)
    wl = Workload(name=name, dtype=dtype, B=B, Hq=Hq, Hkv=Hkv, D=D, bs=bs, num_blocks=num_blocks,
                  seq_lens_pre=seq_lens_pre, block_tables_pre=bt_pre, block_tables=bt,
                  slot_mapping=slot, cow_pairs=np.asarray(cow, dtype=np.int64).reshape(-1, 2),
                  seed=seed, valid_pre=valid, group_offsets=offsets,
                  prefix_lens=np.asarray(plens, dtype=np.int32))
    wl.scale = float(np.float32(1.0 / math.sqrt(D)))
    return wl


# Config index -> seed offset (seed = 1000 + index), matching the five workloads of the
# benchmark definition: tiny fp32, MHA, GQA, long-context GQA, shared-prefix.
CONFIG_INDEX = {"tiny": 0, "tiny_post": 0, "mha": 1, "gqa16": 2, "gqa32": 2, "long": 3,
                "share_fork": 4, "share_tails": 4}


def make(name: str, seed: int | None = None, scale_down: int = 1, block_size: int | None = None,
         contiguous: bool = False, dtype: str | None = None) -> Workload:
    """Build a named workload.

    Full-size names: ``tiny`` (lengths are pre-step), ``tiny_post`` (lengths include the
    new token), ``mha``, ``gqa16``, ``gqa32``, ``long``, ``share_fork``, ``share_tails``.
    ``scale_down > 1`` divides the batch and the lengths for fast parity tests while keeping
    the head shapes, block size and length distribution.  ``block_size`` overrides the
    workload's block size; ``contiguous`` lays every sequence's blocks out consecutively
    (a contiguous-cache control for the cost of the scattered placement); ``dtype`` ("bf16"
    or "f32") overrides the element type of the bf16 workloads.
    """
    kw = {"contiguous": contiguous}
    if seed is None:
        seed = 1000 + CONFIG_INDEX[name]
    rng = np.random.default_rng(seed)
    s = max(int(scale_down), 1)
    if name in ("tiny", "tiny_post"):
        L = np.array([1, 7, 16, 33], dtype=np.int32)
        if name == "tiny_post":
            L = L - 1
        return _build(name, "f32", 4, 4, 4, 64, 16, L, seed, rng, pool_factor=1.0, min_pool=32)
    if name == "mha":
        B = max(64 // s, 2)
        L = rng.integers(128 // s, 2048 // s + 1, size=B)
        return _build(name, dtype or "bf16", B, 40, 40, 128, block_size or 16, L, seed, rng, **kw)
    if name in ("gqa16", "gqa32"):
        bs = block_size or (16 if name == "gqa16" else 32)
        B = max(256 // s, 2)
        z = rng.standard_normal(B)
        L = np.clip(np.round(np.exp(math.log(1024) + 0.8 * z)), 16, 4096).astype(np.int64) // s
        L = np.maximum(L, 1)
        return _build(name, dtype or "bf16", B, 32, 8, 128, bs, L, seed, rng, **kw)
    if name == "long":
        B = max(8 // s, 1)
        L = rng.integers(32768 // s, 131072 // s + 1, size=B)
        return _build(name, dtype or "bf16", B, 64, 8, 128, block_size or 16, L, seed, rng, **kw)
    if name in ("share_fork", "share_tails"):
        n_groups, branches = max(32 // s, 1), 4
        B = n_groups * branches
        groups = np.repeat(np.arange(n_groups), branches)
        prefix = 1024 // s
        if name == "share_fork":
            r = rng.integers(1, 16, size=n_groups)  # shared, partially filled last block
            shared = prefix + r
            L = shared[groups]
        else:
            shared = np.full(n_groups, prefix)
            L = prefix + rng.integers(0, 256 // s + 1, size=B)
        return _build(name, "bf16", B, 32, 8, 128, block_size or 16, L, seed, rng,
                      groups=groups, shared_tokens=shared)
    raise KeyError(name)


def custom(name, dtype, B, Hq, Hkv, D, bs, seq_lens_pre, seed, pool_factor=1.25, min_pool=0):
    """A workload with explicit shapes and pre-step lengths (private blocks only)."""
    rng = np.random.default_rng(seed)
    return _build(name, dtype, B, Hq, Hkv, D, bs, np.asarray(seq_lens_pre), seed, rng,
                  pool_factor=pool_factor, min_pool=min_pool)


def grouped(name, dtype, Hq, Hkv, D, bs, group_sizes, shared_tokens, tails, seed,
            pool_factor=1.25):
    """Groups of consecutive sequences that share a prefix of ``shared_tokens[g]`` tokens
    (same physical blocks), each member followed by ``tails[b]`` tokens of its own.  A prefix
    that ends inside a block is a fork: its members hold no tokens of their own yet, they
    share the partly filled block, and the step copies it on write for all but its last
    holder."""
    rng = np.random.default_rng(seed)
    groups = np.repeat(np.arange(len(group_sizes)), group_sizes)
    shared = np.asarray(shared_tokens, dtype=np.int64)
    own = np.asarray(tails, dtype=np.int64)
    # Members write their own tokens after the prefix, so a prefix that ends inside a
    # block leaves them none.
    fork = (shared % bs != 0)[groups]
    assert np.all(own[fork] == 0), "a prefix ending inside a block is a fork: no own tokens"
    L = shared[groups] + own
    return _build(name, dtype, len(groups), Hq, Hkv, D, bs, L, seed, rng,
                  pool_factor=pool_factor, groups=groups, shared_tokens=shared)


def prefill(seed: int = 1005, B: int = 16, chunk: int = 512, max_ctx: int = 4096, Hq: int = 32,
            Hkv: int = 8, D: int = 128, bs: int = 16):
    """A chunked-append batch: sequence b has ctx_b ~ U{0..max_ctx} cached tokens followed by
    ``chunk`` new query tokens (already in the cache).  Returns (workload, cu_q) where the
    workload's ``seq_lens_pre`` are the full lengths ctx_b + chunk."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(0, max_ctx + 1, size=B)
    wl = custom("prefill", "bf16", B, Hq, Hkv, D, bs, ctx + chunk, seed)
    cu_q = (np.arange(B + 1) * chunk).astype(np.int32)
    return wl, cu_q


def prefill_flops(wl: Workload, cu_q: np.ndarray) -> int:
    """Multiply-add flops of causal multi-query attention: 4 D per (query row, visible token)."""
    total = 0
    for b in range(wl.B):
        L, Q = int(wl.seq_lens_pre[b]), int(cu_q[b + 1] - cu_q[b])
        vis = (L - Q) * Q + Q * (Q + 1) // 2
        total += 4 * wl.D * wl.Hq * vis
    return int(total)


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def host_tensors(wl: Workload, seed_offset: int = 0) -> dict:
    """q, the step's new k/v and the pre-step caches as NumPy arrays (uint16 bf16 bits or
    float32).  Cache slots that hold no token are NaN."""
    rng = np.random.default_rng(wl.seed * 7919 + 17 + seed_offset)
    NB, bs, Hkv, D = wl.num_blocks, wl.bs, wl.Hkv, wl.D
    f = {
        "q": rng.standard_normal((wl.B, wl.Hq, D), dtype=np.float32),
        "k_new": rng.standard_normal((wl.B, Hkv, D), dtype=np.float32),
        "v_new": rng.standard_normal((wl.B, Hkv, D), dtype=np.float32),
        "k_cache": rng.standard_normal((NB, bs, Hkv, D), dtype=np.float32),
        "v_cache": rng.standard_normal((NB, bs, Hkv, D), dtype=np.float32),
    }
    invalid = ~wl.valid_pre
    for key in ("k_cache", "v_cache"):
        f[key][invalid] = np.nan
    if wl.dtype == "bf16":
        f = {k: _to_bf16_bits(v) for k, v in f.items()}
    return f


def device_tensors(wl: Workload, device, seed_offset: int = 0) -> dict:
    """The same kinds of tensors generated directly on ``device`` with torch's seeded
    generator (for full-size pools that do not fit comfortably in host memory).
    Returns torch tensors (bfloat16 or float32)."""
    import torch
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    gen = torch.Generator(device=device)
    gen.manual_seed(wl.seed * 7919 + 17 + seed_offset)
    NB, bs, Hkv, D = wl.num_blocks, wl.bs, wl.Hkv, wl.D

    def randn(shape):
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(tdt)

    out = {"q": randn((wl.B, wl.Hq, D)), "k_new": randn((wl.B, Hkv, D)),
           "v_new": randn((wl.B, Hkv, D))}
    invalid = torch.from_numpy(~wl.valid_pre).to(device)
    chunk = max(1, (1 << 27) // (bs * Hkv * D))
    for key in ("k_cache", "v_cache"):
        c = torch.empty((NB, bs, Hkv, D), dtype=tdt, device=device)
        for i in range(0, NB, chunk):
            j = min(NB, i + chunk)
            c[i:j] = randn((j - i, bs, Hkv, D))
        c[invalid] = float("nan")
        out[key] = c
    return out


def valid_post(wl: Workload) -> np.ndarray:
    """bool [NB, bs]: the slots that hold a token after the step (the pre-step tokens and
    every sequence's new token)."""
    v = wl.valid_pre.copy()
    for s_ in wl.slot_mapping:
        if s_ >= 0:
            v[int(s_) // wl.bs, int(s_) % wl.bs] = True
    return v


def compact_sample(wl: Workload, n_seq: int, k_cache=None, v_cache=None, seed_offset: int = 0):
    """The post-step decode inputs of sequences 0..n_seq-1 over a compact pool holding only
    the blocks they use (a shared block once), with their block tables renumbered.

    With ``k_cache``/``v_cache`` (torch tensors of the full pool, e.g. on the device after
    the step), the blocks are gathered from them; otherwise they are drawn here (seeded
    N(0,1), NaN in slots that hold no token).  Returns NumPy arrays (uint16 bf16 bits or
    float32): q (drawn here unless the caller overrides it), k_cache, v_cache,
    block_tables, seq_lens."""
    n_seq = max(1, min(int(n_seq), wl.B))
    lens = wl.seq_lens_post[:n_seq]
    ids, remap = [], {}
    tables = np.full((n_seq, max(1, max(_ceil_div(int(L), wl.bs) for L in lens))), -1, np.int32)
    for b in range(n_seq):
        for j in range(_ceil_div(int(lens[b]), wl.bs)):
            pid = int(wl.block_tables[b, j])
            if pid not in remap:
                remap[pid] = len(ids)
                ids.append(pid)
            tables[b, j] = remap[pid]
    ids = np.asarray(ids, dtype=np.int64)
    rng = np.random.default_rng(wl.seed * 7919 + 29 + seed_offset)
    shape = (len(ids), wl.bs, wl.Hkv, wl.D)
    if k_cache is not None:
        import torch
        sel = torch.from_numpy(ids).to(k_cache.device)
        out = {}
        for key, c in (("k_cache", k_cache), ("v_cache", v_cache)):
            t = c.index_select(0, sel).cpu().contiguous()
            out[key] = t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 \
                else t.numpy()
    else:
        invalid = ~valid_post(wl)[ids]
        out = {}
        for key in ("k_cache", "v_cache"):
            x = rng.standard_normal(shape, dtype=np.float32)
            x[invalid] = np.nan
            out[key] = _to_bf16_bits(x) if wl.dtype == "bf16" else x
    q = rng.standard_normal((n_seq, wl.Hq, wl.D), dtype=np.float32)
    out["q"] = _to_bf16_bits(q) if wl.dtype == "bf16" else q
    out["block_tables"] = tables
    out["seq_lens"] = np.ascontiguousarray(lens, dtype=np.int32)
    return out


def unique_blocks_touched(wl: Workload) -> int:
    """Distinct physical blocks the decode reads (shared blocks count once)."""
    ids = set()
    for b in range(wl.B):
        n = _ceil_div(int(wl.seq_lens_post[b]), wl.bs)
        ids.update(int(x) for x in wl.block_tables[b, :n])
    return len(ids)


def decode_algorithmic_bytes(wl: Workload) -> int:
    """Bytes one decode call must move at minimum: each distinct K and V block touched once,
    q and out once, the used block-table entries and the lengths (one attention layer of the
    page's per-request cache formula, summed over the batch)."""
    kv = unique_blocks_touched(wl) * wl.block_bytes * 2
    qo = 2 * wl.B * wl.Hq * wl.D * wl.elt
    tables = sum(_ceil_div(int(n), wl.bs) for n in wl.seq_lens_post) * 4
    return int(kv + qo + tables + 4 * wl.B)


def decode_token_bytes(wl: Workload) -> int:
    """Like ``decode_algorithmic_bytes`` but counting only the cached tokens themselves (no
    unused slots of the last blocks; shared tokens once per group)."""
    row = wl.Hkv * wl.D * wl.elt * 2
    tokens = int(wl.seq_lens_post.sum())
    if wl.group_offsets is not None:
        for g in range(len(wl.prefix_lens)):
            n = int(wl.group_offsets[g + 1] - wl.group_offsets[g])
            tokens -= (n - 1) * int(wl.prefix_lens[g])
    qo = 2 * wl.B * wl.Hq * wl.D * wl.elt
    tables = sum(_ceil_div(int(n), wl.bs) for n in wl.seq_lens_post) * 4
    return int(tokens * row + qo + tables + 4 * wl.B)


def write_bytes(wl: Workload) -> int:
    """Bytes of the cache update: read the new K/V rows and the slots, write the rows."""
    row = wl.Hkv * wl.D * wl.elt
    return int(2 * 2 * wl.B * row + 8 * wl.B)


def copy_bytes(wl: Workload) -> int:
    """Bytes of the copy-on-write block copies: read and write both caches' blocks."""
    return int(len(wl.cow_pairs) * wl.block_bytes * 2 * 2 + 16 * len(wl.cow_pairs))
