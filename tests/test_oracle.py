"""Pins for the fp64 oracle, against things other than the oracle itself.

Each test names the fact it checks and where that fact comes from: values printed on the
pages (golden files), the pages' invariants (the attention is ordinary softmax attention and
only the storage layout changes), closed forms, a library routine in a special case, and
brute force in high-precision decimal arithmetic.  ``test_oracle_mutants.py`` shows that
planted mistakes in the oracle fail these pins.
"""
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_344_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line.startswith("# columns:"):
                rows.append(("header", line))
            elif line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


def _oracle(o=None):
    return o if o is not None else oracle.default()


# --------------------------------------------------------------------------------------
# Block-count rule ("Paged Attention Explained": Practical Example; Step 1)
# --------------------------------------------------------------------------------------

def test_block_count_worked_example(o=None):
    o = _oracle(o)
    rows = [r for r in _rows("block_count_example.txt") if r[0] != "header"]
    assert len(rows) == 5
    for tokens, bs, blocks, unused in rows:
        got = o.calculate_blocks(tokens, bs)
        assert got == blocks, (tokens, bs)
        assert got * bs - tokens == unused


def test_block_count_errors_and_edges(o=None):
    o = _oracle(o)
    with pytest.raises(ValueError):
        o.calculate_blocks(-1, 16)
    with pytest.raises(ValueError):
        o.calculate_blocks(10, 0)
    with pytest.raises(ValueError):
        o.calculate_blocks(10, -16)
    assert o.calculate_blocks(0, 16) == 0
    for n in range(0, 200):
        for bs in (1, 7, 16, 32):
            assert o.calculate_blocks(n, bs) == math.ceil(n / bs)


# --------------------------------------------------------------------------------------
# Helpers: small paged problems built by the tests themselves
# --------------------------------------------------------------------------------------

def _place(K, V, table, NB, bs, fill=np.nan):
    """Store contiguous K,V [L,Hkv,D] (float32) in a pool [NB,bs,Hkv,D] at table's blocks."""
    L, Hkv, D = K.shape
    kc = np.full((NB, bs, Hkv, D), fill, dtype=np.float32)
    vc = np.full((NB, bs, Hkv, D), fill, dtype=np.float32)
    for t in range(L):
        kc[table[t // bs], t % bs] = K[t]
        vc[table[t // bs], t % bs] = V[t]
    return kc, vc


def _decode_one(o, q, K, V, scale, bs=16, NB=None, perm_seed=0):
    """Oracle output for one sequence (q [Hq,D], contiguous K,V [L,Hkv,D]) paged at
    a random placement."""
    L = K.shape[0]
    nblk = -(-L // bs)
    NB = NB or max(nblk * 2, 1)
    table = np.random.default_rng(perm_seed).permutation(NB)[:nblk].astype(np.int32)
    kc, vc = _place(K, V, table, NB, bs)
    bt = np.full((1, max(nblk, 1)), -1, dtype=np.int32)
    bt[0, :nblk] = table
    return o.paged_decode(q[None].astype(np.float32), kc, vc, bt, np.array([L], np.int32), scale)[0]


# --------------------------------------------------------------------------------------
# Block-table resolution ("Paged Attention Explained": Step 3 and Step 4)
# --------------------------------------------------------------------------------------

def test_block_table_example(o=None):
    """The hand example (logical 0,1,2 -> physical 7,3,12): the cache write puts each of
    40 tokens at the hand-worked (block, offset), and decoding through this table equals
    decoding the same tokens placed at physical blocks 0,1,2."""
    o = _oracle(o)
    rows = _rows("block_table_example.txt")
    split = [i for i, r in enumerate(rows) if r[0] == "header"]
    mapping = rows[split[0] + 1:split[1]]
    positions = rows[split[1] + 1:]
    table = np.array([p for _, p in sorted(mapping)], dtype=np.int32)
    assert list(table) == [7, 3, 12]
    bs, NB, Hkv, D, L = 16, 16, 2, 8, 40
    rng = np.random.default_rng(5)
    K = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    V = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    kc = np.full((NB, bs, Hkv, D), np.nan, np.float32)
    vc = kc.copy()
    slots = np.array([table[t // bs] * bs + t % bs for t in range(L)], dtype=np.int64)
    assert o.kv_write(K, V, kc, vc, slots) == 0
    for t, phys, off in positions:
        np.testing.assert_array_equal(kc[phys, off], K[t])
        np.testing.assert_array_equal(vc[phys, off], V[t])
    q = rng.standard_normal((1, 4, D), dtype=np.float32)
    bt = table[None]
    out_paged = o.paged_decode(q, kc, vc, bt, np.array([L], np.int32), 0.3)
    kc2, vc2 = _place(K, V, np.array([0, 1, 2]), 3, bs)
    out_flat = o.paged_decode(q, kc2, vc2, np.array([[0, 1, 2]], np.int32),
                              np.array([L], np.int32), 0.3)
    np.testing.assert_array_equal(out_paged, out_flat)


def _random_problem(seed, B=3, Hq=4, Hkv=2, D=16, bs=16, lens=(1, 17, 40), NB=24):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, D), dtype=np.float32)
    Ks = [rng.standard_normal((L, Hkv, D), dtype=np.float32) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D), dtype=np.float32) for L in lens]
    return q, Ks, Vs


def _pool_from(Ks, Vs, bs, NB, perm_seed):
    """Place sequences in a shuffled pool; returns caches, table, lengths."""
    B = len(Ks)
    nblk = [-(-K.shape[0] // bs) for K in Ks]
    perm = np.random.default_rng(perm_seed).permutation(NB).astype(np.int32)
    Hkv, D = Ks[0].shape[1:]
    kc = np.full((NB, bs, Hkv, D), np.nan, np.float32)
    vc = kc.copy()
    MB = max(max(nblk), 1)
    bt = np.full((B, MB), -1, np.int32)
    cur = 0
    for b in range(B):
        ids = perm[cur:cur + nblk[b]]
        cur += nblk[b]
        bt[b, :nblk[b]] = ids
        for t in range(Ks[b].shape[0]):
            kc[ids[t // bs], t % bs] = Ks[b][t]
            vc[ids[t // bs], t % bs] = Vs[b][t]
    lens = np.array([K.shape[0] for K in Ks], np.int32)
    return kc, vc, bt, lens


def test_permutation_invariance(o=None):
    """Any placement of the physical blocks gives the identical result (bitwise: the
    resolved contiguous copy is the same, so is the arithmetic)."""
    o = _oracle(o)
    q, Ks, Vs = _random_problem(1)
    outs = []
    for perm_seed in range(4):
        kc, vc, bt, lens = _pool_from(Ks, Vs, 16, 24, perm_seed)
        outs.append(o.paged_decode(q, kc, vc, bt, lens, 0.25))
    for out in outs[1:]:
        np.testing.assert_array_equal(out, outs[0])


def test_block_size_invariance(o=None):
    """The same logical K/V in pools of block size 1, 8, 16 and 32 decode identically."""
    o = _oracle(o)
    q, Ks, Vs = _random_problem(2, lens=(5, 33, 64))
    outs = []
    for bs in (1, 8, 16, 32):
        NB = sum(-(-K.shape[0] // bs) for K in Ks) + 3
        kc, vc, bt, lens = _pool_from(Ks, Vs, bs, NB, 7)
        outs.append(o.paged_decode(q, kc, vc, bt, lens, 0.25))
    for out in outs[1:]:
        np.testing.assert_array_equal(out, outs[0])


def test_equals_contiguous_sdpa_float64(o=None):
    """Equals PyTorch's scaled_dot_product_attention in float64 on the contiguous tensors
    (an independent library routine), with grouped heads expanded explicitly."""
    o = _oracle(o)
    for seed, (Hq, Hkv) in enumerate([(4, 4), (8, 2), (6, 3), (8, 1)]):
        q, Ks, Vs = _random_problem(10 + seed, Hq=Hq, Hkv=Hkv, D=24, lens=(3, 48, 70))
        kc, vc, bt, lens = _pool_from(Ks, Vs, 16, 20, seed)
        scale = 1.0 / math.sqrt(24)
        out = o.paged_decode(q, kc, vc, bt, lens, scale)
        G = Hq // Hkv
        for b in range(len(Ks)):
            K = torch.from_numpy(Ks[b]).double()  # [L,Hkv,D]
            V = torch.from_numpy(Vs[b]).double()
            Kh = K.repeat_interleave(G, dim=1).permute(1, 0, 2)[None]  # [1,Hq,L,D]
            Vh = V.repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
            qq = torch.from_numpy(q[b]).double()[None, :, None, :]  # [1,Hq,1,D]
            ref = torch.nn.functional.scaled_dot_product_attention(qq, Kh, Vh, scale=scale)
            np.testing.assert_allclose(out[b], ref[0, :, 0, :].numpy(), rtol=1e-12, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv(o=None):
    """Grouped heads: query head h reads KV head h // G, i.e. the result equals MHA over
    K/V whose heads are repeated G times."""
    o = _oracle(o)
    q, Ks, Vs = _random_problem(3, Hq=8, Hkv=2, D=8, lens=(9, 30, 16))
    kc, vc, bt, lens = _pool_from(Ks, Vs, 16, 12, 1)
    out = o.paged_decode(q, kc, vc, bt, lens, 0.5)
    Ks4 = [np.repeat(K, 4, axis=1) for K in Ks]
    Vs4 = [np.repeat(V, 4, axis=1) for V in Vs]
    kc4, vc4, bt4, lens4 = _pool_from(Ks4, Vs4, 16, 12, 1)
    out4 = o.paged_decode(q, kc4, vc4, bt4, lens4, 0.5)
    np.testing.assert_array_equal(out, out4)


# --------------------------------------------------------------------------------------
# Special cases and closed forms
# --------------------------------------------------------------------------------------

def test_single_token_returns_v_exactly(o=None):
    o = _oracle(o)
    rng = np.random.default_rng(4)
    for dtype in ("f32", "bf16"):
        wl = workloads.custom("one", dtype, 3, 4, 2, 32, 16, [0, 0, 0], seed=4)
        t = workloads.host_tensors(wl)
        lens = wl.seq_lens_pre + 1
        # place the new token by hand (block table after the step, offset 0)
        kc, vc = t["k_cache"].copy(), t["v_cache"].copy()
        for b in range(wl.B):
            kc[wl.block_tables[b, 0], 0] = t["k_new"][b]
            vc[wl.block_tables[b, 0], 0] = t["v_new"][b]
        out = o.paged_decode(t["q"], kc, vc, wl.block_tables, lens, rng.uniform(0.1, 3))
        v = t["v_new"]
        if dtype == "bf16":
            v = (v.astype(np.uint32) << 16).view(np.float32)
        for b in range(wl.B):
            for h in range(wl.Hq):
                np.testing.assert_array_equal(out[b, h], v[b, h // wl.G].astype(np.float64))


def test_identical_keys_and_zero_query_give_mean_of_v(o=None):
    o = _oracle(o)
    rng = np.random.default_rng(6)
    L, Hkv, D = 37, 2, 8
    V = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    Kc = np.repeat(rng.standard_normal((1, Hkv, D), dtype=np.float32), L, axis=0)
    q = rng.standard_normal((2, D), dtype=np.float32)
    mean = V.astype(np.float64).mean(axis=0)  # [Hkv, D]
    out = _decode_one(o, q, Kc, V, 0.7)
    np.testing.assert_allclose(out, mean, rtol=1e-14, atol=1e-14)
    K = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    out_q0 = _decode_one(o, np.zeros_like(q), K, V, 0.7)
    np.testing.assert_allclose(out_q0, mean, rtol=1e-14, atol=1e-14)
    out_s0 = _decode_one(o, q, K, V, 0.0)
    np.testing.assert_allclose(out_s0, mean, rtol=1e-14, atol=1e-14)


def _softmax_decimal(q, K, V, scale):
    """Brute force in 40-digit decimal arithmetic, straight from the definition
    (exp without any shift)."""
    getcontext().prec = 40
    L, D = K.shape
    s = [Decimal(float(scale)) * sum(Decimal(float(q[d])) * Decimal(float(K[t, d]))
                                      for d in range(D)) for t in range(L)]
    w = [x.exp() for x in s]
    tot = sum(w)
    return [float(sum(w[t] * Decimal(float(V[t, d])) for t in range(L)) / tot) for d in range(D)]


def test_brute_force_tiny_inputs(o=None):
    o = _oracle(o)
    rng = np.random.default_rng(8)
    for trial in range(12):
        L = int(rng.integers(1, 6))
        D = int(rng.integers(1, 5))
        bs = int(rng.integers(1, 4))
        K = rng.standard_normal((L, 1, D), dtype=np.float32) * 2
        V = rng.standard_normal((L, 1, D), dtype=np.float32)
        q = rng.standard_normal((1, D), dtype=np.float32)
        scale = float(rng.uniform(0.1, 2.0))
        out = _decode_one(o, q, K, V, scale, bs=bs, perm_seed=trial)
        ref = _softmax_decimal(q[0], K[:, 0], V[:, 0], scale)
        np.testing.assert_allclose(out[0], ref, rtol=1e-14, atol=1e-15)


def test_two_token_closed_form(o=None):
    """L = 2: out = sigmoid(s1 - s0) V1 + sigmoid(s0 - s1) V0."""
    o = _oracle(o)
    rng = np.random.default_rng(9)
    for _ in range(10):
        D = 6
        K = rng.standard_normal((2, 1, D), dtype=np.float32)
        V = rng.standard_normal((2, 1, D), dtype=np.float32)
        q = rng.standard_normal((1, D), dtype=np.float32) * 3
        scale = 0.8
        s0 = scale * float(np.dot(q[0].astype(np.float64), K[0, 0].astype(np.float64)))
        s1 = scale * float(np.dot(q[0].astype(np.float64), K[1, 0].astype(np.float64)))
        sig = lambda x: 1.0 / (1.0 + math.exp(-x))
        ref = sig(s1 - s0) * V[1, 0].astype(np.float64) + sig(s0 - s1) * V[0, 0].astype(np.float64)
        out = _decode_one(o, q, K, V, scale, bs=1)
        np.testing.assert_allclose(out[0], ref, rtol=1e-13, atol=1e-14)


def test_linear_in_v(o=None):
    """out(V1 + V2) = out(V1) + out(V2) with values on a grid where the sums are exact."""
    o = _oracle(o)
    rng = np.random.default_rng(11)
    L, Hkv, D = 45, 2, 8
    K = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    V1 = (rng.integers(-512, 512, (L, Hkv, D)) / 128.0).astype(np.float32)
    V2 = (rng.integers(-512, 512, (L, Hkv, D)) / 128.0).astype(np.float32)
    q = rng.standard_normal((4, D), dtype=np.float32)
    a = _decode_one(o, q, K, V1, 0.4)
    b = _decode_one(o, q, K, V2, 0.4)
    c = _decode_one(o, q, K, V1 + V2, 0.4)
    np.testing.assert_allclose(c, a + b, rtol=1e-12, atol=1e-12)


def test_empty_sequence_gives_zeros_and_nan_slots_are_never_read(o=None):
    o = _oracle(o)
    wl = workloads.make("tiny")
    t = workloads.host_tensors(wl)
    lens = wl.seq_lens_pre.copy()
    lens[1] = 0
    bt = wl.block_tables_pre.copy()
    out = o.paged_decode(t["q"], t["k_cache"], t["v_cache"], bt, lens, wl.scale)
    assert np.all(out[1] == 0.0)
    assert np.isfinite(out).all()  # unused slots are NaN in the pool and must not leak


def test_out_of_range_lengths_are_reported(o=None):
    """A length longer than its table row covers is an error, even when the memory after
    the row holds valid block ids (here: the next row)."""
    o = _oracle(o)
    rng = np.random.default_rng(13)
    kc = rng.standard_normal((4, 16, 1, 8), dtype=np.float32)
    vc = rng.standard_normal((4, 16, 1, 8), dtype=np.float32)
    q = rng.standard_normal((2, 1, 8), dtype=np.float32)
    bt = np.array([[0, 1], [2, 3]], np.int32)
    o.paged_decode(q, kc, vc, bt, np.array([32, 5], np.int32), 0.5)
    with pytest.raises(ValueError):
        o.paged_decode(q, kc, vc, bt, np.array([33, 5], np.int32), 0.5)


# --------------------------------------------------------------------------------------
# Cache write and copy-on-write copies
# --------------------------------------------------------------------------------------

def test_kv_write_whole_pool_bytes(o=None):
    """Only the addressed slots change (checked with a flat row view of the pool, a
    different formulation from block/offset), slot < 0 is skipped, NaN bytes elsewhere
    survive bit for bit, out-of-range slots are counted and skipped."""
    o = _oracle(o)
    for dtype in ("f32", "bf16"):
        wl = workloads.make("tiny") if dtype == "f32" else workloads.make("gqa16", scale_down=64)
        t = workloads.host_tensors(wl)
        kc, vc = t["k_cache"].copy(), t["v_cache"].copy()
        slots = wl.slot_mapping.copy()
        slots[0] = -1
        bad = o.kv_write(t["k_new"], t["v_new"], kc, vc, slots)
        assert bad == 0
        ek = t["k_cache"].copy().reshape(wl.num_blocks * wl.bs, wl.Hkv, wl.D)
        ev = t["v_cache"].copy().reshape(wl.num_blocks * wl.bs, wl.Hkv, wl.D)
        keep = slots >= 0
        ek[slots[keep]] = t["k_new"][keep]
        ev[slots[keep]] = t["v_new"][keep]
        assert kc.tobytes() == ek.tobytes() and vc.tobytes() == ev.tobytes()
        slots2 = wl.slot_mapping.copy()
        slots2[-1] = wl.num_blocks * wl.bs
        assert o.kv_write(t["k_new"], t["v_new"], kc, vc, slots2) == 1


def test_write_then_decode_round_trip(o=None):
    """Writing tokens 0..L-1 through their slots and decoding equals decoding the same
    tokens laid out contiguously (the write and the table resolution agree)."""
    o = _oracle(o)
    rng = np.random.default_rng(12)
    L, Hkv, D, bs, NB = 50, 2, 8, 16, 9
    K = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    V = rng.standard_normal((L, Hkv, D), dtype=np.float32)
    table = np.array([8, 2, 5, 0], np.int32)
    kc = np.full((NB, bs, Hkv, D), np.nan, np.float32)
    vc = kc.copy()
    slots = np.array([table[t // bs] * bs + t % bs for t in range(L)], np.int64)
    o.kv_write(K, V, kc, vc, slots)
    q = rng.standard_normal((1, 4, D), dtype=np.float32)
    out = o.paged_decode(q, kc, vc, table[None], np.array([L], np.int32), 0.3)
    kc2, vc2 = _place(K, V, np.arange(4), 4, bs)
    ref = o.paged_decode(q, kc2, vc2, np.arange(4, dtype=np.int32)[None],
                         np.array([L], np.int32), 0.3)
    np.testing.assert_array_equal(out, ref)


def test_copy_blocks_bytes_and_cow_isolation(o=None):
    """Copies make dst byte-identical to src and touch nothing else.  In the shared-prefix
    fork, after the copies and writes each branch decodes exactly as if it had private
    blocks, and the branches do not see one another's new tokens."""
    o = _oracle(o)
    wl = workloads.make("share_fork", scale_down=16)
    assert len(wl.cow_pairs) == 3 * (wl.B // 4)
    t = workloads.host_tensors(wl)
    kc, vc = t["k_cache"].copy(), t["v_cache"].copy()
    before_k, before_v = kc.copy(), vc.copy()
    assert o.copy_blocks(kc, vc, wl.cow_pairs) == 0
    dsts = set(int(d) for d in wl.cow_pairs[:, 1])
    for s, d in wl.cow_pairs:
        assert kc[d].tobytes() == before_k[s].tobytes()
        assert vc[d].tobytes() == before_v[s].tobytes()
    for blk in range(wl.num_blocks):
        if blk not in dsts:
            assert kc[blk].tobytes() == before_k[blk].tobytes()
            assert vc[blk].tobytes() == before_v[blk].tobytes()
    o.kv_write(t["k_new"], t["v_new"], kc, vc, wl.slot_mapping)
    out = o.paged_decode(t["q"], kc, vc, wl.block_tables, wl.seq_lens_post, wl.scale)
    # independent layout: every branch gets private copies of its own tokens
    as_f = (lambda a: (a.astype(np.uint32) << 16).view(np.float32))
    for b in range(wl.B):
        L = int(wl.seq_lens_pre[b])
        ids = wl.block_tables_pre[b]
        K = np.stack([as_f(before_k[ids[i // wl.bs], i % wl.bs]) for i in range(L)]
                     + [as_f(t["k_new"][b])])
        V = np.stack([as_f(before_v[ids[i // wl.bs], i % wl.bs]) for i in range(L)]
                     + [as_f(t["v_new"][b])])
        ref = _decode_one(o, as_f(t["q"][b]), K, V, wl.scale, bs=wl.bs, perm_seed=b)
        np.testing.assert_allclose(out[b], ref, rtol=0, atol=0)
    bad = np.array([[0, wl.num_blocks]], np.int64)
    assert o.copy_blocks(kc, vc, bad) == 1


def test_row_selection_matches_full(o=None):
    o = _oracle(o)
    wl = workloads.make("gqa16", scale_down=32)
    t = workloads.host_tensors(wl)
    o.kv_write(t["k_new"], t["v_new"], t["k_cache"], t["v_cache"], wl.slot_mapping)
    full = o.paged_decode(t["q"], t["k_cache"], t["v_cache"], wl.block_tables, wl.seq_lens_post,
                          wl.scale)
    rows = [(0, 0), (wl.B - 1, wl.Hq - 1), (3, 17)]
    part = o.paged_decode(t["q"], t["k_cache"], t["v_cache"], wl.block_tables, wl.seq_lens_post,
                          wl.scale, rows=rows)
    for i, (b, h) in enumerate(rows):
        np.testing.assert_array_equal(part[i], full[b, h])


# --------------------------------------------------------------------------------------
# Multi-query (prefill / chunked append) attention
# --------------------------------------------------------------------------------------

def _prefill_problem(seed, lens, qlens, Hq=4, Hkv=2, D=16, bs=16):
    rng = np.random.default_rng(seed)
    Ks = [rng.standard_normal((L, Hkv, D), dtype=np.float32) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D), dtype=np.float32) for L in lens]
    NB = sum(-(-L // bs) for L in lens) + 3
    kc, vc, bt, sl = _pool_from(Ks, Vs, bs, NB, seed)
    cu = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = rng.standard_normal((int(cu[-1]), Hq, D), dtype=np.float32)
    return q, Ks, Vs, kc, vc, bt, sl, cu


def test_prefill_single_query_equals_decode(o=None):
    """With one query per sequence, the multi-query attention is the decode, bit for bit."""
    o = _oracle(o)
    q, Ks, Vs, kc, vc, bt, sl, cu = _prefill_problem(31, [5, 40, 17], [1, 1, 1])
    pre = o.paged_prefill(q, kc, vc, bt, sl, cu, 0.3)
    dec = o.paged_decode(q, kc, vc, bt, sl, 0.3)
    np.testing.assert_array_equal(pre, dec)


def test_prefill_equals_causal_sdpa_float64(o=None):
    """Equals PyTorch's scaled_dot_product_attention in float64 with an explicit causal mask
    on the contiguous tensors: query i of a chunk of Q sees tokens 0 .. L - Q + i."""
    o = _oracle(o)
    for seed, (Hq, Hkv) in enumerate([(4, 4), (8, 2), (6, 3)]):
        lens, qlens = [33, 7, 64], [9, 7, 1]
        q, Ks, Vs, kc, vc, bt, sl, cu = _prefill_problem(40 + seed, lens, qlens, Hq, Hkv, D=24)
        out = o.paged_prefill(q, kc, vc, bt, sl, cu, 0.2)
        G = Hq // Hkv
        for b, (L, Q) in enumerate(zip(lens, qlens)):
            K = torch.from_numpy(Ks[b]).double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
            V = torch.from_numpy(Vs[b]).double().repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
            qq = torch.from_numpy(q[cu[b]:cu[b + 1]]).double().permute(1, 0, 2)[None]  # [1,Hq,Q,D]
            mask = torch.arange(L)[None, :] <= (L - Q + torch.arange(Q))[:, None]   # [Q, L]
            ref = torch.nn.functional.scaled_dot_product_attention(qq, K, V, attn_mask=mask,
                                                                   scale=0.2)
            np.testing.assert_allclose(out[cu[b]:cu[b + 1]], ref[0].permute(1, 0, 2).numpy(),
                                       rtol=1e-12, atol=1e-12)


def test_prefill_brute_force_tiny(o=None):
    o = _oracle(o)
    rng = np.random.default_rng(44)
    for trial in range(6):
        L = int(rng.integers(2, 6))
        Q = int(rng.integers(1, L + 1))
        D = int(rng.integers(1, 4))
        q, Ks, Vs, kc, vc, bt, sl, cu = _prefill_problem(50 + trial, [L], [Q], Hq=1, Hkv=1, D=D,
                                                         bs=2)
        out = o.paged_prefill(q, kc, vc, bt, sl, cu, 0.7)
        for i in range(Q):
            vis = L - Q + i + 1
            ref = _softmax_decimal(q[i, 0], Ks[0][:vis, 0], Vs[0][:vis, 0], 0.7)
            np.testing.assert_allclose(out[i, 0], ref, rtol=1e-14, atol=1e-15)


def test_prefill_rejects_chunks_longer_than_sequences(o=None):
    o = _oracle(o)
    q, Ks, Vs, kc, vc, bt, sl, cu = _prefill_problem(60, [5], [5])
    o.paged_prefill(q, kc, vc, bt, sl, cu, 0.5)
    with pytest.raises(ValueError):
        o.paged_prefill(q, kc, vc, bt, np.array([4], np.int32), cu, 0.5)
