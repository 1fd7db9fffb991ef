"""GPU parity of the fused step (paged_decode_step): copy-on-write copy, cache write of the
new token and decode in one launch must leave the same pool, byte for byte, as the oracle's
copy_blocks + kv_write, and give the oracle's attention."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import (assert_attention_close, device_inputs, gpu_step, oracle_step, raw,
                      to_host_bits, widen, workspace_for)

pytestmark = pytest.mark.gpu

CASES = [("tiny", 1), ("tiny_post", 1), ("mha", 8), ("gqa16", 8), ("gqa32", 8), ("long", 16),
         ("share_fork", 4), ("share_tails", 4)]


@pytest.fixture(autouse=True)
def _clean():
    pkv.device_errors(clear=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("P", [0, 16, 256])
@pytest.mark.parametrize("name,sd", CASES)
def test_fused_step_matches_oracle(name, sd, P):
    wl = workloads.make(name, scale_down=sd)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, partition_size=P, fused=True)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, f"{name} P={P}")
    assert pkv.device_errors() == 0


def test_fused_step_is_repeatable_and_equals_separate_calls():
    """Running the step twice leaves the same pool and output (the copy and the write are
    idempotent), and equals the three separate calls."""
    wl = workloads.make("share_fork", scale_down=4)
    host = workloads.host_tensors(wl)
    dev_a = device_inputs(wl, host)
    dev_b = device_inputs(wl, host)
    out1 = gpu_step(wl, dev_a, fused=True)
    out2 = gpu_step(wl, dev_a, fused=True)
    sep = gpu_step(wl, dev_b)
    assert torch.equal(raw(dev_a["k_cache"]), raw(dev_b["k_cache"]))
    assert torch.equal(raw(dev_a["v_cache"]), raw(dev_b["v_cache"]))
    assert torch.equal(raw(out1), raw(out2))
    assert torch.equal(raw(out1), raw(sep))


def test_fused_step_empty_sequences_and_no_copies():
    """Sequences of length 0 write nothing and give zero rows; cow_src may be omitted."""
    wl = workloads.custom("e", "bf16", 5, 16, 4, 128, 16, [0, 30, 0, 64, 5], seed=21)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    seq = wl.seq_lens_post.copy()
    seq[[0, 2]] = 0
    dev["seq_lens"] = torch.from_numpy(seq).cuda()
    out = torch.empty_like(dev["q"])
    ws = workspace_for(wl)
    pkv.paged_decode_step(out, dev["q"], dev["k_new"], dev["v_new"], dev["k_cache"],
                          dev["v_cache"], dev["block_tables"], dev["seq_lens"], wl.max_seq_len,
                          wl.scale, workspace=ws)
    slots = wl.slot_mapping.copy()
    slots[[0, 2]] = -1
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    oracle.kv_write(host["k_new"], host["v_new"], kc, vc, slots)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    ref = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, seq, wl.scale)
    got = widen(out)
    assert_attention_close(got, ref, "bf16", "fused with empty rows")
    assert np.all(got[[0, 2]] == 0.0)
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("P", [0, 64])
@pytest.mark.parametrize("name,sd", [("share_fork", 4), ("share_tails", 4), ("share_fork", 1),
                                     ("mha", 8)])
def test_fused_shared_prefix_step(name, sd, P):
    wl = workloads.make(name, scale_down=sd)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, partition_size=P, fused=True, shared=True)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, f"{name} P={P}")
    assert pkv.device_errors() == 0


def test_fused_shared_prefix_random_groups():
    rng = np.random.default_rng(5)
    sizes = [1, 3, 9, 2, 5, 4]
    shared = [int(x) * 16 for x in rng.integers(0, 10, size=len(sizes))]
    tails = [int(x) for x in rng.integers(0, 50, size=sum(sizes))]
    wl = workloads.grouped("grp", "bf16", 32, 8, 128, 16, sizes, shared, tails, seed=12)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, fused=True, shared=True)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, "random groups")
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("P", [0, 16, 48])
def test_fused_step_partition_shorter_than_block(P, shared):
    """Blocks of 32 tokens with partitions of 16 or 48: the step copies (copy-on-write) and
    rewrites the block of each new token, so the library rounds the partition up to whole
    blocks and no other partition reads that block while it is rewritten.  P = 0 with the
    shared-prefix step runs the one-CTA-per-group kernel, whose writes leave out the row
    each new token fills when they copy a block."""
    wl = workloads.make("share_fork", scale_down=4, block_size=32)
    assert len(wl.cow_pairs) > 0 and wl.bs == 32
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, partition_size=P, fused=True, shared=shared)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, f"bs=32 P={P} shared={shared}")
    assert pkv.device_errors() == 0


def _group_step(wl, dev, cow_src=None, block_tables=None):
    """The shared-prefix step with the library's partition length: every group of at most
    16 / G members runs one CTA per (group, KV head)."""
    out = torch.full_like(dev["q"], float("nan"))
    n = pkv.paged_attention_decode_shared_prefix_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D,
                                                                wl.max_seq_len, wl.bs, 0)
    ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
    if cow_src is None and len(wl.cow_pairs):
        cow_src = wl.cow_src
    pkv.paged_decode_step_shared_prefix(
        out, dev["q"], dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
        dev["block_tables"] if block_tables is None else block_tables, dev["seq_lens"],
        wl.max_seq_len, wl.scale, torch.from_numpy(wl.group_offsets).cuda(),
        torch.from_numpy(wl.prefix_lens).cuda(), int(np.diff(wl.group_offsets).max()),
        cow_src=None if cow_src is None else torch.from_numpy(np.asarray(cow_src, np.int32)).cuda(),
        workspace=ws)
    return out


def _group_workload(Hq, Hkv, D, bs, seed):
    """Eight groups of 1 .. 16 / G members: forks (a prefix ending inside a block, copied on
    write by all but its last holder), prefixes of whole blocks with private tails of 0 ..
    3 blocks, and prefixes of 0 tokens."""
    mc = max(1, 16 // (Hq // Hkv))
    rng = np.random.default_rng(seed)
    sizes = [int(x) for x in rng.integers(1, mc + 1, size=8)]
    sizes[0] = mc
    shared, tails = [], []
    for g, m in enumerate(sizes):
        full = int(rng.integers(0, 5)) * bs
        if g % 3 == 1 and m > 1:
            shared.append(full + int(rng.integers(1, bs)))
            tails += [0] * m
        else:
            shared.append(full)
            tails += [int(x) for x in rng.integers(0, 3 * bs + 1, size=m)]
    return workloads.grouped("grpstep", "bf16", Hq, Hkv, D, bs, sizes, shared, tails, seed=seed)


@pytest.mark.parametrize("Hq,Hkv,D,bs", [(32, 8, 128, 16), (16, 16, 64, 16), (32, 2, 128, 16),
                                         (32, 8, 256, 32), (16, 4, 128, 64)])
def test_fused_group_step_edge_cases(Hq, Hkv, D, bs):
    """The one-CTA-per-group fused step with G = 1, 4, 8 and 16, head dims 64 to 256 and
    blocks of 16 to 64 tokens: the pool must equal the oracle's copy_blocks + kv_write byte
    for byte, and the attention the oracle's.  Then two members of private-tail groups are
    emptied (nothing written, zero rows) and one copy-on-write source names the block it
    would copy into (no copy)."""
    wl = _group_workload(Hq, Hkv, D, bs, seed=Hq * 31 + D + bs)
    mc = max(1, 16 // (Hq // Hkv))
    assert int(np.diff(wl.group_offsets).max()) <= mc
    assert len(wl.cow_pairs) > 0 or mc == 1  # G = 16: one member a group, nothing forks
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    out = _group_step(wl, dev)
    kc, vc, ref = oracle_step(wl, host)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert_attention_close(widen(out), ref, wl.dtype, f"G={Hq // Hkv} D={D} bs={bs}")
    assert pkv.device_errors() == 0

    # Empty members and a copy source equal to its destination, from the pre-step pool.
    forked = {int(d) for _, d in wl.cow_pairs} | {int(s_) for s_, _ in wl.cow_pairs}
    private = [b for b in range(wl.B) if int(wl.slot_mapping[b]) // wl.bs not in forked]
    empty = private[:2]
    self_copy = private[2] if len(private) > 2 else None
    dev = device_inputs(wl, host)
    seq = wl.seq_lens_post.copy()
    seq[empty] = 0
    dev["seq_lens"] = torch.from_numpy(seq).cuda()
    cow = wl.cow_src.copy()
    if self_copy is not None:
        cow[self_copy] = int(wl.slot_mapping[self_copy]) // wl.bs
    out = _group_step(wl, dev, cow_src=cow)
    slots = wl.slot_mapping.copy()
    slots[empty] = -1
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    assert oracle.copy_blocks(kc, vc, wl.cow_pairs) == 0
    assert oracle.kv_write(host["k_new"], host["v_new"], kc, vc, slots) == 0
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    ref = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, seq, wl.scale)
    got = widen(out)
    assert_attention_close(got, ref, wl.dtype, "empty members, self copy")
    assert np.all(got[empty] == 0.0)
    assert pkv.device_errors() == 0


def test_fused_group_step_flags_bad_ids():
    """A copy-on-write source outside the pool is flagged and not read; a new-token block
    outside the pool is flagged, read as zeros and not written (the row the token would
    have gone to keeps its bytes).  Memory stays in bounds."""
    wl = _group_workload(32, 8, 128, 16, seed=77)
    host = workloads.host_tensors(wl)
    dev = device_inputs(wl, host)
    new_block = wl.slot_mapping // wl.bs
    b = int(np.nonzero(new_block == int(wl.cow_pairs[0][1]))[0][0])  # a copying member
    cow = wl.cow_src.copy()
    cow[b] = wl.num_blocks + 3
    _group_step(wl, dev, cow_src=cow)
    torch.cuda.synchronize()
    assert pkv.device_errors(clear=True) & pkv.DEVERR_COPY

    dev = device_inputs(wl, host)
    forked = {int(d) for _, d in wl.cow_pairs} | {int(s_) for s_, _ in wl.cow_pairs}
    c = next(x for x in range(wl.B) if int(new_block[x]) not in forked)
    lb, row = divmod(int(wl.seq_lens_post[c]) - 1, wl.bs)
    bt = wl.block_tables.copy()
    bt[c, lb] = wl.num_blocks + 9
    before = to_host_bits(dev["k_cache"])[int(new_block[c]), row].copy()
    _group_step(wl, dev, block_tables=torch.from_numpy(bt).cuda())
    torch.cuda.synchronize()
    assert pkv.device_errors(clear=True) & pkv.DEVERR_BLOCK_ID
    assert np.array_equal(to_host_bits(dev["k_cache"])[int(new_block[c]), row], before)
