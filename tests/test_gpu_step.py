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
