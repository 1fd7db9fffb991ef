"""GPU parity: the CUDA library against the fp64 oracle on the same seeded inputs.

Sizes here are scaled-down versions of the five workloads (same head shapes, block sizes
and length distributions) so the oracle finishes in seconds while every kernel still runs
many tiles, several partitions and ragged tails.  Full-size sampled checks live in
``test_gpu_fullsize.py``.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import (assert_attention_close, device_inputs, gpu_step, oracle_step, raw,
                      to_device, to_host_bits, widen, workspace_for)

pytestmark = pytest.mark.gpu

SMALL = [("tiny", 1), ("tiny_post", 1), ("mha", 8), ("gqa16", 8), ("gqa32", 8), ("long", 16),
         ("share_fork", 4), ("share_tails", 4)]
PATHS = {"auto": pkv.PKV_PATH_AUTO, "cuda_cores": pkv.PKV_PATH_CUDA_CORES,
         "tensor_cores": pkv.PKV_PATH_TENSOR_CORES}


@pytest.fixture(autouse=True)
def _clean_state():
    pkv.device_errors(clear=True)
    old = pkv.set_decode_path(pkv.PKV_PATH_AUTO)
    yield
    pkv.set_decode_path(old)
    torch.cuda.synchronize()


def _case(name, scale_down):
    wl = workloads.make(name, scale_down=scale_down)
    host = workloads.host_tensors(wl)
    return wl, host


@pytest.mark.parametrize("name,sd", SMALL)
def test_write_and_copy_bit_exact(name, sd):
    """The whole pool after copy_blocks + paged_kv_write equals the oracle's byte for byte
    (written rows, copied blocks, untouched rows and the NaN-poisoned free slots)."""
    wl, host = _case(name, sd)
    dev = device_inputs(wl, host)
    if len(wl.cow_pairs):
        pkv.copy_blocks(dev["k_cache"], dev["v_cache"], dev["cow_pairs"])
    pkv.paged_kv_write(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
                       dev["slot_mapping"])
    kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
    oracle.copy_blocks(kc, vc, wl.cow_pairs)
    oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping)
    assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"]).tobytes() == vc.tobytes()
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name,sd", SMALL)
def test_decode_matches_oracle(name, sd, path):
    wl, host = _case(name, sd)
    if path == "tensor_cores" and wl.dtype != "bf16":
        pytest.skip("fp32 always runs on CUDA cores")
    pkv.set_decode_path(PATHS[path])
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev)
    _, _, ref = oracle_step(wl, host)
    assert_attention_close(widen(out), ref, wl.dtype, f"{name}/{path}")
    assert pkv.device_errors() == 0


@pytest.mark.parametrize("path", ["cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("P", [16, 64, 512, 4096, 1 << 20])
def test_partition_invariance(P, path):
    """Any partition length gives the oracle's result: one partition, a partition per
    stage, and sizes in between (the log-sum-exp merge of split partitions is exact up to
    rounding)."""
    pkv.set_decode_path(PATHS[path])
    wl, host = _case("long", 16)
    dev = device_inputs(wl, host)
    out = gpu_step(wl, dev, partition_size=P)
    _, _, ref = oracle_step(wl, host)
    assert_attention_close(widen(out), ref, wl.dtype, f"P={P}")


@pytest.mark.parametrize("ctas", [1, 3, 37, 296])
@pytest.mark.parametrize("name,sd", [("mha", 8), ("gqa16", 8), ("long", 16), ("share_fork", 4),
                                     ("tiny", 1)])
def test_balanced_split_any_worker_count(name, sd, ctas):
    """The work-balanced kernel cuts the stage stream into one range per warp; with 1 to
    296 CTAs units are cut into every pattern of pieces (inside one worker, across two,
    across many, one stage per worker) and must still give the oracle's result."""
    old = pkv.set_decode_ctas(ctas)
    old_split = pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED)
    try:
        wl, host = _case(name, sd)
        dev = device_inputs(wl, host)
        out = gpu_step(wl, dev)
        _, _, ref = oracle_step(wl, host)
        assert_attention_close(widen(out), ref, wl.dtype, f"{name} ctas={ctas}")
        assert pkv.device_errors() == 0
    finally:
        pkv.set_decode_ctas(old)
        pkv.set_decode_split(old_split)


def test_workspace_reuse_and_streams():
    """Two calls on one workspace (its counters must come back to zero) and a call on a
    side stream give identical results."""
    wl, host = _case("long", 16)
    dev = device_inputs(wl, host)
    ws = workspace_for(wl, 256)
    out1 = gpu_step(wl, dev, partition_size=256, workspace=ws)
    out2 = torch.empty_like(out1)
    pkv.paged_attention_decode(out2, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"],
                               dev["seq_lens"], wl.max_seq_len, wl.scale, workspace=ws,
                               partition_size=256)
    s = torch.cuda.Stream()
    out3 = torch.empty_like(out1)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pkv.paged_attention_decode(out3, dev["q"], dev["k_cache"], dev["v_cache"],
                                   dev["block_tables"], dev["seq_lens"], wl.max_seq_len, wl.scale,
                                   workspace=ws, partition_size=256)
    s.synchronize()
    assert torch.equal(raw(out1), raw(out2)) and torch.equal(raw(out1), raw(out3))
    assert int(ws[:wl.B * wl.Hkv * 4].view(torch.int32).abs().sum()) == 0  # counters back at 0


EDGE = [
    # (dtype, B, Hq, Hkv, D, bs, lengths)
    ("bf16", 6, 8, 8, 128, 16, [0, 1, 15, 16, 31, 32]),      # empty row, block edges
    ("bf16", 5, 32, 8, 128, 32, [0, 31, 32, 33, 200]),
    ("bf16", 4, 6, 2, 128, 16, [1, 17, 100, 300]),            # G = 3
    ("bf16", 3, 32, 2, 128, 16, [5, 70, 600]),                # G = 16
    ("bf16", 3, 16, 4, 64, 16, [9, 64, 333]),                 # D = 64
    ("bf16", 3, 8, 2, 256, 16, [9, 64, 333]),                 # D = 256
    ("bf16", 3, 16, 8, 128, 64, [1, 130, 700]),               # bs = 64
    ("bf16", 2, 8, 4, 128, 256, [255, 1030]),                 # bs = 256
    ("f32", 4, 8, 2, 128, 16, [1, 16, 47, 130]),              # fp32 D = 128, G = 4
    ("f32", 3, 16, 2, 64, 32, [3, 64, 95]),                   # fp32 G = 8
    ("f32", 3, 2, 1, 64, 16, [40, 7, 0]),                     # fp32 G = 2
]


@pytest.mark.parametrize("path", ["auto", "cuda_cores", "tensor_cores"])
@pytest.mark.parametrize("case", EDGE, ids=[f"{c[0]}-G{c[2]//c[3]}-D{c[4]}-bs{c[5]}" for c in EDGE])
def test_edge_shapes(case, path):
    dtype, B, Hq, Hkv, D, bs, lens = case
    if path == "tensor_cores" and dtype != "bf16":
        pytest.skip("fp32 always runs on CUDA cores")
    pkv.set_decode_path(PATHS[path])
    pre = np.maximum(np.array(lens) - 1, 0)
    wl = workloads.custom("edge", dtype, B, Hq, Hkv, D, bs, pre, seed=77)
    host = workloads.host_tensors(wl)
    # rows whose listed length is 0 decode an empty sequence (no write for them)
    zero = np.array(lens) == 0
    wl.slot_mapping[zero] = -1
    seq = wl.seq_lens_post.copy()
    seq[zero] = 0
    dev = device_inputs(wl, host)
    dev["seq_lens"] = torch.from_numpy(seq).cuda()
    for P in (0, 16):
        pkv.paged_kv_write(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
                           dev["slot_mapping"])
        out = torch.empty_like(dev["q"])
        n = pkv.paged_attention_decode_workspace_size(B, Hq, Hkv, D, int(seq.max()), bs, P)
        ws = torch.zeros(max(n, 1), dtype=torch.uint8, device="cuda")
        pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"],
                                   dev["block_tables"], dev["seq_lens"], int(seq.max()), wl.scale,
                                   workspace=ws, partition_size=P)
        kc, vc = host["k_cache"].copy(), host["v_cache"].copy()
        oracle.kv_write(host["k_new"], host["v_new"], kc, vc, wl.slot_mapping)
        ref = oracle.paged_decode(host["q"], kc, vc, wl.block_tables, seq, wl.scale)
        got = widen(out)
        assert_attention_close(got, ref, dtype, f"{case} P={P}")
        assert np.all(got[zero] == 0.0)
    assert pkv.device_errors() == 0


def test_device_error_flags_and_safety():
    """Out-of-range slots, block ids and lengths are flagged and never dereferenced."""
    wl, host = _case("gqa16", 32)
    dev = device_inputs(wl, host)
    before = dev["k_cache"].clone()
    bad_slots = dev["slot_mapping"].clone()
    bad_slots[0] = wl.num_blocks * wl.bs + 5
    bad_slots[1:] = -1
    pkv.paged_kv_write(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"], bad_slots)
    assert pkv.device_errors() == pkv.DEVERR_SLOT
    assert torch.equal(raw(before), raw(dev["k_cache"]))

    # a table entry outside the pool: flagged, read as zeros, outputs stay finite
    pkv.paged_kv_write(dev["k_new"], dev["v_new"], dev["k_cache"], dev["v_cache"],
                       dev["slot_mapping"])
    bt = dev["block_tables"].clone()
    bt[0, 0] = wl.num_blocks + 3
    out = torch.empty_like(dev["q"])
    ws = workspace_for(wl)
    pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"], bt, dev["seq_lens"],
                               wl.max_seq_len, wl.scale, workspace=ws)
    assert pkv.device_errors() == pkv.DEVERR_BLOCK_ID
    assert torch.isfinite(out.float()).all()

    sl = dev["seq_lens"].clone()
    sl[1] = wl.max_seq_len + 100
    pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"], dev["block_tables"],
                               sl, wl.max_seq_len, wl.scale, workspace=ws)
    assert pkv.device_errors() & pkv.DEVERR_SEQLEN

    pairs = torch.tensor([[0, wl.num_blocks]], dtype=torch.int64, device="cuda")
    pkv.copy_blocks(dev["k_cache"], dev["v_cache"], pairs)
    assert pkv.device_errors() == pkv.DEVERR_COPY
