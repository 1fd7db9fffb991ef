"""GPU parity of the length-ordered decode grid.

With at most 64 sequences and partitions of 2048 tokens or more, the decode's CTAs take
their (sequence, partition, KV head) in length order instead of from their grid
coordinates: every full partition first, then each sequence's last partition from the
longest to the shortest.  Every item must be taken exactly once: a missed one leaves
rows wrong, a doubled one takes a second merge ticket, which the second call on the same
workspace would show.  Cases: ragged lengths around the partition length (one token, one
short of a partition, exactly one, one over, several), empty sequences, the largest batch
the order serves, and the fused step.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import (assert_attention_close, device_inputs, gpu_step, oracle_step,
                      to_host_bits, widen, workspace_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean():
    pkv.device_errors(clear=True)
    yield
    torch.cuda.synchronize()


RAGGED = [1, 2046, 2047, 2048, 6000, 9999, 3, 4095, 4096, 12000]


def _lens(case):
    if case == "ragged":
        return RAGGED
    rng = np.random.default_rng(64)
    return [int(x) for x in rng.integers(1, 9000, size=64)]  # the largest batch it serves


@pytest.mark.parametrize("P", [2048, 4096])
@pytest.mark.parametrize("case", ["ragged", "b64"])
@pytest.mark.parametrize("fused", [False, True])
def test_length_order_matches_oracle(case, P, fused):
    wl = workloads.custom("ord", "bf16", len(_lens(case)), 16, 4, 128, 16, _lens(case), seed=41)
    host = workloads.host_tensors(wl)
    ws = workspace_for(wl, P)
    kc, vc, ref = oracle_step(wl, host)
    for call in range(2):  # the second call reuses the workspace the first left behind
        dev = device_inputs(wl, host)
        out = gpu_step(wl, dev, partition_size=P, workspace=ws, fused=fused)
        assert to_host_bits(dev["k_cache"]).tobytes() == kc.tobytes()
        assert_attention_close(widen(out), ref, wl.dtype, f"{case} P={P} fused={fused} #{call}")
    assert pkv.device_errors() == 0


def test_length_order_with_empty_sequences():
    """Empty sequences are last partitions of 0 tokens: zero rows, nothing written."""
    lens = [5000, 300, 2048, 77, 7000, 1]
    wl = workloads.custom("ord0", "bf16", len(lens), 16, 4, 128, 16, lens, seed=43)
    host = workloads.host_tensors(wl)
    seq = wl.seq_lens_pre.astype(np.int32)  # a plain decode of the pre-step cache
    empty = [1, 3]
    seq[empty] = 0
    ws = workspace_for(wl, 2048)
    for call in range(2):
        dev = device_inputs(wl, host)
        dev["seq_lens"] = torch.from_numpy(seq).cuda()
        out = torch.full_like(dev["q"], float("nan"))
        pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"],
                                   dev["block_tables"], dev["seq_lens"], wl.max_seq_len,
                                   wl.scale, workspace=ws, partition_size=2048)
        ref = oracle.paged_decode(host["q"], host["k_cache"], host["v_cache"], wl.block_tables,
                                  seq, wl.scale)
        got = widen(out)
        assert_attention_close(got, ref, wl.dtype, f"empty sequences #{call}")
        assert np.all(got[empty] == 0.0)
    assert pkv.device_errors() == 0
