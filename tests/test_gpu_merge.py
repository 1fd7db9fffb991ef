"""GPU parity of the partition merge, on each of its paths.

The last CTA of a (sequence, KV head) merges the partitions' partials with a log-sum-exp
rescale.  With at most 32 partials each lane reads one partial's (max, sum); with more,
the weights take a loop over the partials; the output is then summed 16 partials at a
time plus a remainder.  When the weights do not fit in the shared memory the stages leave
free (partitions x heads above it), the merge sums the partials one at a time.  One long
sequence with G = 8 and partition lengths 2048, 64 and 16 runs each path, against the fp64
oracle, and twice on the same workspace, so that a ticket left behind would show.
"""
import pytest
import torch

import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, device_inputs, gpu_step, oracle_step, widen, workspace_for

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean():
    pkv.device_errors(clear=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("P,parts", [(2048, 20), (64, 626), (16, 2501)])
def test_merge_paths_match_oracle(P, parts):
    lens = [40000]  # 40001 tokens after the step
    wl = workloads.custom("merge", "bf16", len(lens), 64, 8, 128, 16, lens, seed=51)
    assert -(-int(wl.seq_lens_post[0]) // P) == parts
    host = workloads.host_tensors(wl)
    _, _, ref = oracle_step(wl, host)
    ws = workspace_for(wl, P)
    for call in range(2):
        dev = device_inputs(wl, host)
        out = gpu_step(wl, dev, partition_size=P, workspace=ws)
        assert_attention_close(widen(out), ref, wl.dtype, f"P={P} #{call}")
    assert pkv.device_errors() == 0
