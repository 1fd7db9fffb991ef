"""Multi-query attention at the benchmark's full size, in the launch configuration
``bench.py --mode prefill`` times (persistent longest-first schedule with a workspace; the
one-CTA-per-item launch too).

Workload: 16 sequences, each appending 512 query tokens to U{0..4096} cached tokens,
Hq=32, Hkv=8, D=128, bs=16, bf16, K/V generated on the device.  The oracle cannot compute all
8192 x 32 rows, so it checks sampled query rows: a single query row of the multi-query
attention is the decode of that query over its visible prefix (tokens 0 .. L - Q + i), so the
oracle's decode of that row, over the sequence's blocks copied back from the device, is its
expected value.  Every output row must be finite.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, to_host_bits, widen

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("schedule", ["persistent", "per_item"])
def test_prefill_fullsize_sampled_rows(schedule):
    torch.cuda.empty_cache()
    pkv.device_errors(clear=True)
    wl, cu_q = workloads.prefill()
    dev = workloads.device_tensors(wl, "cuda")
    T = int(cu_q[-1])
    gen = torch.Generator(device="cuda")
    gen.manual_seed(4242)
    q = torch.randn((T, wl.Hq, wl.D), generator=gen, device="cuda").to(torch.bfloat16)
    out = torch.full_like(q, float("nan"))
    max_q = int(np.diff(cu_q).max())
    ws = None
    if schedule == "persistent":
        n = pkv.paged_attention_prefill_workspace_size(wl.B, wl.Hq, wl.Hkv, max_q)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    pkv.paged_attention_prefill(out, q, dev["k_cache"], dev["v_cache"],
                                torch.from_numpy(wl.block_tables).cuda(),
                                torch.from_numpy(wl.seq_lens_pre).cuda(),
                                torch.from_numpy(cu_q).cuda(), max_q,
                                int(wl.seq_lens_pre.max()), wl.scale, workspace=ws)
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0
    got = widen(out)
    assert np.isfinite(got).all()

    rng = np.random.default_rng(77)
    lens = wl.seq_lens_pre
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens))} |
                  set(int(x) for x in rng.choice(wl.B, size=4, replace=False)))
    q_host = to_host_bits(q)
    for b in seqs:
        L, Q = int(lens[b]), int(cu_q[b + 1] - cu_q[b])
        ctx = L - Q
        nblk = -(-L // wl.bs)
        ids = torch.from_numpy(wl.block_tables[b, :nblk].astype(np.int64)).cuda()
        kc = to_host_bits(dev["k_cache"][ids])
        vc = to_host_bits(dev["v_cache"][ids])
        table = np.arange(nblk, dtype=np.int32)[None]
        for i in sorted({0, Q - 1} | set(int(x) for x in rng.integers(0, Q, size=6))):
            row = int(cu_q[b]) + i
            ref = oracle.paged_decode(np.ascontiguousarray(q_host[row:row + 1]), kc, vc, table,
                                      np.array([ctx + i + 1], np.int32), wl.scale)
            assert_attention_close(got[row:row + 1], ref, "bf16",
                                   f"{schedule} b={b} i={i} visible={ctx + i + 1}")
