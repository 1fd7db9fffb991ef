"""Parity at the benchmark's full sizes, in the launch configuration ``bench.py`` times
(automatic partition length and kernel choice, one step = copy_blocks -> paged_kv_write ->
paged_attention_decode).

The oracle cannot run every output row at these sizes, so it checks sampled (sequence,
KV head) pairs: for each, its input is rebuilt from the generator's pre-step state (the
sequence's blocks before the step plus the new token, written by the oracle's own cache
update), never from what the GPU wrote.  The cache update and the copy-on-write copies are
checked bit for bit on every touched block, and every other block must be unchanged.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_344_b200 as pkv
from paged_kv_cache_344_b200 import workloads
from gpu_util import assert_attention_close, gpu_step, meta_to_device, raw, to_host_bits, widen

pytestmark = pytest.mark.gpu

FULL = [("mha", ""), ("gqa16", ""), ("gqa32", ""), ("long", ""), ("share_fork", ""),
        ("share_tails", ""), ("share_fork", "shared_prefix"), ("share_tails", "shared_prefix"),
        ("mha", "fused_step"), ("long", "fused_step"), ("share_fork", "fused_step"),
        ("share_fork", "fused_shared_prefix"), ("share_tails", "fused_shared_prefix")]


def _sample_units(wl, rng, n):
    lens = wl.seq_lens_post
    bs = [int(np.argmax(lens)), int(np.argmin(lens))]
    bs += list(rng.integers(0, wl.B, size=n - 2))
    return [(int(b), int(rng.integers(0, wl.Hkv))) for b in bs]


@pytest.mark.parametrize("name,entry", FULL, ids=[f"{n}-{e}" if e else n for n, e in FULL])
def test_fullsize_step(name, entry):
    torch.cuda.empty_cache()
    pkv.device_errors(clear=True)
    wl = workloads.make(name)
    dev = workloads.device_tensors(wl, "cuda")
    dev.update(meta_to_device(wl))
    rng = np.random.default_rng(2024)
    units = _sample_units(wl, rng, 12 if name == "long" else 24)

    # Pre-step state the oracle needs, captured before any kernel of ours runs.
    pre = {}
    for b, kvh in units:
        n_pre = -(-int(wl.seq_lens_pre[b]) // wl.bs)
        ids = torch.from_numpy(wl.block_tables_pre[b, :n_pre].astype(np.int64)).cuda()
        pre[(b, kvh)] = {k: to_host_bits(dev[k][ids][:, :, kvh:kvh + 1]) for k in ("k_cache", "v_cache")}
    touched = sorted(set(int(x) for x in wl.cow_pairs.reshape(-1)) |
                     set(int(s) // wl.bs for s in wl.slot_mapping if s >= 0))
    tid = torch.tensor(touched, dtype=torch.int64, device="cuda")
    before_touched = {k: to_host_bits(dev[k][tid]) for k in ("k_cache", "v_cache")}
    before_all = {k: dev[k].clone() for k in ("k_cache", "v_cache")}
    host_new = {k: to_host_bits(dev[k]) for k in ("q", "k_new", "v_new")}

    out = gpu_step(wl, dev, shared=entry.endswith("shared_prefix"), fused=entry.startswith("fused"))
    torch.cuda.synchronize()
    assert pkv.device_errors() == 0

    # 1) cache update + copy-on-write: oracle on a mini pool of the touched blocks.
    remap = {blk: i for i, blk in enumerate(touched)}
    pairs = np.array([[remap[int(s)], remap[int(d)]] for s, d in wl.cow_pairs], np.int64).reshape(-1, 2)
    slots = np.array([remap[int(s) // wl.bs] * wl.bs + int(s) % wl.bs for s in wl.slot_mapping],
                     np.int64)
    kc, vc = before_touched["k_cache"].copy(), before_touched["v_cache"].copy()
    assert oracle.copy_blocks(kc, vc, pairs) == 0
    assert oracle.kv_write(host_new["k_new"], host_new["v_new"], kc, vc, slots) == 0
    assert to_host_bits(dev["k_cache"][tid]).tobytes() == kc.tobytes()
    assert to_host_bits(dev["v_cache"][tid]).tobytes() == vc.tobytes()
    keep = torch.ones(wl.num_blocks, dtype=torch.bool, device="cuda")
    keep[tid] = False
    for k in ("k_cache", "v_cache"):
        assert torch.equal(raw(dev[k][keep]), raw(before_all[k][keep]))
    del before_all

    # 2) decode: sampled (b, kvh) units, all G heads each.
    G = wl.G
    got = widen(out)
    for b, kvh in units:
        L_pre = int(wl.seq_lens_pre[b])
        n_post = -(-(L_pre + 1) // wl.bs)
        kc = np.empty((n_post, wl.bs, 1, wl.D), dtype=pre[(b, kvh)]["k_cache"].dtype)
        vc = np.empty_like(kc)
        n_pre = pre[(b, kvh)]["k_cache"].shape[0]
        kc[:n_pre] = pre[(b, kvh)]["k_cache"]
        vc[:n_pre] = pre[(b, kvh)]["v_cache"]
        kc[n_pre:] = np.nan if kc.dtype == np.float32 else np.uint16(0x7FC0)
        vc[n_pre:] = kc[n_pre:]
        slot = np.array([L_pre], np.int64)  # identity table: logical block j is block j
        oracle.kv_write(np.ascontiguousarray(host_new["k_new"][b:b + 1, kvh:kvh + 1]),
                        np.ascontiguousarray(host_new["v_new"][b:b + 1, kvh:kvh + 1]), kc, vc, slot)
        q = np.ascontiguousarray(host_new["q"][b:b + 1, kvh * G:(kvh + 1) * G])
        ref = oracle.paged_decode(q, kc, vc, np.arange(n_post, dtype=np.int32)[None],
                                  np.array([L_pre + 1], np.int32), wl.scale)
        assert_attention_close(got[b:b + 1, kvh * G:(kvh + 1) * G], ref, wl.dtype,
                               f"{name} b={b} kvh={kvh} L={L_pre + 1}")
    assert np.isfinite(got).all()
