"""Benchmark: one decode step of paged KV-cache attention on B200, per the benchmark contract.

A step is one pass of the whole hot path over one batch: copy-on-write block copies (when
the workload has any), the cache update of one new token per sequence, and the decode
attention.  Inputs are seeded synthetic tensors resident in HBM.  The JSON line reports

* ``value``: algorithmic bytes of the step / step time (GB/s), summed over ranks;
* ``tokens_per_s``: decode tokens (one per sequence) per second, summed over ranks;
* ``roofline``: the decode kernel alone against the measured HBM copy bandwidth.  Its
  launches run back to back between two CUDA events on its stream, each step on a pool of
  inputs that the previous step did not touch, and its time is the region's over the
  launches (a step of several launches times its decode with a pair of events instead);
* ``e2e``: the same metric through the public API with the step's inputs copied from pinned
  host memory and the output copied back, inside the timed region;
* ``cpu_baseline``: the fp64 oracle on this host's cores on a bounded sample (rank 0, N=1).

``--impl reference`` times the oracle (the CPU reference of this method) instead.
Multi-GPU (torchrun): every rank runs its own replica (weak scaling, no data-path
collective); ranks only agree on the barrier and on the max step time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_344_b200 import workloads  # noqa: E402

METRIC = "paged decode attention: achieved HBM GB/s (% of B200 peak) and decode tokens/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024

DESCR = {
    "tiny": "tiny fp32: B=4, lengths {1,7,16,33}+1, Hq=Hkv=4, D=64, bs=16, pool 32",
    "mha": "MHA bf16: B=64, Hq=Hkv=40, D=128, bs=16, seq_len U[128,2048]+1, pool 1.25x, shuffled",
    "gqa16": "GQA bf16: B=256, Hq=32, Hkv=8, D=128, bs=16, lognormal(1024,0.8) in [16,4096]+1",
    "gqa32": "GQA bf16: B=256, Hq=32, Hkv=8, D=128, bs=32, lognormal(1024,0.8) in [16,4096]+1",
    "long": "long-context GQA bf16: B=8, Hq=64, Hkv=8, D=128, bs=16, seq_len U[32768,131072]+1",
    "share_fork": "shared-prefix bf16: 32 groups x 4 branches, Hq=32, Hkv=8, D=128, bs=16, "
                  "prefix 1024+U[1,15] shared (refcount 4), CoW of the partial block",
    "share_tails": "shared-prefix bf16: 32 groups x 4 branches, Hq=32, Hkv=8, D=128, bs=16, "
                   "1024-token shared prefix + private tails U[0,256]",
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = {"decode": ("pkv_ptx.cuh", "pkv_decode.cuh"),
                  "shared": ("pkv_ptx.cuh", "pkv_decode.cuh", "pkv_decode_shared.cuh"),
                  "prefill": ("pkv_ptx.cuh", "pkv_decode.cuh", "pkv_prefill.cuh")}

# Decode workloads of the benchmark definition reported beside the headline, each timed
# the same way (``per_config``).
PER_CONFIG = ["mha", "gqa16", "gqa32", "long", "share_fork", "share_tails"]


def kernel_source_sha(kind: str = "decode") -> str:
    """Hash of the device-code sources a kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_344_b200", "csrc")
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


# A device-side wait enqueued right before each timed region.  While it runs, the host
# enqueues the first timed launches, so that host start-up work (the clock sampler's
# first NVML calls, the first launches' argument marshalling) never shows up inside the
# region as GPU idle time.  It lies outside the timed events.
PRIME_CYCLES = 4_000_000  # about 2 ms at 1965 MHz


def prime_queue():
    import torch
    torch.cuda._sleep(PRIME_CYCLES)


MAX_POOLS = 16


def pools_for(working_set: int) -> int:
    """How many copies of a decode workload's inputs the timed steps cycle through.

    A working set of 8 L2s or more is one pool.  A smaller one is replicated into enough
    pools (each with its own K/V caches, q and new tokens; the block tables, lengths and
    groups are shared, as a model's layers share them) that together they hold 8 L2s: step i
    runs on pool i mod R, so no step finds the previous one's blocks in L2, and the launches
    run back to back.  0: more than MAX_POOLS pools would be needed, and L2 is flushed
    between steps instead."""
    if working_set >= 8 * L2_BYTES:
        return 1
    n = -(-8 * L2_BYTES // max(working_set, 1))
    return n if n <= MAX_POOLS else 0


class L2Flush:
    """Evicts the L2 between timed steps: a write pass over a buffer twice the L2's size,
    then a read pass over a second one.  The write pass alone leaves the L2 full of dirty
    lines of its buffer, and their write-back then lands inside the next timed step (about
    3 us of a 37-52 us shared-prefix step, measured with the two orders interleaved on one
    B200).  After the read pass the L2 holds clean lines of a buffer the step never reads."""

    def __init__(self, dev_name):
        import torch
        n = 2 * L2_BYTES // 4
        self.w = torch.ones(n, dtype=torch.int32, device=dev_name)
        self.r = torch.ones(n, dtype=torch.int32, device=dev_name)
        self.sink = torch.empty((), dtype=torch.int64, device=dev_name)

    def __call__(self):
        import torch
        self.w.add_(1)
        torch.sum(self.r, dim=0, out=self.sink)


def recorded_traffic(config: str, partition: int, kind: str = "decode"):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel sources (and, for decode, the same partition length); else None."""
    prefix = "prefill" if kind == "prefill" else "decode"
    path = os.path.join(ROOT, "profiles", f"{prefix}_{config}_ncu.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    q = re.search(r"partition_tokens:\s*([0-9]+)", text)
    if not m or not s or s.group(1) != kernel_source_sha(kind):
        return None
    if kind in ("decode", "shared") and (not q or int(q.group(1)) != partition):
        return None
    return float(m.group(1))


# ----------------------------------------------------------------------------------------
# multi-GPU plumbing: replicas only (no data-path collective); ranks agree on the max time
# ----------------------------------------------------------------------------------------
def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank device-timed value over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the bytes every rank moved over the slowest rank's time."""
    return world * bytes_per_step_per_rank * steps / (max_ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled in a thread)
# ----------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz, self.ok = [], 0, None, False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            # The first queries of a process are slow and can hold up the next kernel
            # launch; take them here, before any timed region starts.
            pynvml.nvmlDeviceGetClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._reasons()
            self.ok = True
        except Exception as e:  # no NVML: report clocks as unavailable
            self.err = str(e)

    def _handle(self, idx):
        import torch
        nv = self.nv
        try:
            p = torch.cuda.get_device_properties(idx)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId_v2(bus.encode())
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return f(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons())
            except Exception:
                pass
            self._first.set()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._first = threading.Event()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            self._first.wait(1.0)  # the thread's start-up lies before the timed region
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}

    def rejected(self):
        s = self.summary()
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
        if bad & set(s["reasons"]):
            return True
        return bool(s["sm_mhz"] and s["sm_max_mhz"] and s["sm_mhz"] < 0.5 * s["sm_max_mhz"]
                    and not s["reasons"])


# ----------------------------------------------------------------------------------------
# CPU side: the oracle on a bounded sample
# ----------------------------------------------------------------------------------------
def oracle_sample_size(wl, budget_rows: int) -> int:
    """Sequences 0..n-1 whose query-row x token work stays under ``budget_rows``."""
    acc, n = 0, 0
    for b in range(wl.B):
        acc += int(wl.seq_lens_post[b]) * wl.Hq
        n = b + 1
        if acc >= budget_rows:
            break
    return n


def sample_bytes(wl, sample) -> int:
    """Algorithmic bytes of the sample's decode (its distinct blocks once, q, out, tables)."""
    nb = sample["k_cache"].shape[0]
    n = sample["q"].shape[0]
    tables = sum(-(-int(L) // wl.bs) for L in sample["seq_lens"])
    return int(nb * wl.block_bytes * 2 + 2 * n * wl.Hq * wl.D * wl.elt + tables * 4 + 4 * n)


def time_oracle(wl, sample):
    """Seconds of one fp64 oracle decode of the sample, its bytes, tokens and threads."""
    import oracle
    t0 = time.perf_counter()
    oracle.paged_decode(sample["q"], sample["k_cache"], sample["v_cache"],
                        sample["block_tables"], sample["seq_lens"], wl.scale)
    dt = time.perf_counter() - t0
    return dt, sample_bytes(wl, sample), int(sample["seq_lens"].sum()), oracle.num_threads()


def cpu_baseline_of(wl, dev, budget_rows: int):
    """The oracle on sequences 0..n-1 of the workload, over their blocks gathered from the
    device pool after the step (so the sample is the step's own post-step state)."""
    import torch
    n_seq = oracle_sample_size(wl, budget_rows)
    sample = workloads.compact_sample(wl, n_seq, dev["k_cache"], dev["v_cache"])
    q = dev["q"][:n_seq].detach().cpu().contiguous()
    sample["q"] = q.view(torch.int16).numpy().view(np.uint16) if q.dtype == torch.bfloat16 \
        else q.numpy()
    dt, nbytes, tokens, cores = time_oracle(wl, sample)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"decode of sequences 0..{n_seq - 1} of {wl.B} ({tokens} cached tokens, "
                      f"{n_seq * wl.Hq} query rows, {sample['k_cache'].shape[0]} distinct blocks),"
                      f" fp64, {dt:.2f} s",
            "tokens_per_s": round(n_seq / dt, 3)}


# ----------------------------------------------------------------------------------------
# GPU side
# ----------------------------------------------------------------------------------------
def config_dict(args, name, wl, fused: bool, use_shared: bool, has_cow: bool, world: int):
    """The workload's description; both arms report the same dict."""
    step_bytes = (workloads.decode_algorithmic_bytes(wl) + workloads.write_bytes(wl) +
                  workloads.copy_bytes(wl))
    working_set = workloads.decode_algorithmic_bytes(wl)
    pools = pools_for(working_set)
    entry = "paged_attention_decode_shared_prefix" if use_shared else "paged_attention_decode"
    return {"workload": name, "description": DESCR.get(name, name),
            "step": (("paged_decode_step_shared_prefix" if use_shared else "paged_decode_step")
                     + " (copy-on-write + cache write + decode in one launch)" if fused else
                     ("copy_blocks + " if has_cow else "") + "paged_kv_write + " + entry),
            "bytes_per_step": step_bytes,
            "l2": (f"flushed between steps: a write pass, then a read pass, over two 0.26 GB buffers "
                   f"(working set {working_set / 1e9:.2f} GB)" if pools == 0 else
                   f"inputs larger than L2 ({working_set / 1e9:.2f} GB vs 0.13 GB L2)" if pools == 1
                   else f"inputs larger than L2: {pools} pools of {working_set / 1e9:.2f} GB (own K/V, "
                        f"q and new tokens; shared tables), step i on pool i mod {pools}"),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "block_size": wl.bs, "placement": "contiguous" if args.contiguous else "shuffled"}


def run_decode(args, name, rank, world, local_rank, steps, warmup, with_e2e, with_cpu):
    """One workload: warm-up, ``steps`` timed decode steps (device events on the launching
    stream), optionally the end-to-end pipelined measurement and the oracle baseline."""
    import torch
    import torch.distributed as dist
    import paged_kv_cache_344_b200 as pkv

    dev_name = f"cuda:{local_rank}"
    wl = workloads.make(name, block_size=args.block_size or None, contiguous=args.contiguous,
                        dtype=args.dtype or None)
    dev = workloads.device_tensors(wl, dev_name, seed_offset=rank)
    meta = {
        "block_tables": torch.from_numpy(wl.block_tables).to(dev_name),
        "seq_lens": torch.from_numpy(wl.seq_lens_post).to(dev_name),
        "slot_mapping": torch.from_numpy(wl.slot_mapping).to(dev_name),
        "cow_pairs": torch.from_numpy(wl.cow_pairs).to(dev_name),
    }
    use_shared = args.decode == "shared_prefix" or (args.decode == "auto"
                                                    and name.startswith("share"))
    if use_shared:
        ws_bytes = pkv.paged_attention_decode_shared_prefix_workspace_size(
            wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len, wl.bs, args.partition)
        meta["group_offsets"] = torch.from_numpy(wl.group_offsets).to(dev_name)
        meta["prefix_lens"] = torch.from_numpy(wl.prefix_lens).to(dev_name)
        max_group = int(np.diff(wl.group_offsets).max())
    else:
        ws_bytes = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D,
                                                             wl.max_seq_len, wl.bs, args.partition)
    part = pkv.paged_attention_decode_partition_size(wl.B, wl.Hkv, wl.max_seq_len, wl.bs,
                                                     args.partition)
    ws = torch.zeros(max(ws_bytes, 1), dtype=torch.uint8, device=dev_name)
    out = torch.empty_like(dev["q"])
    has_cow = len(wl.cow_pairs) > 0
    launches_per_step = 1 if args.step == "fused" else 2 + int(has_cow)
    stream = torch.cuda.current_stream()

    # The CoW step restores its own precondition: copying block src -> dst again is
    # idempotent, and rewriting the same token to the same slot is too.
    fused = args.step == "fused"
    if fused:
        meta["cow_src"] = torch.from_numpy(wl.cow_src).to(dev_name)

    def step(d_in, ev_pair=None, outbuf=None):
        o = out if outbuf is None else outbuf
        if fused:
            if ev_pair is not None:
                ev_pair[0].record(stream)
            cow = d_in["cow_src"] if has_cow else None
            if use_shared:
                pkv.paged_decode_step_shared_prefix(
                    o, d_in["q"], d_in["k_new"], d_in["v_new"], d_in["k_cache"],
                    d_in["v_cache"], d_in["block_tables"], d_in["seq_lens"], wl.max_seq_len,
                    wl.scale, d_in["group_offsets"], d_in["prefix_lens"], max_group,
                    cow_src=cow, workspace=ws, partition_size=args.partition)
            else:
                pkv.paged_decode_step(o, d_in["q"], d_in["k_new"], d_in["v_new"], d_in["k_cache"],
                                      d_in["v_cache"], d_in["block_tables"], d_in["seq_lens"],
                                      wl.max_seq_len, wl.scale, cow_src=cow, workspace=ws,
                                      partition_size=args.partition)
            if ev_pair is not None:
                ev_pair[1].record(stream)
            return
        if has_cow:
            pkv.copy_blocks(d_in["k_cache"], d_in["v_cache"], d_in["cow_pairs"])
        pkv.paged_kv_write(d_in["k_new"], d_in["v_new"], d_in["k_cache"], d_in["v_cache"],
                           d_in["slot_mapping"])
        if ev_pair is not None:
            ev_pair[0].record(stream)
        if use_shared:
            pkv.paged_attention_decode_shared_prefix(
                o, d_in["q"], d_in["k_cache"], d_in["v_cache"], d_in["block_tables"],
                d_in["seq_lens"], wl.max_seq_len, wl.scale, d_in["group_offsets"],
                d_in["prefix_lens"], max_group, workspace=ws, partition_size=args.partition)
        else:
            pkv.paged_attention_decode(o, d_in["q"], d_in["k_cache"], d_in["v_cache"],
                                       d_in["block_tables"], d_in["seq_lens"], wl.max_seq_len,
                                       wl.scale, workspace=ws, partition_size=args.partition)
        if ev_pair is not None:
            ev_pair[1].record(stream)

    d_in = dict(dev)
    d_in.update(meta)
    cfg = config_dict(args, name, wl, fused, use_shared, has_cow, world)
    step_bytes = cfg["bytes_per_step"]
    decode_bytes = workloads.decode_algorithmic_bytes(wl)
    n_pools = pools_for(decode_bytes)
    flush = n_pools == 0
    flush_l2 = L2Flush(dev_name) if flush else None
    d_ins = [d_in]
    for r in range(1, n_pools):
        d_r = workloads.device_tensors(wl, dev_name, seed_offset=rank + 1000 * r)
        d_r.update(meta)
        d_ins.append(d_r)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for i in range(max(warmup, len(d_ins))):  # every pool at least once
        step(d_ins[i % len(d_ins)])
    prime_queue()  # its first launch loads the kernel; not inside a timed region
    if flush:
        flush_l2()  # likewise the flush's kernels, which run before every timed step
    barrier()

    # Timing events cost GPU time.  On the long-context workload a pair recorded around
    # every fused launch added about 5 us a step, and the event just before a launch
    # lengthened the launch it bracketed (367.4 us a step with no per-step events, 372.9 with
    # one pair, 378.1 with two; the launch itself read 370.3 inside its pair).  So when a
    # step is one launch and nothing runs between steps, the region holds only those
    # launches back to back and region / K is the launch's average duration, the gaps
    # between launches included: no per-step event is recorded.  With a flush between
    # steps one pair brackets each fused launch; a step of several launches also gets a
    # pair around its decode alone.
    per_step_events = flush or not fused

    def timed_region():
        ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(steps)]
        ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        # A CUDA event is created at its first record; the first creations of a process
        # are slow.  Record every event once here, so that none is created between a
        # step's launch and its end event inside the region.
        for a, b in ev_dec + ev_step + [(t_start, t_end)]:
            a.record(stream)
            b.record(stream)
        barrier()
        with ClockSampler(local_rank) as clocks:
            torch.cuda.nvtx.range_push("timed_region")
            prime_queue()
            t_start.record(stream)
            for i in range(steps):
                if flush:
                    flush_l2()  # evict the previous step's blocks from L2 (untimed below)
                d_i = d_ins[i % len(d_ins)]
                if not per_step_events:
                    step(d_i)
                elif fused:
                    step(d_i, ev_dec[i])  # the step is this one launch
                else:
                    ev_step[i][0].record(stream)
                    step(d_i, ev_dec[i])
                    ev_step[i][1].record(stream)
            t_end.record(stream)
            torch.cuda.nvtx.range_pop()
            barrier()
        region_ms = t_start.elapsed_time(t_end)
        if not per_step_events:
            return region_ms, [region_ms / steps] * steps, clocks
        dec_ms = [a.elapsed_time(b) for a, b in ev_dec]
        step_ms = dec_ms if fused else [a.elapsed_time(b) for a, b in ev_step]
        total_ms = sum(step_ms) if flush else region_ms
        return total_ms, dec_ms, clocks

    total_ms, dec_ms, clocks = timed_region()
    remeasured = False
    if clocks.rejected():
        total_ms, dec_ms, clocks = timed_region()
        remeasured = True

    # max over ranks (device-timed)
    total_ms_max = max_over_ranks(total_ms, world, dev_name)
    ms_per_step = total_ms_max / steps
    value = whole_job_gbs(step_bytes, steps, world, total_ms_max)
    tokens_per_s = world * wl.B * steps / (total_ms_max * 1e-3)

    peak, peak_src = load_peaks()
    dec_avg_ms = statistics.fmean(dec_ms)
    kernel_bytes = step_bytes if fused else decode_bytes  # the fused kernel also writes/copies
    achieved = kernel_bytes / (dec_avg_ms * 1e-3) / 1e9
    tc = wl.dtype == "bf16" and (args.path != "cuda_cores" or wl.G > 8)
    grouped = use_shared and args.partition == 0 and int(np.diff(wl.group_offsets).max()) <= \
        max(1, 16 // wl.G)
    kernel = ("paged_decode_group_kernel" if grouped else
              "paged_decode_shared_kernel" if use_shared else
              "paged_decode_kernel" if fused else
              "paged_decode_balanced_kernel" if args.split == "balanced" else "paged_decode_kernel") \
        + ("<MmaConsumer>" if tc else "<SimtConsumer>")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4),
                "traffic": recorded_traffic(name, part, "shared" if use_shared else "decode"),
                "kernel": kernel, "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                "frac_of_8TBps_spec": round(achieved / SPEC_HBM_GBS, 4),
                "decode_us": round(dec_avg_ms * 1e3, 2),
                "launch_time": ("CUDA events around each launch" if per_step_events else
                                "timed region / steps (launches back to back, no per-step events)"),
                "algorithmic_bytes_per_launch": kernel_bytes,
                "achieved_token_exact": round(workloads.decode_token_bytes(wl) / (dec_avg_ms * 1e-3) / 1e9, 1)}
    res = {"value": round(value, 1), "ms_per_step": round(ms_per_step, 5),
           "tokens_per_s": round(tokens_per_s, 1), "config": cfg,
           "launch": {"decode_entry": "paged_attention_decode_shared_prefix" if use_shared
                      else "paged_attention_decode", "decode_path": args.path,
                      "decode_split": args.split, "partition_tokens": part},
           "roofline": roofline, "gpu_launches": launches_per_step * steps,
           "clocks": clocks.summary(), "dtype": wl.dtype}
    if remeasured:
        res["clocks"]["remeasured"] = True

    if with_e2e:
        res["e2e"] = run_e2e(step, d_in, out, has_cow, stream, step_bytes, wl, world, dev_name,
                             steps, warmup, barrier)
    res["cpu_baseline"] = None
    if with_cpu and rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_of(wl, dev, args.cpu_budget_rows)
    return res


def run_e2e(step, d_in, out, has_cow, stream, step_bytes, wl, world, dev_name, steps, warmup,
            barrier):
    """e2e through the public API: every step copies its inputs from pinned host memory and
    reads its output back.  As in a serving loop, the copies of step i+1's inputs and of
    step i's output run on a copy stream and overlap the computation of step i (two sets
    of step buffers; the KV cache itself stays resident)."""
    import torch
    in_keys = [k for k in ("q", "k_new", "v_new", "block_tables", "seq_lens", "slot_mapping",
                           "cow_pairs", "group_offsets", "prefix_lens", "cow_src")
               if k in d_in and (k != "cow_pairs" or has_cow)]
    host_in = {k: d_in[k].cpu().pin_memory() for k in in_keys}
    bufs = [dict(d_in), dict(d_in)]
    for k in in_keys:
        bufs[1][k] = torch.empty_like(d_in[k])
    outs = [torch.empty_like(out), torch.empty_like(out)]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(host_in[k].numel() * host_in[k].element_size() for k in in_keys)
    d2h = host_out[0].numel() * host_out[0].element_size()
    copy_s = torch.cuda.Stream()
    ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("h2d", "comp", "d2h")}

    def h2d_(i):
        j = i % 2
        with torch.cuda.stream(copy_s):
            if i >= 2:
                copy_s.wait_event(ev["comp"][j])  # step i-2 has read buffer set j
            for k in in_keys:
                bufs[j][k].copy_(host_in[k], non_blocking=True)
            ev["h2d"][j].record(copy_s)

    def comp_(i):
        j = i % 2
        stream.wait_event(ev["h2d"][j])
        if i >= 2:
            stream.wait_event(ev["d2h"][j])  # output j of step i-2 has been read back
        step(bufs[j], outbuf=outs[j])
        ev["comp"][j].record(stream)

    def d2h_(i):
        j = i % 2
        with torch.cuda.stream(copy_s):
            copy_s.wait_event(ev["comp"][j])
            host_out[j].copy_(outs[j], non_blocking=True)
            ev["d2h"][j].record(copy_s)

    def e2e_run(n):
        h2d_(0)
        for i in range(n):
            if i + 1 < n:
                h2d_(i + 1)
            comp_(i)
            d2h_(i)

    e2e_run(max(3, warmup // 4))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)  # created now, not inside the region
    e1.record(stream)
    barrier()
    e2e_steps = max(10, steps)
    with torch.cuda.stream(copy_s):
        prime_queue()  # the host queues the first steps while the copy stream waits
    e0.record(copy_s)
    e2e_run(e2e_steps)
    e1.record(copy_s)
    barrier()
    e2e_ms_max = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev_name)
    return {"value": round(whole_job_gbs(step_bytes, 1, world, e2e_ms_max), 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": round(e2e_ms_max, 5),
            "tokens_per_s": round(world * wl.B / (e2e_ms_max * 1e-3), 1),
            "pipelining": "inputs of step i+1 and output of step i copied on a second "
                          "stream while step i computes"}


def run_ours(args, rank, world, local_rank):
    """The headline workload with its e2e and oracle legs, then every other decode workload
    of the benchmark definition as a ``per_config`` entry."""
    import torch
    import paged_kv_cache_344_b200 as pkv

    torch.cuda.set_device(local_rank)
    pkv.set_decode_path({"auto": pkv.PKV_PATH_AUTO, "cuda_cores": pkv.PKV_PATH_CUDA_CORES,
                         "tensor_cores": pkv.PKV_PATH_TENSOR_CORES}[args.path])
    pkv.set_decode_split(pkv.PKV_SPLIT_BALANCED if args.split == "balanced" else pkv.PKV_SPLIT_FIXED)
    head = run_decode(args, args.config, rank, world, local_rank, args.steps, args.warmup,
                      with_e2e=True, with_cpu=True)
    peak = head["roofline"]["peak"]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
        "data": "synthetic (seeded N(0,1) q/K/V, shuffled block pool, NaN in unused slots)",
        "tokens_per_s": head["tokens_per_s"],
        "pct_of_8TBps_spec": round(100 * head["value"] / world / SPEC_HBM_GBS, 2),
        "pct_of_measured_peak": round(100 * head["value"] / world / peak, 2),
        "config": head["config"], "launch": head["launch"], "roofline": head["roofline"],
        "cpu_baseline": head["cpu_baseline"], "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"], "clocks": head["clocks"],
    }
    if not args.no_per_config:
        per = {}
        for name in PER_CONFIG:
            if name == args.config:
                continue
            torch.cuda.empty_cache()
            r = run_decode(args, name, rank, world, local_rank, args.steps, args.warmup,
                           with_e2e=False, with_cpu=True)
            per[name] = {"value": r["value"], "unit": "GB/s", "ms_per_step": r["ms_per_step"],
                         "tokens_per_s": r["tokens_per_s"], "config": r["config"],
                         "launch": r["launch"], "roofline": r["roofline"],
                         "cpu_baseline": r["cpu_baseline"], "gpu_launches": r["gpu_launches"],
                         "clocks": r["clocks"]}
        line["per_config"] = per
    return line


def run_prefill(args, rank, world, local_rank):
    """Multi-query (chunked append) attention on the tcgen05 kernel: TFLOP/s."""
    import torch
    import paged_kv_cache_344_b200 as pkv
    torch.cuda.set_device(local_rank)
    dev_name = f"cuda:{local_rank}"
    wl, cu_q = workloads.prefill()
    dev = workloads.device_tensors(wl, dev_name, seed_offset=rank)
    T = int(cu_q[-1])
    gen = torch.Generator(device=dev_name)
    gen.manual_seed(4242 + rank)
    q = torch.randn((T, wl.Hq, wl.D), generator=gen, device=dev_name).to(torch.bfloat16)
    out = torch.empty_like(q)
    bt = torch.from_numpy(wl.block_tables).to(dev_name)
    seq = torch.from_numpy(wl.seq_lens_pre).to(dev_name)
    cu = torch.from_numpy(cu_q).to(dev_name)
    max_q = int(np.diff(cu_q).max())
    stream = torch.cuda.current_stream()
    pkv.set_prefill_path(pkv.PKV_PREFILL_SINGLE_TILE if args.prefill_kernel == "single_tile"
                         else pkv.PKV_PREFILL_AUTO)
    ws = None
    if args.prefill_kernel == "two_tile":  # persistent, longest-first schedule
        n = pkv.paged_attention_prefill_workspace_size(wl.B, wl.Hq, wl.Hkv, int(np.diff(cu_q).max()))
        ws = torch.empty(n, dtype=torch.uint8, device=dev_name)

    def step():
        pkv.paged_attention_prefill(out, q, dev["k_cache"], dev["v_cache"], bt, seq, cu, max_q,
                                    int(wl.seq_lens_pre.max()), wl.scale, workspace=ws)

    for _ in range(args.warmup):
        step()
    prime_queue()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)  # created now, not inside the region
    e1.record(stream)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        prime_queue()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev_name)
    flops = workloads.prefill_flops(wl, cu_q)
    tflops = world * flops / (ms * 1e-3) / 1e12

    # End to end through the same call: every step copies its q from pinned host memory to
    # the device and reads its output back into pinned host memory.  Two buffer sets and two
    # copy streams (one per direction) overlap step i's attention with the copy of step i+1's
    # q and of step i-1's output.
    q_host = q.cpu().pin_memory()
    out_host = [torch.empty_like(q_host).pin_memory() for _ in range(2)]
    q_dev, out_dev = [q, q.clone()], [out, torch.empty_like(out)]
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("h2d", "comp", "d2h")}

    def step_on(j):
        pkv.paged_attention_prefill(out_dev[j], q_dev[j], dev["k_cache"], dev["v_cache"], bt, seq,
                                    cu, max_q, int(wl.seq_lens_pre.max()), wl.scale, workspace=ws)

    def e2e_run(n):
        for i in range(n + 1):
            if i < n:  # copy in step i's q
                j = i % 2
                with torch.cuda.stream(h2d_s):
                    if i >= 2:
                        h2d_s.wait_event(ev["comp"][j])  # step i-2 has finished reading q_dev[j]
                    q_dev[j].copy_(q_host, non_blocking=True)
                    ev["h2d"][j].record(h2d_s)
            if i >= 1:  # compute step i-1, then copy its output out
                jj = (i - 1) % 2
                stream.wait_event(ev["h2d"][jj])
                if i - 1 >= 2:
                    stream.wait_event(ev["d2h"][jj])  # out_dev[jj] of step i-3 has been read
                step_on(jj)
                ev["comp"][jj].record(stream)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(ev["comp"][jj])
                    out_host[jj].copy_(out_dev[jj], non_blocking=True)
                    ev["d2h"][jj].record(d2h_s)

    e_steps = max(3, min(args.steps, 50))
    e2e_run(2)
    torch.cuda.synchronize()
    e0.record(stream)
    h2d_s.wait_event(e0)  # no copy of the timed steps starts before the region does
    e2e_run(e_steps)
    for k in range(2):  # the end of the timed region waits for the last read-backs
        stream.wait_event(ev["d2h"][k])
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev_name)
    qbytes = q.numel() * q.element_size()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, f_s, n_s, cores = prefill_oracle_sample(wl, cu_q, dev, q, args.cpu_budget_flops)
        cpu = {"value": round(f_s / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
               "kind": "oracle",
               "sample": f"multi-query attention of sequences 0..{n_s - 1} of {wl.B} "
                         f"({f_s / 1e9:.1f} GFLOP), fp64, {dt:.2f} s"}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured bf16_tflops (burst)"
    except Exception:
        peak, src = 1590.0, "fallback"
    return {"metric": "paged multi-query (chunked append) attention: TFLOP/s",
            "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "prefill: B=16, chunk 512 appended to U{0..4096} cached tokens, "
                                   "Hq=32, Hkv=8, D=128, bs=16", "flops_per_step": flops},
            "roofline": {"bound": "tensor", "achieved": round(tflops / world, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tflops / world / peak, 4),
                         "traffic": (recorded_traffic("chunked_append", 0, "prefill")
                                     if args.prefill_kernel == "two_tile" else None),
                         "peak_source": src,
                         "kernel": ("paged_prefill_kernel" if args.prefill_kernel == "single_tile"
                                    else "paged_prefill_pp_kernel"),
                         "schedule": args.prefill_kernel},
            "cpu_baseline": cpu,
            "e2e": {"value": round(world * flops / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": qbytes, "d2h_bytes_per_step": qbytes,
                    "ms_per_step": round(e_ms, 4),
                    "pipelining": "q of step i+1 and output of step i-1 copied on two copy "
                                  "streams while step i computes"},
            "gpu_launches": args.steps * (2 if ws is not None else 1),
            "clocks": clocks.summary()}


def run_paging(args, local_rank):
    """The paging-overhead control and the block-size sweep ([Index] "Limitations": the
    block-table walk may cost a little against a contiguous allocation; [Explained] "2.
    Partial Block Waste": block size trades wasted slots against management overhead).
    For each workload: the decode alone (CUDA events on its stream) over the shuffled pool,
    over a pool whose blocks are laid out in order, with the table-free kernel on the same
    logical K/V as the shuffled pool, and over shuffled pools of 8/16/32/64-token blocks."""
    import torch
    import paged_kv_cache_344_b200 as pkv
    torch.cuda.set_device(local_rank)
    dev_name = f"cuda:{local_rank}"
    flush_l2 = L2Flush(dev_name)

    def time_decode(fn, nbytes):
        flush = nbytes < 8 * L2_BYTES
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        prime_queue()
        for a, b in ev:
            if flush:
                flush_l2()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.median(x.elapsed_time(y) for x, y in ev) * 1e3

    def paged(name, **kw):
        wl = workloads.make(name, **kw)
        dev = workloads.device_tensors(wl, dev_name)
        bt = torch.from_numpy(wl.block_tables).to(dev_name)
        sl = torch.from_numpy(wl.seq_lens_post).to(dev_name)
        n = pkv.paged_attention_decode_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.D, wl.max_seq_len,
                                                      wl.bs, 0)
        ws = torch.zeros(max(n, 1), dtype=torch.uint8, device=dev_name)
        out = torch.empty_like(dev["q"])

        def fn():
            pkv.paged_attention_decode(out, dev["q"], dev["k_cache"], dev["v_cache"], bt, sl,
                                       wl.max_seq_len, wl.scale, workspace=ws)
        return wl, dev, ws, fn

    res = {}
    for name in args.paging_configs.split(","):
        r = {}
        wl, dev, ws, fn = paged(name)
        r["bytes_per_call"] = workloads.decode_algorithmic_bytes(wl)
        r["token_bytes_per_call"] = workloads.decode_token_bytes(wl)
        r["shuffled_us"] = round(time_decode(fn, r["bytes_per_call"]), 2)
        # the same logical K/V, unpaged: [B, stride, Hkv, D] and no table at all
        stride = wl.max_seq_len
        cont = []
        for key in ("k_cache", "v_cache"):
            c = torch.zeros((wl.B, stride, wl.Hkv, wl.D), dtype=dev[key].dtype, device=dev_name)
            for b in range(wl.B):
                L = int(wl.seq_lens_post[b])
                nb = -(-L // wl.bs)
                ids = torch.from_numpy(wl.block_tables[b, :nb].astype(np.int64)).to(dev_name)
                c[b, :L] = dev[key][ids].reshape(nb * wl.bs, wl.Hkv, wl.D)[:L]
            cont.append(c)
        del dev
        torch.cuda.empty_cache()
        q = torch.randn((wl.B, wl.Hq, wl.D), device=dev_name).to(cont[0].dtype)
        out = torch.empty_like(q)
        sl = torch.from_numpy(wl.seq_lens_post).to(dev_name)

        def fn_c():
            pkv.paged_attention_decode_contiguous(out, q, cont[0], cont[1], sl, wl.max_seq_len,
                                                  wl.scale, workspace=ws)
        r["table_free_us"] = round(time_decode(fn_c, r["bytes_per_call"]), 2)
        del cont
        torch.cuda.empty_cache()
        _, _, _, fn_o = paged(name, contiguous=True)
        r["in_order_pool_us"] = round(time_decode(fn_o, r["bytes_per_call"]), 2)
        torch.cuda.empty_cache()
        r["paging_overhead_vs_table_free"] = round(r["shuffled_us"] / r["table_free_us"] - 1, 4)
        sweep = {}
        for bs in (8, 16, 32, 64):
            wlb, devb, _, fnb = paged(name, block_size=bs)
            nbytes = workloads.decode_algorithmic_bytes(wlb)
            us = time_decode(fnb, nbytes)
            sweep[str(bs)] = {"decode_us": round(us, 2), "algorithmic_bytes": nbytes,
                              "GBs": round(nbytes / (us * 1e-6) / 1e9, 1),
                              "GBs_token_exact": round(workloads.decode_token_bytes(wlb) /
                                                       (us * 1e-6) / 1e9, 1),
                              "unused_slot_fraction": round(
                                  1 - workloads.decode_token_bytes(wlb) / nbytes, 4)}
            del devb
            torch.cuda.empty_cache()
        r["block_size_sweep"] = sweep
        res[name] = r
    return {"metric": "paging overhead (table-free control) and block-size sweep: decode us",
            "unit": "us", "steps": args.steps, "warmup": args.warmup, "per_config": res}


def prefill_oracle_sample(wl, cu_q, dev, q, budget_flops: float):
    """The fp64 oracle's multi-query attention on sequences 0..n-1 (cumulative causal flops
    up to ``budget_flops``), over a compact host pool of just their blocks; returns
    (seconds, flops, n, threads)."""
    import torch
    import oracle
    sel, acc = [], 0
    for b in range(wl.B):
        L, Q = int(wl.seq_lens_pre[b]), int(cu_q[b + 1] - cu_q[b])
        acc += 4 * wl.D * wl.Hq * ((L - Q) * Q + Q * (Q + 1) // 2)
        sel.append(b)
        if acc >= budget_flops:
            break
    kc, vc, tables, off = [], [], [], 0
    nmax = max(-(-int(wl.seq_lens_pre[b]) // wl.bs) for b in sel)
    for b in sel:
        n = -(-int(wl.seq_lens_pre[b]) // wl.bs)
        ids = torch.from_numpy(wl.block_tables[b, :n].astype(np.int64)).to(dev["k_cache"].device)
        kc.append(dev["k_cache"][ids].cpu())
        vc.append(dev["v_cache"][ids].cpu())
        row = np.full(nmax, -1, np.int32)
        row[:n] = np.arange(off, off + n, dtype=np.int32)
        tables.append(row)
        off += n

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    kc, vc = bits(torch.cat(kc)), bits(torch.cat(vc))
    qh = bits(q[int(cu_q[0]):int(cu_q[len(sel)])].cpu())
    cu = np.ascontiguousarray(cu_q[:len(sel) + 1] - cu_q[0]).astype(np.int32)
    seq = np.ascontiguousarray(wl.seq_lens_pre[:len(sel)]).astype(np.int32)
    t0 = time.perf_counter()
    oracle.paged_prefill(qh, kc, vc, np.stack(tables), seq, cu, wl.scale)
    return time.perf_counter() - t0, acc, len(sel), oracle.num_threads()


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on this host's cores, each step a bounded sample
    of the same workload (the blocks of its first sequences, drawn on the host)."""
    if rank != 0:
        return None
    wl = workloads.make(args.config, block_size=args.block_size or None,
                        contiguous=args.contiguous, dtype=args.dtype or None)
    n_seq = oracle_sample_size(wl, args.cpu_budget_rows // max(args.steps, 1))
    sample = workloads.compact_sample(wl, n_seq)
    nw = max(1, n_seq // 8)  # warm-up: the first sequences of the same sample
    warm = dict(sample, q=sample["q"][:nw], block_tables=sample["block_tables"][:nw],
                seq_lens=sample["seq_lens"][:nw])
    for _ in range(args.warmup):
        time_oracle(wl, warm)
    total_t, total_b, cores = 0.0, 0, 1
    for _ in range(args.steps):
        dt, nb, _, cores = time_oracle(wl, sample)
        total_t += dt
        total_b += nb
    val = total_b / total_t / 1e9
    use_shared = args.decode == "shared_prefix" or (args.decode == "auto"
                                                    and args.config.startswith("share"))
    cfg = config_dict(args, args.config, wl, args.step == "fused", use_shared,
                      len(wl.cow_pairs) > 0, world)
    sample_txt = (f"decode of sequences 0..{n_seq - 1} of {wl.B} per step "
                  f"({sample['k_cache'].shape[0]} distinct blocks), fp64")
    return {"impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total_t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample_txt},
            "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="long", choices=sorted(DESCR),
                    help="headline workload (default: the long-context GQA decode, the largest "
                         "single-GPU configuration)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the headline workload (no per_config entries)")
    ap.add_argument("--cpu-budget-rows", type=int, default=400_000_000,
                    help="query-row x token budget of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-flops", type=float, default=1.5e10,
                    help="prefill mode: causal flops of the oracle's timed sample")
    ap.add_argument("--mode", choices=["decode", "prefill", "paging"], default="decode",
                    help="decode step (default), multi-query chunked-append attention, or the "
                         "paging-overhead control and block-size sweep")
    ap.add_argument("--paging-configs", default="mha,gqa16,long",
                    help="paging mode: the workloads to measure")
    ap.add_argument("--prefill-kernel", choices=["two_tile", "per_item", "single_tile"],
                    default="two_tile",
                    help="prefill kernel: warp-specialised two-tile, persistent with the "
                         "longest-first schedule (default); the same, one CTA per item; or "
                         "single-tile")
    ap.add_argument("--path", choices=["auto", "cuda_cores", "tensor_cores"], default="auto",
                    help="decode kernel family (library default: auto)")
    ap.add_argument("--decode", choices=["auto", "plain", "shared_prefix"], default="auto",
                    help="decode entry point (auto: shared-prefix decode for the shared-prefix "
                         "workloads, the plain decode otherwise)")
    ap.add_argument("--block-size", type=int, default=0,
                    help="override the workload's block size (block-size sweep)")
    ap.add_argument("--dtype", choices=["", "bf16", "f32"], default="",
                    help="element type override for the mha/gqa/long workloads (f32 runs the "
                         "CUDA-core consumer)")
    ap.add_argument("--contiguous", action="store_true",
                    help="lay each sequence's blocks out consecutively (contiguous-cache control)")
    ap.add_argument("--step", choices=["separate", "fused"], default="fused",
                    help="run the step as one fused launch (paged_decode_step[_shared_prefix]) "
                         "or as copy_blocks + paged_kv_write + decode")
    ap.add_argument("--split", choices=["fixed", "balanced"], default="fixed",
                    help="decode work split (library default: fixed-length partitions)")
    ap.add_argument("--partition", type=int, default=0,
                    help="decode partition length in tokens (0 = library choice)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local_rank}"))
    try:
        if args.mode == "prefill":
            line = run_prefill(args, rank, world, local_rank)
        elif args.mode == "paging":
            line = run_paging(args, local_rank)
        else:
            line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
