"""The N>1 path of bench.py on CPU: two gloo ranks, each with its own replica workload.

The decode shards by sequences with no exchange step, so multi-GPU runs are replicas:
every rank builds its own seeded pool (a different seed offset per rank) and times its own
steps; the only collective is the max of the device-timed step time, and the whole-job
throughput is (ranks x bytes per rank) / that max."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from paged_kv_cache_344_b200 import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workloads.make("gqa16", scale_down=32)
        t = workloads.host_tensors(wl, seed_offset=rank)
        local_ms = 10.0 + 5.0 * rank  # stand-in for a device-timed value
        m = bench.max_over_ranks(local_ms, world, "cpu")
        out[rank] = (m, float(t["q"].astype(np.float64).sum()), int(wl.num_blocks))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 15.0          # both ranks agree on the slowest rank
    assert out[0][1] != out[1][1]                  # replicas: different seeded data
    assert out[0][2] == out[1][2]                  # same workload shape on every rank
    # whole-job value: all ranks' bytes over the slowest rank's time
    assert bench.whole_job_gbs(10**9, 10, 2, 15.0) == pytest.approx(2 * 10**10 / 0.015 / 1e9)


def test_single_rank_needs_no_collective():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
