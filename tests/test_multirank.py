"""The multi-rank bench path on CPU: two gloo ranks reduce their step times to
the slowest rank's, and the whole-job throughput counts every rank's work
(weak scaling: each rank runs the same workload as an independent replica)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(times[rank], dist, torch.device("cpu"))
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_time():
    world, times = 2, [3.25, 4.5]
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == max(times)


def test_whole_job_throughput_is_weak_scaling():
    assert bench.max_over_ranks(2.5, None, None) == 2.5
    one = bench.whole_job_throughput(1e12, 1, 10.0)
    assert one == pytest.approx(100.0)
    # two replicas, each as slow as one alone: twice the throughput
    assert bench.whole_job_throughput(1e12, 2, 10.0) == pytest.approx(2 * one)
