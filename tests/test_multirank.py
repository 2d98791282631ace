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


# ---------------------------------------------------------------- head-sharded split


def test_shard_ranges_cover_every_slice_exactly_once():
    for n in range(1, 60):
        for world in range(1, min(n, 9) + 1):
            ranges = [bench.shard_range(n, world, r) for r in range(world)]
            covered = [i for lo, hi in ranges for i in range(lo, hi)]
            assert covered == list(range(n)), (n, world)
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        bench.shard_range(3, 4, 0)


def _shard_rank(rank, world, port, out):
    import numpy as np

    import oracle
    from workloads import generate, small_config
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = small_config("shard", dtype="fp32", batch=1, heads=5, L=320, d=32, block=64, keep_ratio=0.4, seed=7)
        kk = oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
        lo, hi = bench.shard_range(cfg.batch * cfg.heads, world, rank)
        q, k, v = generate(cfg, heads=range(lo, hi), redraws={})
        mine = [oracle.pisa_head(q[0, n], k[0, n], v[0, n], cfg.block, kk) for n in range(hi - lo)]
        outs = np.stack([r["out"] for r in mine])
        sels = np.stack([r["sel"] for r in mine])
        import dataclasses
        part = dataclasses.replace(cfg, heads=hi - lo)
        flops = sum(bench.effective_flops(part, sels))
        job_flops = bench.sum_over_ranks(flops, dist, torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, (lo, hi, outs))
        if rank == 0:
            out[0] = (gathered, job_flops)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_the_heads_and_reassemble_the_single_rank_result():
    """Each rank computes its shard of the batch x heads slices (the oracle
    on a tiny fp32 case stands in for the GPU path); the shards put back in
    order equal the one-process result, and the job's FLOPs are the sum of
    the shards'."""
    import numpy as np

    import oracle
    from workloads import generate, small_config
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    gathered, job_flops = out[0]
    cfg = small_config("shard", dtype="fp32", batch=1, heads=5, L=320, d=32, block=64, keep_ratio=0.4, seed=7)
    kk = oracle.keep_count(cfg.L, cfg.block, cfg.keep_ratio)
    q, k, v = generate(cfg, redraws={})
    whole = [oracle.pisa_head(q[0, h], k[0, h], v[0, h], cfg.block, kk) for h in range(cfg.heads)]
    parts = sorted(gathered, key=lambda g: g[0])
    assert [(lo, hi) for lo, hi, _ in parts] == [bench.shard_range(cfg.heads, world, r) for r in range(world)]
    joined = np.concatenate([o for _, _, o in parts])
    np.testing.assert_array_equal(joined, np.stack([r["out"] for r in whole]))
    sel = np.stack([r["sel"] for r in whole])[None]
    assert job_flops == pytest.approx(sum(bench.effective_flops(cfg, sel)), rel=1e-12)
