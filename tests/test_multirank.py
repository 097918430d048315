"""Host logic of the multi-GPU bench on CPU: two gloo ranks, no GPU.

The path shards by sequence with no data exchange; the only collectives are timing
plumbing (a barrier and the max over ranks of the timed duration).  These tests run that
plumbing with world_size 2 on the CPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        w, r, l = bench.dist_env()
        bench.barrier(cpu)
        mx = bench.reduce_max(10.0 + 5 * rank, cpu)
        wl = bench.workload("mid_prefill")
        seed = bench.rank_seed(wl, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        world_seen = bench.dist_world()
        q.put((rank, (w, r, l), mx, seeds, world_seen))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(2))
    for rank, env, mx, seeds, world_seen in res:
        assert env == (2, rank, rank)
        assert mx == 15.0  # max over ranks of 10 and 15
        assert len(set(seeds)) == 2  # independent batches per rank
        assert world_seen == 2


def _ref_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import argparse

    import bench
    args = argparse.Namespace(steps=1, warmup=0, cpu_seconds=0.5)
    wl = bench.workload("tiny")
    line = bench.run_reference(args, wl, world, rank)
    q.put((rank, line))


def test_reference_arm_runs_on_rank0_only():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_ref_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = dict(q.get() for _ in range(2))
    assert res[1] is None
    line = res[0]
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_units_and_bytes():
    import bench
    wl = bench.workload("mid_prefill")
    assert bench.units_per_step(wl) == 2 * 4 * 4096
    b = bench.bytes_per_token_head(wl)
    assert b["rows"] == (2 * 32 + 32) * 128 * 4
    assert b["step"] == 51464  # rows + scoring I/O + recurrence I/O
    assert bench.scoring_flops_per_token_head(wl) == 4 * 256 * 128
