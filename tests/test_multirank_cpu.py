"""The bench's multi-rank host logic on two CPU ranks (gloo).

Decode shards by sequence: every rank owns its own batch, runs the same step
with no data-path collective, and the reported figure is all ranks' queries
over the slowest rank's time. These tests run that logic -- the per-rank
workload, the MAX reduction of the timings and the whole-job rate -- on two
gloo ranks over 127.0.0.1, with no GPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from compressed_sparse_kv_02_b200 import synth
        cfg = bench.rank_config(synth.CONFIGS["pro"], rank)
        # a rank-dependent step time: rank 1 is the slow one
        ms = 0.25 + 0.1 * rank
        ms_max = bench.max_over_ranks(ms, torch.device("cpu"), world)
        rate = bench.whole_job_rate(cfg.batch, world, ms_max)
        q.put((rank, cfg.seed, cfg.batch, ms_max, rate))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_queries():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    (r0, seed0, b0, ms0, rate0), (r1, seed1, b1, ms1, rate1) = got
    assert (r0, r1) == (0, 1)
    assert seed0 != seed1 and b0 == b1  # own sequences, same shapes
    assert ms0 == pytest.approx(0.35) and ms1 == pytest.approx(0.35)  # both see the slowest rank
    assert rate0 == pytest.approx(b0 * 2 / 0.35e-3) and rate1 == rate0


def _worker_fail(rank, world, port, q):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    try:
        import bench
        if rank == 1:
            q.put((rank, "left"))
            return  # leaves between steps: never joins the reduction
        try:
            bench.max_over_ranks(0.25, torch.device("cpu"), world)
            q.put((rank, "no error"))
        except Exception:  # the short process-group timeout ends the collective with an error
            q.put((rank, "error"))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_a_rank_that_leaves_ends_the_others_reduction_with_an_error():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_fail, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    got = dict(q.get(timeout=10) for _ in range(world))
    assert got[1] == "left"
    assert got[0] == "error"
