"""The multi-GPU plan on CPU: world_size-2 gloo ranks, replicas by request,
timing reduced as the max over ranks (no data-path collective)."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [10.0, 25.0][rank]
        m = bench.reduce_max(ms, "cpu")
        plan = bench.replica_plan(rank, world, 1)
        out[rank] = (m, plan["first_request"], plan["seed"], plan["global_batch"])
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_and_max_timing():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == 25.0 and out[1][0] == 25.0          # both ranks see the slowest rank's time
    assert {out[0][1], out[1][1]} == {0, 1}                  # disjoint requests
    assert out[0][2] != out[1][2]                            # different seeds
    assert out[0][3] == out[1][3] == 2                       # weak scaling: global batch grows with N


def _timing_worker(rank, world, port, out):
    """bench.time_region as the bench runs it, on the host clock: both ranks report the slowest
    rank's timed region (barrier on both sides, max over ranks)."""
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        steps = []

        def body():
            for _ in range(3):
                time.sleep(0.02 * (rank + 1))       # rank 1's steps take twice as long
                steps.append(1)

        out[rank] = (bench.time_region(body, bench.HostClock(), "cpu"), len(steps))
    finally:
        dist.destroy_process_group()


def test_two_rank_timed_region_is_the_slowest_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_timing_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0][0] == out[1][0]                            # one number for the job
    assert out[0][0] >= 3 * 0.04 * 1e3 * 0.95                # at least rank 1's own time (ms)
    assert out[0][1] == out[1][1] == 3                       # every rank ran its steps


def test_reduce_max_without_process_group_is_identity():
    assert bench.reduce_max(3.5, "cpu") == 3.5
