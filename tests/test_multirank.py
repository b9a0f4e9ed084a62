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


def test_reduce_max_without_process_group_is_identity():
    assert bench.reduce_max(3.5, "cpu") == 3.5
