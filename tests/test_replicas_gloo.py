"""Host logic of the multi-GPU replica run, exercised as world_size-2 gloo
ranks on the CPU: the slowest rank's timing becomes the job's, and replica
ranks draw distinct layer instances."""
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 0 is slower in the timed region, rank 1 in the end-to-end run
        mine = [10.0 + 5.0 * (rank == 0), 20.0 + 7.0 * (rank == 1)]
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == [15.0, 27.0]
    assert out[1] == [15.0, 27.0]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_replica_instances_distinct():
    seen = {bench.replica_instance_seed(r, i) for r in range(8) for i in range(256)}
    assert len(seen) == 8 * 256
    from bit_w4a4_quantised_b200 import workloads
    a = workloads.c2_action_attn(seed=0, layer=bench.replica_instance_seed(0, 1))
    b = workloads.c2_action_attn(seed=0, layer=bench.replica_instance_seed(1, 1))
    assert not (a.x == b.x).all()
