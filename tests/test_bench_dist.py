"""Multi-rank plumbing of bench.py on CPU: two gloo ranks.

Each rank of a multi-GPU run processes its own batch of independent sequences
(no collective on the data path); the only cross-rank steps are the barriers
around the timed region and the max / sum reductions of the timings.  These
tests run those steps with world size 2 over gloo on 127.0.0.1.
"""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        bench.barrier(world)
        # per-rank timings differ; the job takes as long as the slowest rank
        t = 1.0 + rank
        mx = bench.max_over_ranks(t, world, dev)
        sm = bench.sum_over_ranks(t, world, dev)
        val = bench.weak_scaling_throughput(8, 10, world, mx)
        bench.barrier(world)
        out[rank] = (mx, sm, val)
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert len(out) == world
    for r in range(world):
        mx, sm, val = out[r]
        assert mx == 2.0           # max of 1.0 and 2.0 on every rank
        assert sm == 3.0
        assert val == pytest.approx(8 * 10 * 2 / 2.0)


def _ref_rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    # the oracle arm: ranks other than 0 exit at once, without a device
    if rank != 0:
        out[rank] = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "3", "--warmup", "3"])
    else:
        out[rank] = 0


def test_reference_arm_other_ranks_exit():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_ref_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert out[1] == 0


def test_weak_scaling_single_rank_identity():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.sum_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_throughput(8, 100, 1, 0.5) == pytest.approx(1600.0)
