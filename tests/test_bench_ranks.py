"""Multi-rank host logic of bench.py with two gloo ranks on CPU: the timed
region's max over ranks and the whole-job aggregate."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t = bench.max_over_ranks(1.5 + rank, world)  # rank 1 is the slowest
        out[rank] = t
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1] == 2.5


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_aggregate_counts_every_replica():
    step = 2.0 * 4096 * 7168 * 16384
    one = bench.aggregate_tflops(step, 1, 0.4)
    assert abs(one - step / 0.4e-3 / 1e12) < 1e-9
    assert abs(bench.aggregate_tflops(step, 4, 0.4) - 4 * one) < 1e-9
