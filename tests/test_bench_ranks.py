"""The replicated multi-GPU path of bench.py (one process per GPU, no data
exchange): its whole-job figures are the slowest rank's time and the sum of
all ranks' bytes. Checked with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [2.5, 4.0][rank]
        nbytes = [1.0e9, 3.0e9][rank]
        out[rank] = bench.combine_ranks(ms, nbytes, world, torch.device("cpu"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_max_time_and_total_bytes():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        assert res[r] == (4.0, 4.0e9)


def test_one_rank_is_unchanged():
    assert bench.combine_ranks(1.5, 7.0, 1, torch.device("cpu")) == (1.5, 7.0)
