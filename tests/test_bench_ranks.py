"""The replica timing of `bench.py --gpus N` on CPU: two ranks on the gloo
backend, each with its own time, agree on the slowest one (the path has no
exchange step, so this reduction is the only collective of a multi-GPU run)."""

import os
import socket

import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        out[rank] = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
    finally:
        tdist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_max_over_ranks_without_a_process_group():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
