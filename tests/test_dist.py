"""Data-parallel host logic of bench.py on CPU ranks (gloo, world size 2):
the job's time is the slowest rank's, its work the sum of every rank's, and
each rank draws its own synthetic sample."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        el, fl = bench.reduce_over_ranks(10.0 + 5.0 * rank, 100.0 * (rank + 1), "cpu")
        out[rank] = (el, fl)
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    for rank in range(world):
        el, fl = res[rank]
        assert el == 15.0          # max over ranks
        assert fl == 300.0         # sum over ranks


def test_single_process_is_identity():
    assert bench.reduce_over_ranks(3.5, 7.0, "cpu") == (3.5, 7.0)


def test_ranks_draw_distinct_samples():
    w = synth.WORKLOADS[2]
    a = synth.make_qkv(w.wid, bench.rank_sample(0), 2, 4, 4, 1, 64)[0]
    b = synth.make_qkv(w.wid, bench.rank_sample(1), 2, 4, 4, 1, 64)[0]
    assert not (a == b).all()
