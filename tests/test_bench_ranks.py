"""The multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

bench.py --gpus N runs one replica per rank with no collective in the data path; the only
exchange is the max over ranks of the measured times, and rank 0 alone prints.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench
import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.5])
        w = bench.rank_workload(wl.LLAMA2_7B_MHA_32K, rank)
        out[rank] = (got, w.seed, bench.prints_line(rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_seeds():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:   # no fork of this (threaded) process
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        got, seed, prints = res[rank]
        assert got == [2.0, 10.0, 3.5]           # the slowest rank sets every time
        assert prints == (rank == 0)
    assert res[0][1] != res[1][1]                # each replica draws its own batch
    assert res[0][1] == wl.LLAMA2_7B_MHA_32K.seed


def test_single_process_max_is_identity():
    assert bench.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
