"""Multi-rank logic of bench.py on CPU (gloo, world size 2): the timer is
the max over ranks and the whole-job rate counts every rank's units."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.sync_all(True, device="cpu")
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, True, device="cpu")   # rank 1 is slower
        out[rank] = (ms, bench.whole_job_rate(131072, world, ms))
        bench.sync_all(True, device="cpu")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_rate():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == pytest.approx(2 * 131072 / 0.015)
