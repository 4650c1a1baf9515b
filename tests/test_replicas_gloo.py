"""Multi-rank host logic of the benchmark on CPU with two gloo ranks: replicas draw
distinct requests, the step time is the maximum over ranks, and the whole-job rate
counts every rank's work over that time.  (The data path has no collective.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        import bench
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        out[rank] = (bench.max_over_ranks(ms), bench.rank_seed_base(rank))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] != res[1][1]


def test_whole_job_rate_and_identity_without_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    # 2 ranks x 5 units x 4 steps in 2000 ms
    assert bench.whole_job_rate(5.0, 2, 4, 2000.0) == pytest.approx(20.0)
