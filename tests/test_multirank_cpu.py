"""The multi-GPU path of bench.py, exercised on the CPU with two gloo ranks:
each rank gets its own seeded copy of the serving workload (requests are
independent, so no data crosses ranks), the step time is the max over ranks,
and the reported value counts every rank's rows."""
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
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        wl = bench.rank_workload(rank, requests=4, spare_slots=32)
        ms = 10.0 + 5.0 * rank                        # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world)
        value = bench.job_rows_per_s(wl.requests * 20, world, slowest)
        out[rank] = (wl.seed, wl.requests, wl.ctx0[0], slowest, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_requests_and_take_max_time():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert set(res) == {0, 1}
    seeds = {res[r][0] for r in res}
    assert len(seeds) == 2                              # each rank its own data
    assert all(res[r][1] == 4 and res[r][2] == 512 * 1024 for r in res)
    assert all(res[r][3] == 15.0 for r in res)          # the slowest rank's time on every rank
    assert all(abs(res[r][4] - 2 * 4 * 20 / 0.015) < 1e-6 for r in res)
