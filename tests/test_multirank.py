"""The replica path on CPU: two gloo ranks take the maximum of their times and
report whole-job throughput over both, with no data-path collective."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from parameterized_local_linear_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank timed its own replica: rank r took 1 + r seconds
        t = replicas.max_over_ranks(1.0 + rank)
        rate = replicas.whole_job_rate(units_per_rank=100.0, seconds_max=t)
        replicas.barrier()
        # replicas are independent: a rank's result depends only on its inputs
        x = torch.arange(4, dtype=torch.float64) * (rank + 1)
        out[rank] = (t, rate, float(x.sum()), replicas.world_size())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.0          # max over ranks
    assert res[0][1] == res[1][1] == 2 * 100.0 / 2.0  # units of both ranks / slowest time
    assert res[0][2] == 6.0 and res[1][2] == 12.0  # no exchange of data
    assert res[0][3] == res[1][3] == 2


def test_single_process_defaults():
    assert replicas.world_size() == 1
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.whole_job_rate(10.0, 2.0) == 5.0
