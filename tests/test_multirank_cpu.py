"""The multi-GPU host path of bench.py, exercised with two gloo ranks on the CPU:
each rank gets its own input shard (seed), the timed value is the maximum over
ranks, and the whole-job throughput counts every rank's work over that maximum.
No collective is on the attention data path (the (b, h) shards are independent)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.custom("mr", 1, 2, 64, 64, True, seed=bench.shard_seed(11, rank))
        q = workloads.make_inputs(w)[0]
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)       # rank 1 is the slow one
        out[rank] = (t, float(q.float().sum()), bench.whole_job_tflops(world, 1e12, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0                         # max over ranks
    assert res[0][1] != res[1][1]                                 # distinct shards
    assert res[0][2] == pytest.approx(world * 1e12 / 15e-3 / 1e12)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.shard_seed(5, 0) == 5 and bench.shard_seed(5, 3) == 3005
    assert bench.whole_job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
