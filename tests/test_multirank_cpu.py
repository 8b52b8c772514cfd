"""The multi-GPU host paths, exercised with gloo ranks on the CPU.

* bench.py: each rank gets its own input shard (seed), the timed value is the
  maximum over ranks, and the whole-job throughput counts every rank's work over
  that maximum.
* exact_attention_107_b200.shard: one call's (b, h) pairs are split into
  contiguous balanced ranges, each rank computes its range (here with a CPU
  stand-in for the per-slice kernels, which needs no GPU), and the all-gather
  reassembles full tensors in which every (b, h) was computed exactly once, by the
  rank that owns it.
No collective is on the attention data path (the (b, h) shards are independent)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads
from exact_attention_107_b200 import shard


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


# ----------------------------------------------------------------------------- (b, h) sharding
def _stub_compute(q, k, v, do, scale, causal):
    """CPU stand-in for one slice's kernels: values that identify the slice's pairs, its
    rank and its inputs (o = the q slice plus the rank marker, lse = the pair's global
    index as seen through q's first element, gradients from k, v, dO)."""
    rank = dist.get_rank()
    o = q.float() + 1000.0 * (rank + 1)
    lse = q[..., 0].float().clone()
    out = {"o": o, "lse": lse}
    if do is not None:
        out.update(dq=do.float() * 2, dk=k.float() * 3, dv=v.float() * 4)
    return out


def _shard_worker(rank, world, port, shape, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, D = shape
        g = torch.Generator().manual_seed(5)
        q, k, v, do = (torch.randn(B, H, N, D, generator=g) for _ in range(4))
        # mark every (b, h) pair: q[b, h, 0, 0] = its flat index
        q[:, :, 0, 0] = torch.arange(B * H, dtype=torch.float32).view(B, H)
        res = shard.sharded_attention(q, k, v, do, 0.125, True, rank=rank, world=world, compute=_stub_compute)
        part = shard.sharded_attention(q, k, v, do, 0.125, True, rank=rank, world=world, gather=False,
                                       compute=_stub_compute)
        out[rank] = {n: t.numpy() for n, t in res.items()} | {"range": part["range"]}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, (2, 3, 8, 4)), (3, (1, 2, 4, 4))])
def test_bh_sharding_covers_every_pair_once(world, shape):
    """world 2 over B*H = 6 pairs (3 + 3) and world 3 over 2 pairs (1 + 1 + an empty range)."""
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, _free_port(), shape, out), nprocs=world, join=True)
        res = dict(out)
    B, H, N, D = shape
    ranges = shard.head_ranges(B * H, world)
    assert [tuple(res[r]["range"]) for r in range(world)] == ranges
    g = torch.Generator().manual_seed(5)
    q, k, v, do = (torch.randn(B, H, N, D, generator=g) for _ in range(4))
    q[:, :, 0, 0] = torch.arange(B * H, dtype=torch.float32).view(B, H)
    owner = torch.empty(B * H, dtype=torch.long)
    for r, (s0, e0) in enumerate(ranges):
        owner[s0:e0] = r
    for r in range(world):                                    # every rank holds the same full result
        o = torch.from_numpy(res[r]["o"]).view(B * H, N, D)
        lse = torch.from_numpy(res[r]["lse"]).view(B * H, N)
        assert torch.equal(lse[:, 0], torch.arange(B * H, dtype=torch.float32))   # each pair exactly where it belongs
        marker = (o - q.view(B * H, N, D)).mean(dim=(1, 2))
        assert torch.allclose(marker, 1000.0 * (owner + 1).float())              # computed by its owner
        assert torch.equal(torch.from_numpy(res[r]["dq"]), do * 2)
        assert torch.equal(torch.from_numpy(res[r]["dk"]), k * 3)
        assert torch.equal(torch.from_numpy(res[r]["dv"]), v * 4)


def test_head_ranges_partition():
    for bh in (0, 1, 5, 8, 96, 1000):
        for world in (1, 2, 3, 8):
            rs = shard.head_ranges(bh, world)
            assert len(rs) == world and rs[0][0] == 0 and rs[-1][1] == bh
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))                # contiguous, no overlap
            sizes = [e - s for s, e in rs]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.head_ranges(4, 0)


def test_shard_view_is_a_view_of_the_pairs():
    t = torch.arange(2 * 3 * 4 * 2, dtype=torch.float32).view(2, 3, 4, 2)
    v = shard.shard_view(t, (2, 5))
    assert v.shape == (1, 3, 4, 2) and v.data_ptr() == t[0, 2].data_ptr()
    assert torch.equal(v[0, 1], t[1, 0])                       # bh = 3 is (b=1, h=0)
    assert shard.shard_view(torch.zeros(2, 3, 4), (1, 2)).shape == (1, 1, 4)


def test_devices_split_with_a_stub_on_cpu():
    """The one-process, several-devices path with CPU 'devices' and a stand-in compute."""
    B, H, N, D = 2, 3, 4, 2
    q, k, v = (torch.randn(B, H, N, D) for _ in range(3))

    def stub(q, k, v, do, scale, causal):
        return {"o": q * 2, "lse": q[..., 0] * 0 + q.shape[1]}

    res = shard.sharded_attention_devices(q, k, v, None, 0.5, False, devices=["cpu", "cpu", "cpu", "cpu"],
                                          compute=stub)
    assert torch.equal(res["o"], q * 2)
    # ranges of 6 pairs over 4 devices: sizes 2, 2, 1, 1
    assert res["lse"][..., 0].flatten().tolist() == [2, 2, 2, 2, 1, 1]
