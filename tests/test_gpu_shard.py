"""(b, h) sharding with the real kernels on one GPU: a call split into slices (here all on
cuda:0, one after another) gives the unsharded call's results: O, lse, dK, dV bit for bit
(the same kernels on the same rows), dQ up to the order of its fp32 additions."""
import pytest
import torch

import exact_attention_107_b200 as fa
import workloads
from parity import rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


@pytest.mark.parametrize("shape", [(2, 3, 300, 128, True), (1, 5, 256, 64, False)])
def test_device_split_matches_the_whole_call(shape):
    B, H, N, D, causal = shape
    w = workloads.custom("shard", B, H, N, D, causal, seed=91)
    q, k, v, do = (t.cuda() for t in workloads.make_inputs(w, with_grad_out=True))
    o, lse = fa.attention_forward(q, k, v, w.softmax_scale, causal)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, w.softmax_scale, causal)
    res = fa.sharded_attention_devices(q, k, v, do, w.softmax_scale, causal, devices=["cuda:0"] * 3)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    for name, ref in (("o", o), ("lse", lse), ("dk", dk), ("dv", dv)):
        assert torch.equal(res[name], ref), name
    assert rel_fro(res["dq"].cpu(), dq.cpu()) <= 1e-4


def test_single_rank_sharded_attention_is_the_whole_call():
    w = workloads.custom("shard1", 1, 2, 200, 64, True, seed=92)
    q, k, v, _ = (t.cuda() if t is not None else None for t in workloads.make_inputs(w, with_grad_out=False))
    o, lse = fa.attention_forward(q, k, v, w.softmax_scale, True)
    res = fa.sharded_attention(q, k, v, None, w.softmax_scale, True, rank=0, world=1)
    torch.cuda.synchronize()
    assert torch.equal(res["o"], o) and torch.equal(res["lse"], lse)
