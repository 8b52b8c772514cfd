"""HostStepPipeline: steps streamed from pinned host memory give, step by step, the
results of the device-resident entry points on the same inputs (same kernels, so the
results are bitwise equal, except dQ, whose fp32 additions run in a run-dependent
order), and the first step matches the fp64 oracle."""
import pytest
import torch

import exact_attention_107_b200 as fa
import oracle
import workloads
from parity import check_fwd, check_grads, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_pipelined_steps_match_direct_calls(dtype):
    B, H, N, D, causal = 1, 2, 640, 128, True
    steps = [workloads.make_inputs(workloads.custom("pipe", B, H, N, D, causal, dtype=dtype, seed=40 + i),
                                   with_grad_out=True) for i in range(4)]
    scale = D ** -0.5
    pipe = fa.HostStepPipeline(B, H, N, D, dtype=steps[0][0].dtype)
    outs = [pipe.host_outputs() for _ in steps]
    for (q, k, v, do), out in zip(steps, outs):
        h2d, d2h = pipe.submit(*(t.pin_memory() for t in (q, k, v, do)), out, scale, causal)
        assert h2d == 4 * q.numel() * q.element_size()
        assert d2h == 4 * q.numel() * q.element_size() + B * H * N * 4
    pipe.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    for (q, k, v, do), out in zip(steps, outs):
        qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
        o, lse = fa.attention_forward(qd, kd, vd, scale, causal)
        dq, dk, dv = fa.attention_backward(qd, kd, vd, o, lse, dod, scale, causal)
        torch.cuda.synchronize()
        for name, ref in (("o", o), ("lse", lse), ("dk", dk), ("dv", dv)):
            assert torch.equal(out[name], ref.cpu()), name
        assert rel_fro(out["dq"], dq.cpu()) <= 1e-4
    q, k, v, do = steps[0]
    ref = oracle.attention_backward(q, k, v, do, scale, causal)
    got = {"O": outs[0]["o"], "lse": outs[0]["lse"], "dQ": outs[0]["dq"], "dK": outs[0]["dk"], "dV": outs[0]["dv"]}
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"])
    check_grads(got, ref)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_single_step_from_host_matches_direct_calls(dtype):
    B, H, N, D, causal = 1, 2, 384, 64, False
    q, k, v, do = workloads.make_inputs(workloads.custom("host", B, H, N, D, causal, dtype=dtype, seed=7),
                                        with_grad_out=True)
    scale = D ** -0.5
    out, h2d, d2h = fa.attention_fwd_bwd_from_host(*(t.pin_memory() for t in (q, k, v, do)), scale, causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    assert out["o"].dtype == q.dtype and h2d == 4 * q.numel() * q.element_size()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.attention_forward(qd, kd, vd, scale, causal)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, o, lse, dod, scale, causal)
    torch.cuda.synchronize()
    for name, ref in (("o", o), ("lse", lse), ("dk", dk), ("dv", dv)):
        assert torch.equal(out[name], ref.cpu()), name
    assert rel_fro(out["dq"], dq.cpu()) <= 1e-4


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_forward_only_pipeline(dtype):
    """Forward-only steps (bf16 tensor-core path, fp32 FFMA path) from pinned host memory."""
    B, H, N, D, causal = 1, 2, 256, 64, False
    steps = [workloads.make_inputs(workloads.custom("pipe_fwd", B, H, N, D, causal, dtype=dtype, seed=60 + i),
                                   with_grad_out=False) for i in range(3)]
    scale = D ** -0.5
    pipe = fa.HostStepPipeline(B, H, N, D, dtype=steps[0][0].dtype, backward=False)
    outs = [pipe.host_outputs() for _ in steps]
    assert set(outs[0]) == {"o", "lse"}
    for (q, k, v, _), out in zip(steps, outs):
        h2d, d2h = pipe.submit(*(t.pin_memory() for t in (q, k, v)), None, out, scale, causal)
        assert h2d == 3 * q.numel() * q.element_size()
        assert d2h == q.numel() * q.element_size() + B * H * N * 4
    pipe.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    for (q, k, v, _), out in zip(steps, outs):
        o, lse = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), scale, causal)
        torch.cuda.synchronize()
        assert torch.equal(out["o"], o.cpu()) and torch.equal(out["lse"], lse.cpu())
