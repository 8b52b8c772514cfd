"""GPU parity of the fp16 entry points (fa_fwd_f16, fa_bwd_f16) against the fp64
oracle, on inputs drawn as for the bf16 path and rounded to fp16.  The bounds
(TOL_F16) are tighter than the bf16 ones: fp16 keeps three more significand bits."""
import pytest
import torch

import exact_attention_107_b200 as fa
import oracle
import workloads
from parity import TOL, TOL_F16, check_fwd, check_grads, gpu_fwd_bwd, rel_fro

pytestmark = pytest.mark.gpu

SHAPES = [
    # B, H, N, D, causal
    (1, 2, 128, 64, False), (1, 2, 256, 128, True), (2, 3, 384, 64, True),
    (1, 1, 1, 64, False), (1, 2, 200, 64, True), (1, 2, 129, 128, True),
    (1, 1, 300, 128, False), (1, 4, 1024, 128, True), (1, 3, 1000, 64, False),
    (1, 2, 384, 96, True), (1, 2, 300, 32, False), (1, 2, 384, 256, True), (1, 1, 200, 256, False),
]


@pytest.mark.parametrize("causal", [False, True])
def test_fp16_forward_head_dim_256(causal):
    w, (q, k, v, do) = _inputs(1, 2, 640, 256, causal)
    O, lse = fa.attention_forward(q.cuda(), k.cuda(), v.cuda(), w.softmax_scale, causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, causal)
    check_fwd(O.cpu(), lse.cpu(), ref_O, ref_lse, tol=TOL_F16)


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _inputs(B, H, N, D, causal, dtype="fp16", seed=11, std=1.0):
    w = workloads.custom("fp16", B, H, N, D, causal, dtype=dtype, seed=seed, qkv_std=std)
    return w, workloads.make_inputs(w, with_grad_out=True)


@pytest.mark.parametrize("B,H,N,D,causal", SHAPES)
def test_fp16_fwd_bwd(B, H, N, D, causal):
    w, (q, k, v, do) = _inputs(B, H, N, D, causal)
    assert q.dtype == torch.float16
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, causal)
    assert got["O"].dtype == torch.float16 and got["dQ"].dtype == torch.float16
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"], (B, H, N, D, causal), tol=TOL_F16)
    check_grads(got, ref, (B, H, N, D, causal), tol=TOL_F16)


def test_fp16_gpt2_like_workload():
    """The shape of the GPT-2 causal workload (8 x 12 x 1024 x 64) in fp16."""
    base = workloads.WORKLOADS["c4_gpt2_causal"]
    w, (q, k, v, do) = _inputs(base.B, base.H, base.N, base.D, True, seed=base.seed, std=base.qkv_std)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, True)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, True)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"], tol=TOL_F16)
    check_grads(got, ref, tol=TOL_F16)


def test_fp16_large_logits():
    """Scores of large magnitude with a row max that keeps growing: the lazily
    rescaled probabilities (up to 2^8) and the gradients stay inside fp16's range."""
    B, H, N, D = 1, 2, 768, 128
    w, (q, k, v, do) = _inputs(B, H, N, D, True, seed=5)
    ramp = torch.linspace(0.2, 3.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.float16)
    q = (q.float() * 2.0).to(torch.float16)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, True)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, True)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"], tol=TOL_F16)
    check_grads(got, ref, tol=TOL_F16)


def test_fp16_more_accurate_than_bf16():
    """On inputs exactly representable in both types (bf16 values with small
    exponents are fp16 values too), the fp16 path's O error is well below the bf16
    path's: its P and O roundings are 8x finer."""
    B, H, N, D = 1, 4, 512, 64
    w, xs = _inputs(B, H, N, D, False, dtype="bf16", seed=3)
    # flush the few draws below fp16's normal range, where bf16 values need not be fp16 values
    q, k, v, do = (torch.where(t.abs() < 2.0 ** -14, torch.zeros_like(t), t) for t in xs)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, False)
    got_b = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, False)
    q16, k16, v16, do16 = (t.to(torch.float16) for t in (q, k, v, do))
    for a, b in ((q16, q), (k16, k), (v16, v), (do16, do)):
        assert torch.equal(a.to(torch.bfloat16), b)          # the same values in both types
    got_h = gpu_fwd_bwd(q16, k16, v16, do16, w.softmax_scale, False)
    eb, eh = rel_fro(got_b["O"], ref["O"]), rel_fro(got_h["O"], ref["O"])
    assert eh < eb / 3, (eh, eb)
    for n in ("dQ", "dK", "dV"):
        assert rel_fro(got_h[n], ref[n]) < rel_fro(got_b[n], ref[n]), n
    check_fwd(got_b["O"], got_b["lse"], ref["O"], ref["lse"], tol=TOL)


def test_fp16_binding_rejects_other_dtypes():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 128, device="cuda")
    with pytest.raises(TypeError):
        fa.fa_fwd_f16(q, q, q, q, lse, 0.125, False)
    with pytest.raises(TypeError):
        fa.fa_fwd(q.half(), q.half(), q.half(), q.half(), lse, 0.125, False)
