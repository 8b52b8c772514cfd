"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Small cases that span several tiles and ragged tails come
first; then the five workloads at full size (the long-context one on a seeded
sample of 64 query rows and 64 key rows per head)."""
import math

import pytest
import torch

import exact_attention_107_b200 as fa
import oracle
import workloads
from parity import TOL, check_fwd, check_grads, gpu_forward, gpu_fwd_bwd, max_abs, rel_fro

pytestmark = pytest.mark.gpu

SMALL = [
    # B, H, N, D, causal
    (1, 2, 128, 64, False), (1, 2, 128, 64, True),
    (1, 2, 256, 128, False), (1, 2, 256, 128, True),
    (2, 3, 384, 64, True), (1, 2, 640, 128, False),
    (1, 1, 1, 64, False), (1, 1, 1, 128, True),
    (1, 2, 200, 64, False), (1, 2, 200, 64, True),
    (1, 2, 129, 128, True), (1, 1, 300, 128, False), (2, 1, 77, 64, True),
    (1, 4, 1024, 128, True), (1, 3, 1000, 64, False),
]


def _small(B, H, N, D, causal, std=1.0, seed=11):
    w = workloads.custom("small", B, H, N, D, causal, seed=seed, qkv_std=std)
    return w, workloads.make_inputs(w, with_grad_out=True)


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


@pytest.mark.parametrize("B,H,N,D,causal", SMALL)
def test_forward_small(B, H, N, D, causal):
    w, (q, k, v, do) = _small(B, H, N, D, causal)
    O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, causal)
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, causal)
    check_fwd(O.cpu(), lse.cpu(), ref_O, ref_lse, (B, H, N, D, causal))


@pytest.mark.parametrize("B,H,N,D,causal", SMALL)
def test_backward_small(B, H, N, D, causal):
    w, (q, k, v, do) = _small(B, H, N, D, causal)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, causal)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"])
    check_grads(got, ref, (B, H, N, D, causal))


# Head dims 32 and 96 run the 64- and 128-column kernels on zero-filled columns.
ODD_D = [(1, 2, 256, 32, False), (1, 2, 200, 32, True), (2, 1, 640, 32, True),
         (1, 2, 256, 96, True), (2, 2, 333, 96, False), (1, 1, 1, 96, True)]


@pytest.mark.parametrize("B,H,N,D,causal", ODD_D)
def test_head_dims_32_and_96(B, H, N, D, causal):
    w, (q, k, v, do) = _small(B, H, N, D, causal)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, causal)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"], (B, H, N, D, causal))
    check_grads(got, ref, (B, H, N, D, causal))


# Head dim 256: forward only (its own kernel: one query tile per CTA, two score buffers).
D256 = [(1, 2, 256, 256, False), (1, 2, 384, 256, True), (2, 1, 200, 256, True), (1, 1, 1, 256, False),
        (1, 3, 1000, 256, False), (1, 2, 1024, 256, True)]


@pytest.mark.parametrize("B,H,N,D,causal", D256)
def test_forward_head_dim_256(B, H, N, D, causal):
    w, (q, k, v, do) = _small(B, H, N, D, causal)
    O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, causal)
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, causal)
    check_fwd(O.cpu(), lse.cpu(), ref_O, ref_lse, (B, H, N, D, causal))


@pytest.mark.parametrize("causal", [False, True])
def test_forward_head_dim_256_growing_max(causal):
    """The rescale of the 256-column accumulator, which waits for the previous P V product."""
    B, H, N, D = 1, 2, 1024, 256
    w, (q, k, v, do) = _small(B, H, N, D, causal, seed=5)
    ramp = torch.linspace(0.2, 3.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float() * 2.0).to(torch.bfloat16)
    O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, causal)
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, causal)
    check_fwd(O.cpu(), lse.cpu(), ref_O, ref_lse)


D256_BWD = [(1, 2, 256, 256, False), (1, 2, 384, 256, True), (2, 1, 200, 256, True), (1, 1, 1, 256, False),
            (1, 2, 1000, 256, False), (1, 2, 640, 256, True)]


@pytest.mark.parametrize("B,H,N,D,causal", D256_BWD)
def test_backward_head_dim_256(B, H, N, D, causal):
    """The two-CTA-per-tile backward (each CTA owns one half of D)."""
    w, (q, k, v, do) = _small(B, H, N, D, causal)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, causal)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"], (B, H, N, D, causal))
    check_grads(got, ref, (B, H, N, D, causal))


@pytest.mark.parametrize("D,causal", [(64, False), (128, True)])
def test_large_logits_and_growing_max(D, causal):
    """Scores of large magnitude whose row max keeps growing along the keys, so the
    online softmax must rescale its accumulator many times."""
    B, H, N = 1, 2, 768
    w, (q, k, v, do) = _small(B, H, N, D, causal, std=1.0, seed=5)
    ramp = torch.linspace(0.2, 3.0, N).view(1, 1, N, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    q = (q.float() * 2.0).to(torch.bfloat16)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, causal)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"])
    check_grads(got, ref)


def test_constant_scores_closed_form():
    """K = 0 gives O = mean of V (prefix mean when causal) and lse = ln(count)."""
    B, H, N, D = 1, 2, 384, 64
    w, (q, k, v, do) = _small(B, H, N, D, True)
    k = torch.zeros_like(k)
    O, lse, _ = gpu_forward(q, k, v, 0.125, True)
    counts = torch.arange(1, N + 1, dtype=torch.float64)
    mean = v.double().cumsum(dim=2) / counts.view(1, 1, N, 1)
    assert max_abs(O.cpu(), mean) < TOL["O_max"]
    assert max_abs(lse.cpu(), torch.log(counts).expand(B, H, N)) < TOL["lse_max"]


def test_autograd_wrapper():
    w, (q, k, v, do) = _small(1, 2, 256, 64, True)
    dev = torch.device("cuda")
    qd, kd, vd = (t.to(dev).requires_grad_(True) for t in (q, k, v))
    O = fa.flash_attention(qd, kd, vd, w.softmax_scale, True)
    O.backward(do.to(dev))
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, True)
    assert rel_fro(O.detach().cpu(), ref["O"]) <= TOL["O_fro"]
    check_grads({"dQ": qd.grad.cpu(), "dK": kd.grad.cpu(), "dV": vd.grad.cpu()}, ref)


def test_stage_entry_points_match_fa_bwd():
    """fa_bwd == fa_bwd_preprocess + fa_bwd_dkdv + fa_bwd_dq, bit for bit."""
    w, (q, k, v, do) = _small(2, 2, 300, 128, True)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    O, lse = fa.attention_forward(qd, kd, vd, w.softmax_scale, True)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, O, lse, dod, w.softmax_scale, True)
    B, H, N, D = q.shape
    ws = torch.full((fa.fa_bwd_workspace_size(B, H, N, D),), 0x5A, device=dev, dtype=torch.uint8)  # stale bytes
    fa.fa_bwd_preprocess(O, dod, lse, ws)
    dq2, dk2, dv2 = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    fa.fa_bwd_dkdv(qd, kd, vd, dod, ws, dk2, dv2, w.softmax_scale, True)
    fa.fa_bwd_dq(qd, kd, vd, dod, ws, dq2, w.softmax_scale, True)
    torch.cuda.synchronize()
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    nl, delta = (x.cpu() for x in fa.workspace_views(ws, B, H, N))
    ref_delta = oracle.attention_delta(O.cpu(), do)
    assert max_abs(delta[..., :N], ref_delta) < 1e-4
    assert torch.equal(delta[..., N:], torch.zeros_like(delta[..., N:]))
    assert max_abs(nl[..., :N], -lse.cpu().double() / math.log(2.0)) < 1e-5
    assert torch.isinf(nl[..., N:]).all() and (nl[..., N:] < 0).all()


def test_deterministic():
    w, (q, k, v, do) = _small(1, 4, 512, 64, False)
    a = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, False)
    b = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, False)
    for n in a:
        assert torch.equal(a[n], b[n]), n


# ----------------------------------------------------------------------------- the five workloads
def test_c1_fp32_forward():
    w = workloads.WORKLOADS["c1_fp32_fwd"]
    q, k, v, _ = workloads.make_inputs(w)
    O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, w.causal)
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, w.causal)
    assert rel_fro(O.cpu(), ref_O) <= TOL["f32_fro"]
    assert ((lse.cpu().double() - ref_lse).abs() / ref_lse.abs().clamp_min(1.0)).max() <= TOL["f32_lse"]


def test_fp32_path_small_shapes():
    for (B, H, N, D, causal) in [(1, 1, 1, 32, False), (2, 2, 100, 128, True), (1, 3, 333, 64, True)]:
        w = workloads.custom("f32", B, H, N, D, causal, dtype="fp32", seed=3)
        q, k, v, _ = workloads.make_inputs(w, with_grad_out=False)
        O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, causal)
        ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, causal)
        assert rel_fro(O.cpu(), ref_O) <= TOL["f32_fro"], (B, H, N, D, causal)
        assert max_abs(lse.cpu(), ref_lse) <= TOL["f32_lse"] * max(1.0, ref_lse.abs().max().item())


def test_c2_forward():
    w = workloads.WORKLOADS["c2_bf16_fwd"]
    q, k, v, _ = workloads.make_inputs(w)
    O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, w.causal)
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, w.causal)
    check_fwd(O.cpu(), lse.cpu(), ref_O, ref_lse, w.name)


@pytest.mark.parametrize("name", ["c3_bf16_fwdbwd", "c4_gpt2_causal"])
def test_fwd_bwd_workload(name):
    w = workloads.WORKLOADS[name]
    q, k, v, do = workloads.make_inputs(w)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, w.causal)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, w.causal)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"], name)
    check_grads(got, ref, name)


def test_c5_long_context_sampled():
    w = workloads.WORKLOADS["c5_long_causal"]
    q, k, v, do = workloads.make_inputs(w)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, w.causal)
    BH = w.B * w.H
    qrows = {bh: workloads.sample_rows(w, bh) for bh in range(BH)}
    krows = {bh: workloads.sample_rows(w, bh, seed_base=3000) for bh in range(BH)}
    ref = oracle.attention_sampled_rows(q, k, v, do, w.softmax_scale, True, qrows, krows, chunk=1024)
    cat = {n: [] for n in ("O", "lse", "dQ", "dK", "dV", "rO", "rlse", "rdQ", "rdK", "rdV")}
    for bh in range(BH):
        b, h = divmod(bh, w.H)
        r, c = qrows[bh], krows[bh]
        for n, rows in (("O", r), ("dQ", r), ("dK", c), ("dV", c)):
            cat[n].append(got[n][b, h, rows])
            cat["r" + n].append(ref[bh][n])
        cat["lse"].append(got["lse"][b, h, r])
        cat["rlse"].append(ref[bh]["lse"])
    j = {n: torch.cat(v) for n, v in cat.items()}
    check_fwd(j["O"], j["lse"], j["rO"], j["rlse"], "c5 sampled")
    check_grads({"dQ": j["dQ"], "dK": j["dK"], "dV": j["dV"]}, {"dQ": j["rdQ"], "dK": j["rdK"], "dV": j["rdV"]},
                "c5 sampled")
    # properties over every row: finite, lse bounded by max score + ln(count)
    assert torch.isfinite(got["O"].float()).all() and torch.isfinite(got["dK"].float()).all()
    assert torch.isfinite(got["dQ"].float()).all() and torch.isfinite(got["dV"].float()).all()


def test_device_status_clean():
    assert fa.fa_device_status(reset=False) == 0
