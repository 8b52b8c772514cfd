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


@pytest.mark.parametrize("deterministic", [False, True])
def test_nan_in_q_propagates(deterministic):
    """One NaN in query row i (causal).  Every score of row i is NaN, so O_i, lse_i and dQ_i
    are NaN in every column, and so are dV_j and dK_j for every allowed key j <= i (each
    sums a product with P_ij or dS_ij); rows of O, dQ and dV other than those stay finite
    (masked P_ij of keys j > i are exactly 0).  Row 205 is a query column whose P^T
    entries the backward computes on the FMA-pipe exponential (205 mod 32 = 13), which
    must pass a NaN on the way the MUFU ex2 does."""
    B, H, N, D, i = 1, 1, 384, 64, 205
    w, (q, k, v, do) = _small(B, H, N, D, True)
    q = q.clone()
    q[0, 0, i, 5] = float("nan")
    dev = torch.device("cuda")
    O, lse, (qd, kd, vd) = gpu_forward(q, k, v, w.softmax_scale, True)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, O, lse, do.to(dev), w.softmax_scale, True,
                                       deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    O, lse, dq, dk, dv = (t[0, 0].float().cpu() for t in (O, lse, dq, dk, dv))
    other = torch.arange(N) != i
    assert torch.isnan(O[i]).all() and torch.isnan(lse[i]) and torch.isnan(dq[i]).all()
    assert torch.isfinite(O[other]).all() and torch.isfinite(lse[other]).all() and torch.isfinite(dq[other]).all()
    assert torch.isnan(dv[: i + 1]).all() and torch.isnan(dk[: i + 1]).all()
    assert torch.isfinite(dv[i + 1:]).all()


def _stale_workspace(nbytes, dev):
    return torch.full((nbytes,), 0x5A, device=dev, dtype=torch.uint8)    # stale bytes: nothing may read them


def test_fused_stage_entry_points_match_fa_bwd():
    """fa_bwd == fa_bwd_preprocess + fa_bwd_dkdvdq + fa_bwd_dq_finish on a workspace full of
    stale bytes (the preprocess must zero the dQ accumulator): dK and dV bit for bit, dQ up to
    the order of its fp32 additions."""
    w, (q, k, v, do) = _small(2, 2, 300, 128, True)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    O, lse = fa.attention_forward(qd, kd, vd, w.softmax_scale, True)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, O, lse, dod, w.softmax_scale, True)
    B, H, N, D = q.shape
    ws = _stale_workspace(fa.fa_bwd_workspace_size(B, H, N, D), dev)
    fa.fa_bwd_preprocess(O, dod, lse, ws)
    dq2, dk2, dv2 = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    fa.fa_bwd_dkdvdq(qd, kd, vd, dod, ws, dk2, dv2, w.softmax_scale, True)
    fa.fa_bwd_dq_finish(ws, dq2, w.softmax_scale)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    assert rel_fro(dq2.cpu(), dq.cpu()) <= 1e-4
    # the accumulator holds dQ / scale in the tile layout [D/4][128 rows][4] per 128-row query tile
    npad = (N + 127) // 128 * 128
    acc = ws.view(torch.float32)[2 * B * H * npad:].view(B, H, npad // 128, D // 4, 128, 4)
    acc = acc.permute(0, 1, 2, 4, 3, 5).reshape(B, H, npad, D)
    assert torch.equal(acc[:, :, N:], torch.zeros_like(acc[:, :, N:]))      # padded rows: only zeros added
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, True)
    assert rel_fro(acc[:, :, :N].cpu() * w.softmax_scale, ref["dQ"]) <= TOL["grad_fro"]


def test_deterministic_stage_entry_points_match():
    """fa_bwd_deterministic == fa_bwd_preprocess + fa_bwd_dkdv + fa_bwd_dq, bit for bit."""
    w, (q, k, v, do) = _small(2, 2, 300, 128, True)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    O, lse = fa.attention_forward(qd, kd, vd, w.softmax_scale, True)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, O, lse, dod, w.softmax_scale, True, deterministic=True)
    B, H, N, D = q.shape
    ws = _stale_workspace(fa.fa_bwd_deterministic_workspace_size(B, H, N, D), dev)
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


DET = [(1, 2, 128, 64, True), (1, 2, 640, 128, False), (2, 3, 384, 64, True), (1, 2, 129, 128, True),
       (1, 1, 1, 64, False), (1, 2, 200, 32, True), (2, 2, 333, 96, False)]


@pytest.mark.parametrize("B,H,N,D,causal", DET)
def test_backward_deterministic_small(B, H, N, D, causal):
    """The three-stage backward (fa_bwd_deterministic) against the oracle."""
    w, (q, k, v, do) = _small(B, H, N, D, causal)
    dev = torch.device("cuda")
    O, lse, (qd, kd, vd) = gpu_forward(q, k, v, w.softmax_scale, causal)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, O, lse, do.to(dev), w.softmax_scale, causal, deterministic=True)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    check_grads({"dQ": dq.cpu(), "dK": dk.cpu(), "dV": dv.cpu()}, ref, (B, H, N, D, causal))


def test_deterministic():
    """fa_bwd_deterministic is bit-reproducible; fa_bwd is too for dK, dV (owned by one CTA
    each) and up to the order of the fp32 additions for dQ."""
    w, (q, k, v, do) = _small(1, 4, 512, 64, False)
    dev = torch.device("cuda")
    O, lse, (qd, kd, vd) = gpu_forward(q, k, v, w.softmax_scale, False)
    dod = do.to(dev)
    runs = [fa.attention_backward(qd, kd, vd, O, lse, dod, w.softmax_scale, False, deterministic=True)
            for _ in range(2)]
    for a, b in zip(*runs):
        assert torch.equal(a, b)
    runs = [fa.attention_backward(qd, kd, vd, O, lse, dod, w.softmax_scale, False) for _ in range(2)]
    assert torch.equal(runs[0][1], runs[1][1]) and torch.equal(runs[0][2], runs[1][2])
    assert rel_fro(runs[0][0].cpu(), runs[1][0].cpu()) <= 1e-4
    b = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, False)
    assert torch.equal(b["O"], O.cpu()) and torch.equal(b["lse"], lse.cpu())


# ----------------------------------------------------------------------------- the five workloads
def test_c1_fp32_forward():
    w = workloads.WORKLOADS["c1_fp32_fwd"]
    q, k, v, _ = workloads.make_inputs(w)
    O, lse, _ = gpu_forward(q, k, v, w.softmax_scale, w.causal)
    ref_O, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, w.causal)
    assert rel_fro(O.cpu(), ref_O) <= TOL["f32_fro"]
    assert ((lse.cpu().double() - ref_lse).abs() / ref_lse.abs().clamp_min(1.0)).max() <= TOL["f32_lse"]


def test_fp32_path_small_shapes():
    # one row, ragged tails, several key chunks of each head dim (chunks of 64 keys at D <= 64
    # and 32 at D = 128; 8 query rows per CTA)
    for (B, H, N, D, causal) in [(1, 1, 1, 32, False), (2, 2, 100, 128, True), (1, 3, 333, 64, True),
                                 (1, 2, 1000, 64, False), (1, 1, 520, 128, True), (2, 1, 97, 32, False)]:
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
    # properties over every row and key of the full-size output
    assert torch.isfinite(got["O"].float()).all() and torch.isfinite(got["dK"].float()).all()
    assert torch.isfinite(got["dQ"].float()).all() and torch.isfinite(got["dV"].float()).all()
    _check_whole_output_invariants(q, k, do, got, w.softmax_scale)


def _check_whole_output_invariants(q, k, do, got, scale):
    """Invariants of causal attention that hold at any size, checked on every row:
    * lse_i >= s_ii (the diagonal key is allowed) and, by Jensen's inequality,
      lse_i >= scale * q_i . mean(k_0..k_i) + ln(i+1);
    * lse_i <= max_j s_ij + ln(i+1) <= scale * |q_i| * max_{j<=i} |k_j| + ln(i+1);
    * rows of dS sum to zero, so sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0;
    * rows of P sum to one, so sum_j dV_j = sum_i dO_i.
    The gradient sums carry the kernels' rounding errors; if those are independent
    across keys, the norm of their sum is about the Frobenius norm of the error, which
    parity bounds by 1e-2 of the gradient's norm: the checks allow twice that."""
    qd, kd = q.double(), k.double()
    N = q.shape[2]
    cnt = torch.arange(1, N + 1, dtype=torch.float64)
    lse = got["lse"].double()
    diag = scale * (qd * kd).sum(-1)
    kmean = kd.cumsum(2) / cnt.view(1, 1, N, 1)
    jensen = scale * (qd * kmean).sum(-1) + torch.log(cnt)
    kmax = torch.cummax(kd.norm(dim=-1), dim=2).values
    upper = scale * qd.norm(dim=-1) * kmax + torch.log(cnt)
    slack = TOL["lse_max"] + 1e-6 * lse.abs()
    assert (lse >= diag - slack).all()
    assert (lse >= jensen - slack).all()
    assert (lse <= upper + slack).all()
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            dk, dv = got["dK"][b, h].double(), got["dV"][b, h].double()
            assert dk.sum(0).norm() <= 2 * TOL["grad_fro"] * dk.norm(), (b, h)
            assert (dv.sum(0) - do[b, h].double().sum(0)).norm() <= 2 * TOL["grad_fro"] * dv.norm(), (b, h)


def test_long_sequence_131072_sampled():
    """The longest point of the sequence-length sweep, N = 131072 (B1 H1 D128 causal), on
    64 sampled query rows and 64 sampled key rows, plus the whole-output invariants."""
    w = workloads.custom("n131072", 1, 1, 131072, 128, True, seed=1131)
    q, k, v, do = workloads.make_inputs(w, with_grad_out=True)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, True)
    qrows, krows = {0: workloads.sample_rows(w, 0)}, {0: workloads.sample_rows(w, 0, seed_base=3000)}
    ref = oracle.attention_sampled_rows(q, k, v, do, w.softmax_scale, True, qrows, krows, chunk=1024)[0]
    r, c = qrows[0], krows[0]
    check_fwd(got["O"][0, 0, r], got["lse"][0, 0, r], ref["O"], ref["lse"], "n131072 sampled")
    check_grads({"dQ": got["dQ"][0, 0, r], "dK": got["dK"][0, 0, c], "dV": got["dV"][0, 0, c]},
                {"dQ": ref["dQ"], "dK": ref["dK"], "dV": ref["dV"]}, "n131072 sampled")
    _check_whole_output_invariants(q, k, do, got, w.softmax_scale)


def test_device_status_clean():
    assert fa.fa_device_status(reset=False) == 0
