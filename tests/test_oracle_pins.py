"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Closed forms, a hand-worked example (tests/golden), invariants of softmax
attention, brute force on tiny inputs, central finite differences for the
gradients, and torch's own CPU attention (with autograd) as a second witness.
Each family is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one mask) fails at least
one of them; ``test_planted_mistakes_are_caught`` plants such slips in copies
of the oracle's functions and checks that the pins catch every one.
"""
import json
import math
from pathlib import Path

import pytest
import torch

import oracle
from oracle import attention_ref as ref

F64 = torch.float64
GOLDEN = Path(__file__).parent / "golden"


def _sym(x):
    """Decode the symbolic entries used in the hand-worked fixture."""
    if isinstance(x, list):
        return [_sym(e) for e in x]
    if isinstance(x, (int, float)):
        return float(x)
    env = {"ln2": math.log(2.0), "ln3": math.log(3.0)}
    return float(eval(x, {"__builtins__": {}}, env))


def _t(x):
    return torch.tensor(_sym(x), dtype=F64).unsqueeze(0)   # add the batch axis: (1, H, N, D)


def rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=F64) * std


def max_abs(a, b):
    return (a - b).abs().max().item()


# --------------------------------------------------------------------------- hand-worked example
@pytest.mark.parametrize("causal", [False, True])
def test_hand_worked_example(causal):
    g = json.loads((GOLDEN / "hand_worked_n2_d2.json").read_text())
    q, k, v, do = _t(g["Q"]), _t(g["K"]), _t(g["V"]), _t(g["dO"])
    exp = g["causal" if causal else "noncausal"]
    O, lse = oracle.attention_forward(q, k, v, g["scale"], causal)
    assert max_abs(O, _t(exp["O"])) < 1e-14
    assert max_abs(lse, torch.tensor(_sym(exp["lse"]), dtype=F64).unsqueeze(0)) < 1e-14
    out = oracle.attention_backward(q, k, v, do, g["scale"], causal)
    for name in ("dQ", "dK", "dV"):
        assert max_abs(out[name], _t(exp[name])) < 1e-14, name
    O2, lse2 = oracle.attention_forward_online(q, k, v, g["scale"], causal, 1, 1)
    assert max_abs(O2, _t(exp["O"])) < 1e-14
    O3, _ = oracle.attention_bruteforce(q, k, v, g["scale"], causal)
    assert max_abs(O3, _t(exp["O"])) < 1e-14


# --------------------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_constant_scores_give_mean_of_v(causal):
    B, H, N, D = 2, 3, 17, 5
    q = rand((B, H, N, D), 1)
    k = torch.zeros(B, H, N, D, dtype=F64)
    v = rand((B, H, N, D), 2)
    O, lse = oracle.attention_forward(q, k, v, 0.3, causal)
    if causal:
        counts = torch.arange(1, N + 1, dtype=F64)
        mean = v.cumsum(dim=2) / counts.view(1, 1, N, 1)
        assert max_abs(lse, torch.log(counts).expand(B, H, N)) < 1e-13
    else:
        mean = v.mean(dim=2, keepdim=True).expand_as(v)
        assert max_abs(lse, torch.full((B, H, N), math.log(N), dtype=F64)) < 1e-13
    assert max_abs(O, mean) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_equal_key_rows_shift_lse_by_qu(causal):
    B, H, N, D = 1, 2, 12, 4
    q = rand((B, H, N, D), 3)
    u = rand((D,), 4)
    k = u.expand(B, H, N, D).clone()
    v = rand((B, H, N, D), 5)
    scale = 0.7
    O, lse = oracle.attention_forward(q, k, v, scale, causal)
    counts = torch.arange(1, N + 1, dtype=F64) if causal else torch.full((N,), float(N), dtype=F64)
    assert max_abs(lse, scale * (q @ u) + torch.log(counts)) < 1e-12
    mean = v.cumsum(dim=2) / counts.view(1, 1, N, 1) if causal else v.mean(dim=2, keepdim=True).expand_as(v)
    assert max_abs(O, mean) < 1e-12


def test_one_dominant_logit_selects_its_v_row():
    """q_i = gap * e_i and the keys are a permutation of the unit vectors, so row i has
    exactly one score equal to gap (key j* with k_j* = e_i) and N - 1 zero scores:
    O_i = (e^gap v_j* + sum_{j != j*} v_j) / (e^gap + N - 1), lse_i = ln(e^gap + N - 1)."""
    N = D = 6
    perm = [3, 0, 5, 1, 4, 2]                      # k_j = e_perm[j]
    for gap in (10.0, 45.0):
        q = gap * torch.eye(D, dtype=F64).view(1, 1, N, D)
        k = torch.eye(D, dtype=F64)[perm].view(1, 1, N, D)
        v = rand((1, 1, N, D), 6)
        O, lse = oracle.attention_forward(q, k, v, 1.0, False)
        for i in range(N):
            js = perm.index(i)
            w = torch.ones(N, dtype=F64)
            w[js] = math.exp(gap)
            expect = (w.view(N, 1) * v[0, 0]).sum(0) / w.sum()
            assert max_abs(O[0, 0, i], expect) < 1e-13
            assert abs(lse[0, 0, i].item() - math.log(math.exp(gap) + N - 1)) < 1e-13
            # and the selection itself: within (N-1) e^-gap of the dominant row
            assert max_abs(O[0, 0, i], v[0, 0, js]) <= 2 * (N - 1) * math.exp(-gap) * v.abs().max().item()


def test_causal_row0_is_v0():
    q, k, v = rand((2, 2, 10, 8), 7), rand((2, 2, 10, 8), 8), rand((2, 2, 10, 8), 9)
    scale = 0.45
    O, lse = oracle.attention_forward(q, k, v, scale, True)
    assert torch.equal(O[:, :, 0], v[:, :, 0])
    assert max_abs(lse[:, :, 0], scale * (q[:, :, 0] * k[:, :, 0]).sum(-1)) < 1e-14


# --------------------------------------------------------------------------- invariants
@pytest.mark.parametrize("causal", [False, True])
def test_softmax_invariants(causal):
    B, H, N, D = 2, 2, 23, 7
    q, k, v = rand((B, H, N, D), 10, 2.0), rand((B, H, N, D), 11, 2.0), rand((B, H, N, D), 12)
    scale = 1 / math.sqrt(D)
    P = oracle.attention_probs(q, k, scale, causal)
    assert max_abs(P.sum(-1), torch.ones(B, H, N, dtype=F64)) < 1e-13
    if causal:
        assert torch.all(P.triu(diagonal=1) == 0)
    O, lse = oracle.attention_forward(q, k, v, scale, causal)
    S = scale * q @ k.transpose(-1, -2)
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    smax = S.max(-1).values
    counts = torch.arange(1, N + 1, dtype=F64) if causal else torch.full((N,), float(N), dtype=F64)
    assert torch.all(lse >= smax - 1e-12) and torch.all(lse <= smax + torch.log(counts) + 1e-12)
    for i in range(N):   # each O coordinate lies in the hull of the allowed V rows
        hi = i + 1 if causal else N
        lo_v = v[:, :, :hi].min(dim=2).values
        hi_v = v[:, :, :hi].max(dim=2).values
        assert torch.all(O[:, :, i] >= lo_v - 1e-12) and torch.all(O[:, :, i] <= hi_v + 1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    B, H, N, D = 1, 3, 14, 5
    q, k, v = rand((B, H, N, D), 13), rand((B, H, N, D), 14), rand((B, H, N, D), 15)
    u = rand((D,), 16)
    scale = 0.6
    O1, lse1 = oracle.attention_forward(q, k, v, scale, causal)
    O2, lse2 = oracle.attention_forward(q, k + u, v, scale, causal)
    assert max_abs(O1, O2) < 1e-12
    assert max_abs(lse2 - lse1, scale * (q @ u)) < 1e-12


def test_key_permutation_invariance():
    B, H, N, D = 1, 2, 16, 4
    q, k, v = rand((B, H, N, D), 17), rand((B, H, N, D), 18), rand((B, H, N, D), 19)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(3))
    O1, lse1 = oracle.attention_forward(q, k, v, 0.5, False)
    O2, lse2 = oracle.attention_forward(q, k[:, :, perm], v[:, :, perm], 0.5, False)
    assert max_abs(O1, O2) < 1e-13 and max_abs(lse1, lse2) < 1e-13


# --------------------------------------------------------------------------- brute force / online softmax
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bm,bn", [(2, 2), (3, 4), (4, 3), (16, 5), (1, 16)])
def test_online_softmax_matches_naive(causal, bm, bn):
    B, H, N, D = 1, 2, 13, 6
    q, k, v = rand((B, H, N, D), 20, 3.0), rand((B, H, N, D), 21, 3.0), rand((B, H, N, D), 22)
    O1, lse1 = oracle.attention_forward(q, k, v, 0.8, causal)
    O2, lse2 = oracle.attention_forward_online(q, k, v, 0.8, causal, bm, bn)
    assert max_abs(O1, O2) < 1e-13
    assert max_abs(lse1, lse2) < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_bruteforce_matches_naive(causal):
    B, H, N, D = 1, 2, 7, 3
    q, k, v = rand((B, H, N, D), 23), rand((B, H, N, D), 24), rand((B, H, N, D), 25)
    O1, lse1 = oracle.attention_forward(q, k, v, 0.9, causal)
    O2, lse2 = oracle.attention_bruteforce(q, k, v, 0.9, causal)
    assert max_abs(O1, O2) < 1e-13 and max_abs(lse1, lse2) < 1e-13


# --------------------------------------------------------------------------- gradients
def _fd_grads(fwd, q, k, v, do, scale, causal, h=1e-6):
    """Central differences of L = sum(dO * O) with respect to every entry of q, k, v."""
    grads = []
    for which in range(3):
        base = [q.clone(), k.clone(), v.clone()]
        g = torch.zeros_like(base[which])
        flat = base[which].view(-1)
        for idx in range(flat.numel()):
            old = flat[idx].item()
            flat[idx] = old + h
            lp = (do * fwd(*base, scale, causal)[0]).sum().item()
            flat[idx] = old - h
            lm = (do * fwd(*base, scale, causal)[0]).sum().item()
            flat[idx] = old
            g.view(-1)[idx] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


def _check_grads(bwd_out, fd):
    for name, g in zip(("dQ", "dK", "dV"), fd):
        err = (bwd_out[name] - g).norm() / g.norm()
        if not err < 1e-7:
            return f"{name} rel err {err:.2e}"
    return None


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_finite_differences(causal):
    B, H, N, D = 1, 1, 8, 4
    q, k, v, do = (rand((B, H, N, D), s) for s in (30, 31, 32, 33))
    out = oracle.attention_backward(q, k, v, do, 0.7, causal)
    fd = _fd_grads(oracle.attention_forward, q, k, v, do, 0.7, causal)
    assert _check_grads(out, fd) is None


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_identities(causal):
    B, H, N, D = 2, 2, 19, 6
    q, k, v, do = (rand((B, H, N, D), s) for s in (40, 41, 42, 43))
    out = oracle.attention_backward(q, k, v, do, 0.4, causal)
    # rows of dS sum to zero, hence sum_j dK_j = scale * sum_i q_i * (sum_j dS_ij) = 0
    assert out["dK"].sum(dim=2).abs().max() < 1e-12
    # Delta = rowsum(P * dP) = rowsum(dO * O)
    assert max_abs(out["Delta"], oracle.attention_delta(out["O"], do)) < 1e-12
    # sum_j dV_j = sum_i dO_i (columns of P^T sum over the allowed keys to 1 per query row)
    assert max_abs(out["dV"].sum(dim=2), do.sum(dim=2)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_torch_cpu_attention_second_witness(causal):
    """torch's scaled_dot_product_attention on the CPU in fp64, with autograd, as a library witness."""
    B, H, N, D = 2, 3, 33, 8
    q, k, v, do = (rand((B, H, N, D), s) for s in (50, 51, 52, 53))
    scale = 0.31
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    O_t = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    O_t.backward(do)
    out = oracle.attention_backward(q, k, v, do, scale, causal)
    assert max_abs(out["O"], O_t.detach()) < 1e-13
    assert max_abs(out["dQ"], qt.grad) < 1e-12
    assert max_abs(out["dK"], kt.grad) < 1e-12
    assert max_abs(out["dV"], vt.grad) < 1e-12
    S = scale * q @ k.transpose(-1, -2)
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    lse_t = torch.logsumexp(S, dim=-1)
    assert max_abs(out["lse"], lse_t) < 1e-13


# --------------------------------------------------------------------------- sampled-row evaluation
@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_match_full(causal):
    B, H, N, D = 1, 2, 301, 8
    q, k, v, do = (rand((B, H, N, D), s) for s in (60, 61, 62, 63))
    scale = 1 / math.sqrt(D)
    full = oracle.attention_backward(q, k, v, do, scale, causal)
    g = torch.Generator().manual_seed(5)
    rows = {bh: torch.sort(torch.cat([torch.tensor([0, N - 1]), torch.randperm(N - 2, generator=g)[:20] + 1])).values
            for bh in range(B * H)}
    krows = {bh: torch.sort(torch.randperm(N, generator=g)[:22]).values for bh in range(B * H)}
    res = oracle.attention_sampled_rows(q, k, v, do, scale, causal, rows, krows, chunk=64)
    for bh in range(B * H):
        b, h = divmod(bh, H)
        r, c = rows[bh], krows[bh]
        assert max_abs(res[bh]["O"], full["O"][b, h, r]) < 1e-13
        assert max_abs(res[bh]["lse"], full["lse"][b, h, r]) < 1e-13
        assert max_abs(res[bh]["dQ"], full["dQ"][b, h, r]) < 1e-12
        assert max_abs(res[bh]["dK"], full["dK"][b, h, c]) < 1e-12
        assert max_abs(res[bh]["dV"], full["dV"][b, h, c]) < 1e-12


# --------------------------------------------------------------------------- the pins catch planted slips
def _mut_backward_no_delta(q, k, v, do, scale, causal):
    out = oracle.attention_backward(q, k, v, do, scale, causal)
    P = oracle.attention_probs(q, k, scale, causal)
    dP = do @ v.transpose(-1, -2)
    dS = P * dP                                     # slip: Delta term dropped
    out["dQ"] = scale * dS @ k
    return out


def _mut_backward_transposed_dk(q, k, v, do, scale, causal):
    out = oracle.attention_backward(q, k, v, do, scale, causal)
    P = oracle.attention_probs(q, k, scale, causal)
    dP = do @ v.transpose(-1, -2)
    dS = P * (dP - (P * dP).sum(-1, keepdim=True))
    out["dK"] = scale * dS @ q                      # slip: dS instead of dS^T
    return out


def _mut_backward_dq_unscaled(q, k, v, do, scale, causal):
    out = oracle.attention_backward(q, k, v, do, scale, causal)
    out["dQ"] = out["dQ"] / scale                   # slip: scale factor dropped
    return out


def _mut_forward_mask_off_by_one(q, k, v, scale, causal):
    S = scale * q @ k.transpose(-1, -2)
    N = q.shape[2]
    if causal:
        S = S.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(0), float("-inf"))   # slip: j >= i
        S[..., 0, 0] = 0.0
    P = torch.softmax(S, dim=-1)
    return P @ v, torch.logsumexp(S, -1)


def _mut_online_wrong_rescale(q, k, v, scale, causal, bm, bn):
    """Online softmax with the rescale factor inverted (exp(m_new - m))."""
    B, H, N, D = q.shape
    O = torch.empty_like(v)
    for b in range(B):
        for h in range(H):
            for i0 in range(0, N, bm):
                qi = q[b, h, i0:i0 + bm]
                m = torch.full((qi.shape[0], 1), float("-inf"), dtype=F64)
                l = torch.zeros(qi.shape[0], 1, dtype=F64)
                acc = torch.zeros(qi.shape[0], D, dtype=F64)
                for j0 in range(0, N, bn):
                    s_ = scale * qi @ k[b, h, j0:j0 + bn].transpose(0, 1)
                    m_new = torch.maximum(m, s_.max(1, keepdim=True).values)
                    p = torch.exp(s_ - m_new)
                    alpha = torch.exp(m_new - m) if j0 else torch.zeros_like(m)   # slip: sign
                    l = alpha * l + p.sum(1, keepdim=True)
                    acc = alpha * acc + p @ v[b, h, j0:j0 + bn]
                    m = m_new
                O[b, h, i0:i0 + bm] = acc / l
    return O, None


def test_planted_mistakes_are_caught():
    B, H, N, D = 1, 1, 8, 4
    q, k, v, do = (rand((B, H, N, D), s) for s in (70, 71, 72, 73))
    for causal in (False, True):
        fd = _fd_grads(oracle.attention_forward, q, k, v, do, 0.7, causal)
        for mut in (_mut_backward_no_delta, _mut_backward_transposed_dk, _mut_backward_dq_unscaled):
            assert _check_grads(mut(q, k, v, do, 0.7, causal), fd) is not None, mut.__name__
    # the off-by-one causal mask breaks the causal-row-0 and the prefix-mean closed forms
    kz = torch.zeros_like(k)
    O_bad, _ = _mut_forward_mask_off_by_one(q, kz, v, 0.7, True)
    prefix_mean = v.cumsum(dim=2) / torch.arange(1, N + 1, dtype=F64).view(1, 1, N, 1)
    assert max_abs(O_bad, prefix_mean) > 1e-3
    # a mis-scaled online accumulator breaks online == naive
    O1, _ = oracle.attention_forward(q, k, v, 0.7, False)
    O2, _ = _mut_online_wrong_rescale(q, k, v, 0.7, False, 2, 2)
    assert max_abs(O1, O2) > 1e-13
