"""Full-size parity on sampled rows for the fp16 and head-dim-256 paths: the GPU runs the
whole problem; the fp64 oracle evaluates the plain definition on 64 seeded query rows and
64 key rows of a few heads (attention_sampled_rows), and every output is checked finite."""
import pytest
import torch

import oracle
import workloads
from parity import TOL, TOL_F16, check_fwd, check_grads, gpu_fwd_bwd

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _sampled_check(w, heads, tol):
    q, k, v, do = workloads.make_inputs(w, with_grad_out=True)
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, w.causal)
    qrows = {bh: workloads.sample_rows(w, bh) for bh in heads}
    krows = {bh: workloads.sample_rows(w, bh, seed_base=3000) for bh in heads}
    ref = oracle.attention_sampled_rows(q, k, v, do, w.softmax_scale, w.causal, qrows, krows, chunk=1024,
                                        heads=heads)
    cat = {n: [] for n in ("O", "lse", "dQ", "dK", "dV", "rO", "rlse", "rdQ", "rdK", "rdV")}
    for bh in heads:
        b, h = divmod(bh, w.H)
        r, c = qrows[bh], krows[bh]
        for n, rows in (("O", r), ("dQ", r), ("dK", c), ("dV", c)):
            cat[n].append(got[n][b, h, rows])
            cat["r" + n].append(ref[bh][n])
        cat["lse"].append(got["lse"][b, h, r])
        cat["rlse"].append(ref[bh]["lse"])
    j = {n: torch.cat(v) for n, v in cat.items()}
    check_fwd(j["O"], j["lse"], j["rO"], j["rlse"], w.name, tol=tol)
    check_grads({"dQ": j["dQ"], "dK": j["dK"], "dV": j["dV"]}, {"dQ": j["rdQ"], "dK": j["rdK"], "dV": j["rdV"]},
                w.name, tol=tol)
    for n in ("O", "dQ", "dK", "dV"):
        assert torch.isfinite(got[n].float()).all(), n


def test_fp16_long_context_sampled():
    """The long-context workload's shape (B1 H8 N65536 D128, causal) in fp16."""
    base = workloads.WORKLOADS["c5_long_causal"]
    w = workloads.custom("c5_fp16", base.B, base.H, base.N, base.D, True, dtype="fp16", seed=base.seed,
                         scale=base.softmax_scale)
    _sampled_check(w, heads=[0, 5], tol=TOL_F16)


@pytest.mark.parametrize("causal", [True, False])
def test_head_dim_256_sampled(causal):
    """Head dim 256 at N = 16384 (B1 H4), bf16."""
    w = workloads.custom("d256_16k", 1, 4, 16384, 256, causal, seed=1306 + causal)
    _sampled_check(w, heads=[1, 3], tol=TOL)
