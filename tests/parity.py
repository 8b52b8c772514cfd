"""Helpers for comparing the CUDA path with the fp64 oracle (tests only).

Tolerances (bf16 inputs, fp32 accumulation), applied in fp64 on the CPU:
    O       relative Frobenius <= 5e-3 and max-abs <= 2e-2
    lse     max-abs <= 1e-3
    dQ/dK/dV relative Frobenius <= 1e-2 each
fp32 path: O relative Frobenius <= 1e-5, lse max-abs <= 1e-5 * max(1, |lse|).
fp16 path (TOL_F16): the same checks with the bf16 bounds scaled by the ratio of
the two unit roundoffs where 16-bit rounding dominates the error (fp16 keeps 11
significant bits, bf16 8: 2^-11 vs 2^-8, a factor 8), and a factor 3 of margin:
    O relative Frobenius <= 2e-3, max-abs <= 5e-3; lse max-abs <= 1e-3 (fp32
    arithmetic on both paths); dQ/dK/dV relative Frobenius <= 4e-3.
"""
from __future__ import annotations

import torch

import exact_attention_107_b200 as fa

TOL = {"O_fro": 5e-3, "O_max": 2e-2, "lse_max": 1e-3, "grad_fro": 1e-2, "f32_fro": 1e-5, "f32_lse": 1e-5}
TOL_F16 = {"O_fro": 2e-3, "O_max": 5e-3, "lse_max": 1e-3, "grad_fro": 4e-3}


def rel_fro(a, b) -> float:
    a, b = a.double(), b.double()
    return ((a - b).norm() / b.norm().clamp_min(1e-300)).item()


def max_abs(a, b) -> float:
    return (a.double() - b.double()).abs().max().item()


def check_fwd(O, lse, ref_O, ref_lse, label="", tol=TOL):
    e = {"O_fro": rel_fro(O, ref_O), "O_max": max_abs(O, ref_O), "lse_max": max_abs(lse, ref_lse)}
    assert e["O_fro"] <= tol["O_fro"], (label, e)
    assert e["O_max"] <= tol["O_max"], (label, e)
    assert e["lse_max"] <= tol["lse_max"], (label, e)
    return e


def check_grads(got: dict, ref: dict, label="", tol=TOL):
    """Relative Frobenius error of each gradient.  Where an exact gradient is zero
    (e.g. dQ and dK when every row attends to a single key, N = 1), the relative
    error is undefined; the denominator is then floored at 1e-3 of the largest
    reference gradient norm of the problem."""
    floor = 1e-3 * max(ref[n].double().norm().item() for n in ("dQ", "dK", "dV"))
    e = {n: (got[n].double() - ref[n].double()).norm().item() / max(ref[n].double().norm().item(), floor)
         for n in ("dQ", "dK", "dV")}
    for n, v in e.items():
        assert v <= tol["grad_fro"], (label, n, e)
    return e


def gpu_forward(q, k, v, scale, causal):
    dev = torch.device("cuda")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    O, lse = fa.attention_forward(qd, kd, vd, scale, causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    return O, lse, (qd, kd, vd)


def gpu_fwd_bwd(q, k, v, do, scale, causal):
    dev = torch.device("cuda")
    O, lse, (qd, kd, vd) = gpu_forward(q, k, v, scale, causal)
    dod = do.to(dev)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, O, lse, dod, scale, causal)
    torch.cuda.synchronize()
    assert fa.fa_device_status(reset=True) == 0
    return {"O": O.cpu(), "lse": lse.cpu(), "dQ": dq.cpu(), "dK": dk.cpu(), "dV": dv.cpu()}
