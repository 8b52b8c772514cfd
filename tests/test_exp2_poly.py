"""The FMA-pipe exp2 used by the kernels (exp2_poly2 in sm100_ptx.cuh): its
constants are the Remez minimax fit that gen_exp2_poly.py derives, and their
float32 evaluation stays within its stated relative-error bound against the
exact 2^x.  (The kernels' end results are checked against the oracle by the GPU
parity tests.)"""
import importlib.util
import re
import struct
from pathlib import Path

import numpy as np

CSRC = Path(__file__).resolve().parents[1] / "exact_attention_107_b200" / "csrc"


def _gen():
    spec = importlib.util.spec_from_file_location("gen_exp2_poly", CSRC / "gen_exp2_poly.py")
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _header_coefficients():
    text = (CSRC / "sm100_ptx.cuh").read_text()
    out = []
    for k in range(4):
        m = re.search(rf"kExp2C{k} = [0-9.]+f;\s*// 0x([0-9a-f]{{8}})", text)
        assert m, k
        out.append(struct.unpack(">f", bytes.fromhex(m.group(1)))[0])
    return np.array(out, dtype=np.float32)


def test_header_constants_are_the_remez_fit():
    g = _gen()
    fit = g.remez_relative(g.DEGREE).astype(np.float32)
    assert np.array_equal(fit, _header_coefficients())


def test_float32_evaluation_error_bound():
    g = _gen()
    c = _header_coefficients()
    xs = np.concatenate([np.linspace(-125.0, 10.0, 2_000_001), np.arange(-125, 11, dtype=np.float64)])
    rel = np.abs(g.eval_f32(xs, c).astype(np.float64) / np.exp2(xs) - 1.0)
    assert rel.max() < 7.8e-5
    # below the clamp the result is tiny, never negative or garbage
    tiny = g.eval_f32(np.array([-126.0, -300.0, -np.inf]), c)
    assert np.all(tiny > 0) and np.all(tiny < 3e-38)
    # NaN stays NaN (as through the MUFU ex2), so a NaN score is not silently dropped
    assert np.isnan(g.eval_f32(np.array([np.nan, -np.nan]), c)).all()
    # 2^n exactly at the integers where the polynomial is exact to its bound
    ints = np.arange(-125, 11, dtype=np.float64)
    assert np.all(np.abs(g.eval_f32(ints, c) / np.exp2(ints) - 1.0) < 7.8e-5)


def test_minimax_equioscillates():
    """A best approximation equioscillates: the relative error reaches +-E at
    degree+2 points of alternating sign."""
    g = _gen()
    c = g.remez_relative(g.DEGREE)
    f = np.linspace(-0.5, 0.5, 200001)
    err = np.polynomial.polynomial.polyval(f, c) / np.exp2(f) - 1.0
    E = np.abs(err).max()
    peaks = [i for i in range(1, len(f) - 1) if abs(err[i]) >= abs(err[i - 1]) and abs(err[i]) >= abs(err[i + 1])]
    peaks = [0] + peaks + [len(f) - 1]
    big = [err[i] for i in peaks if abs(err[i]) > 0.99 * E]
    assert len(big) >= g.DEGREE + 2
    assert all(np.sign(a) != np.sign(b) for a, b in zip(big, big[1:]))
