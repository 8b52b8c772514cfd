"""Boundary tests that need no GPU: libfa.so loads, exports every symbol that
include/fa.h declares, and rejects bad arguments with the documented status
codes before touching any device."""
import ctypes
import re
from pathlib import Path

import pytest

import exact_attention_107_b200 as fa

HEADER = Path(__file__).resolve().parents[1] / "include" / "fa.h"


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(fa_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == sorted(fa.SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = fa.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings():
    for code in range(13):
        assert fa.status_string(code).startswith("FA_")
    assert fa.status_string(999) == "unknown fa_status"


def test_workspace_size():
    # fa_bwd: two float32 statistics (-lse*log2 e and delta) per padded row, plus the fp32
    # dQ accumulator of DK floats per padded row (DK = 64 for D <= 64, 128 for D in {96, 128});
    # rows = B*H*ceil(N/128)*128.  D = 256 has no fused path: statistics only.
    assert fa.fa_bwd_workspace_size(1, 8, 65536, 128) == 8 * 65536 * (2 + 128) * 4
    assert fa.fa_bwd_workspace_size(1, 1, 3, 64) == 128 * (2 + 64) * 4
    assert fa.fa_bwd_workspace_size(2, 3, 129, 64) == 6 * 256 * (2 + 64) * 4
    assert fa.fa_bwd_workspace_size(1, 1, 128, 32) == 128 * (2 + 64) * 4
    assert fa.fa_bwd_workspace_size(1, 1, 128, 96) == 128 * (2 + 128) * 4
    assert fa.fa_bwd_workspace_size(1, 1, 128, 80) == 0          # unsupported D
    assert fa.fa_bwd_workspace_size(1, 1, 128, 256) == 2 * 128 * 4
    for args in ((1, 8, 65536, 128), (2, 3, 129, 64), (1, 1, 128, 256), (1, 1, 1, 96)):
        B, H, N, D = args
        assert fa.fa_bwd_deterministic_workspace_size(*args) == 2 * B * H * ((N + 127) // 128 * 128) * 4
        assert fa.fa_bwd_workspace_size(*args) % 1024 == 0
    assert fa.fa_bwd_deterministic_workspace_size(1, 1, 128, 80) == 0


def test_noalloc_capacity_check_needs_no_gpu():
    lib = fa.load_library()
    # 8 MiB scratch = 1,048,576 padded rows; one more 128-row block is rejected
    assert lib.fa_bwd_noalloc(*([P] * 9), 1, 1, 1048576 + 1, 64, 0.1, 0, None) == 11
    assert lib.fa_bwd_noalloc(*([P] * 9), 1, 1, 128, 80, 0.1, 0, None) == 3


# Validation happens before any device call, so these run without a GPU.
P = ctypes.c_void_p(0x10000)        # an aligned, never-dereferenced fake address
U = ctypes.c_void_p(0x10008)        # misaligned
Z = None


def _fwd(q=P, k=P, v=P, o=P, lse=P, B=1, H=2, N=256, D=64, scale=0.125, causal=0):
    return fa.load_library().fa_fwd(q, k, v, o, lse, B, H, N, D, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=Z), 1), (dict(lse=Z), 1),
    (dict(B=0), 2), (dict(N=0), 2), (dict(H=-1), 2), (dict(B=2**30, H=2**30), 2),
    (dict(D=48), 3), (dict(D=16), 3), (dict(D=512), 3), (dict(D=80), 3), (dict(D=192), 3),
    (dict(k=U), 4), (dict(o=U), 4),
    (dict(scale=float("nan")), 10), (dict(scale=0.0), 10), (dict(scale=-1.0), 10), (dict(causal=2), 10),
])
def test_fwd_rejects_bad_arguments(kw, code):
    assert _fwd(**kw) == code


def test_fwd_f32_rejects_bad_arguments():
    lib = fa.load_library()
    assert lib.fa_fwd_f32(Z, P, P, P, P, 1, 1, 64, 64, 0.1, 0, None) == 1
    assert lib.fa_fwd_f32(P, P, P, P, P, 1, 1, 64, 48, 0.1, 0, None) == 3
    assert lib.fa_fwd_f32(P, P, P, P, P, 1, 1, 64, 96, 0.1, 0, None) == 3     # 96: 16-bit paths only
    assert lib.fa_fwd_f32(P, P, P, P, P, 300, 300, 64, 64, 0.1, 0, None) == 2   # B*H > 65535


def test_bwd_rejects_bad_arguments():
    lib = fa.load_library()
    ws = lib.fa_bwd_workspace_size(1, 2, 256, 64)
    args = [P] * 9
    assert lib.fa_bwd(*args, P, ws, 1, 2, 256, 64, 0.125, 0, None) != 6       # reaches the device check
    assert lib.fa_bwd(*args, Z, ws, 1, 2, 256, 64, 0.125, 0, None) == 8       # no workspace
    assert lib.fa_bwd(*args, P, ws - 1, 1, 2, 256, 64, 0.125, 0, None) == 8   # too small
    # the deterministic path's smaller workspace does not hold fa_bwd's dQ accumulator
    wsd = lib.fa_bwd_deterministic_workspace_size(1, 2, 256, 64)
    assert lib.fa_bwd(*args, P, wsd, 1, 2, 256, 64, 0.125, 0, None) == 8
    assert lib.fa_bwd(*args[:8], U, P, ws, 1, 2, 256, 64, 0.125, 0, None) == 4
    assert lib.fa_bwd(*args[:3], Z, *args[4:], P, ws, 1, 2, 256, 64, 0.125, 0, None) == 1
    assert lib.fa_bwd(*args, P, ws, 1, 2, 256, 80, 0.125, 0, None) == 3
    assert lib.fa_bwd(*args, P, ws, 1, 2, 256, 192, 0.125, 0, None) == 3
    ws1 = lib.fa_bwd_deterministic_workspace_size(1, 1, 128, 64)
    assert ws1 == 2 * 128 * 4
    assert lib.fa_bwd_dq(P, P, P, P, P, ws1, Z, 1, 1, 128, 64, 0.1, 0, None) == 1
    assert lib.fa_bwd_dkdv(P, P, P, P, P, ws1, P, U, 1, 1, 128, 64, 0.1, 0, None) == 4
    assert lib.fa_bwd_dkdv(P, P, P, P, P, ws1 - 16, P, P, 1, 1, 128, 64, 0.1, 0, None) == 8
    assert lib.fa_bwd_dq(P, P, P, P, U, ws1, P, 1, 1, 128, 64, 0.1, 0, None) == 4
    assert lib.fa_bwd_preprocess(P, P, Z, P, ws1, 1, 1, 128, 64, None) == 1
    assert lib.fa_bwd_preprocess(P, P, P, Z, ws1, 1, 1, 128, 64, None) == 8


def test_deterministic_bwd_rejects_bad_arguments():
    lib = fa.load_library()
    wsd = lib.fa_bwd_deterministic_workspace_size(1, 2, 256, 64)
    args = [P] * 9
    assert lib.fa_bwd_deterministic(*args, P, wsd, 1, 2, 256, 64, 0.125, 0, None) != 6   # reaches the device
    assert lib.fa_bwd_deterministic(*args, P, wsd - 1, 1, 2, 256, 64, 0.125, 0, None) == 8
    assert lib.fa_bwd_deterministic(*args, Z, wsd, 1, 2, 256, 64, 0.125, 0, None) == 8
    assert lib.fa_bwd_deterministic(*args[:2], Z, *args[3:], P, wsd, 1, 2, 256, 64, 0.125, 0, None) == 1
    assert lib.fa_bwd_deterministic(*args, U, wsd, 1, 2, 256, 64, 0.125, 0, None) == 4
    assert lib.fa_bwd_deterministic(*args, P, wsd, 1, 2, 256, 48, 0.125, 0, None) == 3
    assert lib.fa_bwd_deterministic(*args, P, wsd, 1, 2, 256, 64, float("nan"), 0, None) == 10


def test_fused_stages_reject_bad_arguments():
    lib = fa.load_library()
    ws = lib.fa_bwd_workspace_size(1, 1, 128, 64)
    wsd = lib.fa_bwd_deterministic_workspace_size(1, 1, 128, 64)
    assert lib.fa_bwd_dkdvdq(P, P, P, P, P, ws, Z, P, 1, 1, 128, 64, 0.1, 0, None) == 1
    assert lib.fa_bwd_dkdvdq(P, P, P, P, P, ws, P, U, 1, 1, 128, 64, 0.1, 0, None) == 4
    assert lib.fa_bwd_dkdvdq(P, P, P, P, P, wsd, P, P, 1, 1, 128, 64, 0.1, 0, None) == 8   # no accumulator
    assert lib.fa_bwd_dkdvdq(P, P, P, P, P, ws, P, P, 1, 1, 128, 256, 0.1, 0, None) == 3   # D = 256: no fused path
    assert lib.fa_bwd_dkdvdq(P, P, P, P, P, ws, P, P, 1, 1, 128, 64, 0.1, 5, None) == 10
    assert lib.fa_bwd_dq_finish(P, ws, Z, 1, 1, 128, 64, 0.1, None) == 1
    assert lib.fa_bwd_dq_finish(P, ws, U, 1, 1, 128, 64, 0.1, None) == 4
    assert lib.fa_bwd_dq_finish(P, wsd, P, 1, 1, 128, 64, 0.1, None) == 8
    assert lib.fa_bwd_dq_finish(Z, ws, P, 1, 1, 128, 64, 0.1, None) == 8
    assert lib.fa_bwd_dq_finish(P, ws, P, 1, 1, 128, 256, 0.1, None) == 3
    assert lib.fa_bwd_dq_finish(P, ws, P, 1, 1, 128, 64, -1.0, None) == 10
    assert lib.fa_bwd_dq_finish(P, ws, P, 0, 1, 128, 64, 0.1, None) == 2


def test_binding_requires_cuda_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fa_fwd(q, q, q, q, torch.zeros(1, 1, 128), 0.125, False)


@pytest.mark.parametrize("kw,code", [
    (dict(v=Z), 1), (dict(N=0), 2), (dict(D=48), 3), (dict(q=U), 4), (dict(scale=float("inf")), 10),
])
def test_fwd_f16_rejects_bad_arguments(kw, code):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=2, N=256, D=64, scale=0.125, causal=0)
    a.update(kw)
    assert fa.load_library().fa_fwd_f16(*a.values(), None) == code


def test_bwd_f16_rejects_bad_arguments():
    lib = fa.load_library()
    ws = lib.fa_bwd_workspace_size(1, 2, 256, 64)
    args = [P] * 9
    assert lib.fa_bwd_f16(*args, Z, ws, 1, 2, 256, 64, 0.125, 0, None) == 8
    assert lib.fa_bwd_f16(*args[:5], Z, *args[6:], P, ws, 1, 2, 256, 64, 0.125, 0, None) == 1
    assert lib.fa_bwd_f16(*args[:6], U, *args[7:], P, ws, 1, 2, 256, 64, 0.125, 0, None) == 4
    assert lib.fa_bwd_f16(*args, P, ws, 1, 2, 256, 112, 0.125, 0, None) == 3
    assert lib.fa_bwd_f16(*args, P, ws, 1, 2, 256, 64, 0.125, 3, None) == 10


def test_binding_checks_fp16_dtype():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):      # not on a CUDA device: rejected before the dtype
        fa.fa_fwd_f16(q, q, q, q, torch.zeros(1, 1, 128), 0.125, False)
