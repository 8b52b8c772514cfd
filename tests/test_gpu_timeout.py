"""Device-side failure detection, exercised without a fault.

Every pipeline wait in the kernels (a TMA load landing, an MMA finishing, the
element-wise warps handing a tile over) is bounded.  When a bound runs out, the
kernel records FA_ERR_TIMEOUT in the library's device status word, raises its
CTA's abort flag so that the CTA's other waits give up too, collects its own
TMA copies and MMAs still in flight (those waits keep their full limit), frees
its tensor memory and returns: no trap, no hang, and the CUDA context stays
usable.

The test-only library libfa_timeout_test.so is built from the same sources with
the pipeline waits limited to 100 clocks, far less than any tile load takes, so
that every kernel runs a wait out and takes that path.  A child process (its own
CUDA context and library instance) calls each kernel family through the C ABI
and reports the status word after each call; the parent then checks that the
normal library, in this process, still computes parity-clean results."""
import json
import subprocess
import sys
from pathlib import Path

import pytest

import exact_attention_107_b200 as fa
import oracle
import workloads
from parity import check_fwd, check_grads, gpu_fwd_bwd

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parents[1]

CHILD = r"""
import json, sys
import torch
sys.path.insert(0, sys.argv[1])
import exact_attention_107_b200._binding as b
b.LIB_PATH = b.LIB_PATH.with_name("libfa_timeout_test.so")
b._lib = None
fa = b
dev = torch.device("cuda")
g = torch.Generator(device="cuda").manual_seed(0)
out = {}

def tensors(B, H, N, D, dtype):
    q, k, v, do = (torch.randn(B, H, N, D, device=dev, generator=g).to(dtype) for _ in range(4))
    o = torch.empty_like(q)
    lse = torch.zeros(B, H, N, device=dev)
    return q, k, v, do, o, lse

for D in (64, 128, 256):
    B, H, N, causal = 1, 2, 1024, True
    q, k, v, do, o, lse = tensors(B, H, N, D, torch.bfloat16)
    fa.fa_fwd(q, k, v, o, lse, D ** -0.5, causal)
    out[f"fwd_d{D}"] = fa.fa_device_status(True)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, D), device=dev, dtype=torch.uint8)
    fa.fa_bwd(q, k, v, o, do, lse, dq, dk, dv, ws, D ** -0.5, causal)
    out[f"bwd_d{D}"] = fa.fa_device_status(True)
    fa.fa_bwd_deterministic(q, k, v, o, do, lse, dq, dk, dv, ws, D ** -0.5, causal)
    out[f"bwd_det_d{D}"] = fa.fa_device_status(True)
q, k, v, do, o, lse = tensors(1, 2, 512, 64, torch.float16)
fa.fa_fwd_f16(q, k, v, o, lse, 0.125, False)
out["fwd_f16"] = fa.fa_device_status(True)
x = torch.arange(1000, device=dev, dtype=torch.float32)
out["context_usable"] = float((x * 2).sum().item()) == 999000.0
out["status_after_reset"] = fa.fa_device_status(False)
print(json.dumps(out))
"""


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def test_every_kernel_reports_a_timed_out_wait_and_returns():
    lib = ROOT / "exact_attention_107_b200" / "libfa_timeout_test.so"
    assert lib.exists(), "build the test library first (python -m exact_attention_107_b200.build)"
    r = subprocess.run([sys.executable, "-c", CHILD, str(ROOT)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    timeout = 7                                           # FA_ERR_TIMEOUT
    for name, st in res.items():
        if name.startswith(("fwd", "bwd")):
            assert st == timeout, (name, res)
    assert res["context_usable"] is True
    assert res["status_after_reset"] == 0


def test_normal_library_is_parity_clean_after_the_timeout_run():
    w = workloads.custom("after_timeout", 1, 2, 384, 128, True, seed=77)
    q, k, v, do = workloads.make_inputs(w, with_grad_out=True)
    assert fa.fa_device_status(reset=False) == 0
    got = gpu_fwd_bwd(q, k, v, do, w.softmax_scale, True)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, True)
    check_fwd(got["O"], got["lse"], ref["O"], ref["lse"])
    check_grads(got, ref)
