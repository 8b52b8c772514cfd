"""The debug build of the library (libfa_debug.so, compiled with FA_DEBUG_CHECKS).

That build checks on the device every computed global-memory index and shared-memory
offset against its buffer, and warp convergence at the entry of every phase that
issues warp-collective tensor-memory operations; a failed check records
FA_ERR_DEBUG_CHECK in the status word and skips the access.  A child process (its own
CUDA context and library instance) runs every kernel family from the debug build on
shapes with ragged tails, causal and not, each head dimension and element type, and
requires a clean status word after each call and results within the parity
tolerances of the fp64 oracle."""
import json
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parents[1]

CHILD = r"""
import json, sys
import torch
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
import exact_attention_107_b200._binding as b
b.LIB_PATH = b.LIB_PATH.with_name("libfa_debug.so")
b._lib = None
import oracle, workloads
from parity import TOL, TOL_F16, check_fwd, check_grads, rel_fro

out = {}
dev = torch.device("cuda")
cases = [(1, 2, 200, 64, True, "bf16"), (1, 2, 300, 128, False, "bf16"), (1, 2, 384, 96, True, "bf16"),
         (2, 1, 77, 32, True, "bf16"), (1, 2, 320, 256, True, "bf16"), (1, 2, 256, 64, True, "fp16"),
         (1, 1, 1, 128, True, "bf16")]
for B, H, N, D, causal, dt in cases:
    key = f"{B}x{H}x{N}x{D}{'c' if causal else ''}_{dt}"
    w = workloads.custom("dbg", B, H, N, D, causal, dtype=dt, seed=31)
    q, k, v, do = workloads.make_inputs(w, with_grad_out=True)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = b.attention_forward(qd, kd, vd, w.softmax_scale, causal)
    st_f = b.fa_device_status(True)
    dq, dk, dv = b.attention_backward(qd, kd, vd, o, lse, dod, w.softmax_scale, causal)
    st_b = b.fa_device_status(True)
    ref = oracle.attention_backward(q, k, v, do, w.softmax_scale, causal)
    tol = TOL_F16 if dt == "fp16" else TOL
    check_fwd(o.cpu(), lse.cpu(), ref["O"], ref["lse"], key, tol)
    check_grads({"dQ": dq.cpu(), "dK": dk.cpu(), "dV": dv.cpu()}, ref, key, tol)
    res = {"fwd": st_f, "bwd": st_b}
    if dt == "bf16":
        g = b.attention_backward(qd, kd, vd, o, lse, dod, w.softmax_scale, causal, deterministic=True)
        res["bwd_det"] = b.fa_device_status(True)
        check_grads({"dQ": g[0].cpu(), "dK": g[1].cpu(), "dV": g[2].cpu()}, ref, key + " det", tol)
        if D != 256:
            got = [torch.empty_like(qd) for _ in range(3)]
            b.fa_bwd_noalloc(qd, kd, vd, o, dod, lse, *got, w.softmax_scale, causal)
            res["noalloc"] = b.fa_device_status(True)
            assert all(torch.equal(x, y) for x, y in zip(got, g)), key
    out[key] = res
w = workloads.custom("dbg32", 1, 2, 100, 64, True, dtype="fp32", seed=32)
q, k, v, _ = workloads.make_inputs(w, with_grad_out=False)
o, lse = b.attention_forward(q.to(dev), k.to(dev), v.to(dev), w.softmax_scale, True)
out["fp32"] = {"fwd": b.fa_device_status(True)}
ref_o, ref_lse = oracle.attention_forward(q, k, v, w.softmax_scale, True)
assert rel_fro(o.cpu(), ref_o) <= TOL["f32_fro"]
print(json.dumps(out))
"""


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def test_debug_build_runs_clean_and_matches_the_oracle():
    lib = ROOT / "exact_attention_107_b200" / "libfa_debug.so"
    assert lib.exists(), "build the debug library first (python -m exact_attention_107_b200.build)"
    r = subprocess.run([sys.executable, "-c", CHILD, str(ROOT)], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert len(res) == 8
    for case, statuses in res.items():
        for call, st in statuses.items():
            assert st == 0, (case, call, st)
