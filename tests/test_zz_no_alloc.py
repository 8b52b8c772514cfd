"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (code that a host framework hands only its input and output
buffers, with no workspace and no allocator) call fa_bwd_noalloc, which uses
the library's fixed scratch array instead of a caller workspace.  These tests
call it through the C ABI and check its results against fa_bwd's on two calls
in a row with different inputs (so stale scratch contents from the first call
would show up in the second), plus the capacity limit.  The file is named so
that pytest collects it last."""
import pytest
import torch

import exact_attention_107_b200 as fa
import workloads
from parity import TOL, rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _inputs(B, H, N, D, causal, seed):
    w = workloads.custom("noalloc", B, H, N, D, causal, seed=seed)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in workloads.make_inputs(w, with_grad_out=True))
    o, lse = fa.attention_forward(q, k, v, w.softmax_scale, causal)
    return w, q, k, v, do, o, lse


@pytest.mark.parametrize("shape", [(2, 3, 1000, 128, True), (1, 4, 2048, 64, False)])
def test_noalloc_matches_fa_bwd_on_two_calls(shape):
    B, H, N, D, causal = shape
    for call, seed in enumerate((21, 22)):
        w, q, k, v, do, o, lse = _inputs(B, H, N, D, causal, seed)
        ref = fa.attention_backward(q, k, v, o, lse, do, w.softmax_scale, causal)
        got = [torch.empty_like(q) for _ in range(3)]
        fa.fa_bwd_noalloc(q, k, v, o, do, lse, *got, w.softmax_scale, causal)
        torch.cuda.synchronize()
        assert fa.fa_device_status(reset=True) == 0
        for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
            err = rel_fro(a.cpu(), b.cpu())
            assert err <= TOL["grad_fro"], (call, name, err)


def test_noalloc_rejects_problems_beyond_its_scratch():
    q = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    lib = fa.load_library()
    p = q.data_ptr()
    # B*H*N = 64 * 65536 rows needs 16 MiB of scratch, twice the fixed array
    st = lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 64, 65536, 128, 0.08, 1, None)
    assert st == 11
    assert fa.status_string(st).startswith("FA_ERR_NOALLOC_CAPACITY")
