"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Such callers (code that a host framework hands only its input and output
buffers, with no workspace and no allocator) call fa_bwd_noalloc, which runs
the three kernels of fa_bwd_deterministic on the library's fixed scratch array
instead of a caller workspace.  These tests call it through the C ABI on calls
in a row: a large one that fills the scratch array, then smaller ragged ones
whose rows land where the first call left its statistics, so stale scratch
contents would show up.  Each result must equal fa_bwd_deterministic's bit for
bit (the same deterministic kernels), and match fa_bwd's within the gradient
tolerance.  The file is named so that pytest collects it last."""
import pytest
import torch

import exact_attention_107_b200 as fa
import workloads
from parity import TOL, rel_fro

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 * 1024 * 1024      # FA_NOALLOC_SCRATCH_BYTES in include/fa.h


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    yield


def _inputs(B, H, N, D, causal, seed):
    w = workloads.custom("noalloc", B, H, N, D, causal, seed=seed)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in workloads.make_inputs(w, with_grad_out=True))
    o, lse = fa.attention_forward(q, k, v, w.softmax_scale, causal)
    return w, q, k, v, do, o, lse


def test_noalloc_matches_the_deterministic_backward_on_calls_in_a_row():
    # B4 H16 N16384 fills the scratch array exactly (1,048,576 padded rows x 8 bytes).
    calls = [(4, 16, 16384, 64, True, 21), (1, 3, 1000, 128, True, 22), (2, 2, 777, 64, False, 23)]
    assert fa.fa_bwd_deterministic_workspace_size(*calls[0][:4]) == SCRATCH_BYTES
    for B, H, N, D, causal, seed in calls:
        w, q, k, v, do, o, lse = _inputs(B, H, N, D, causal, seed)
        got = [torch.empty_like(q) for _ in range(3)]
        fa.fa_bwd_noalloc(q, k, v, o, do, lse, *got, w.softmax_scale, causal)
        det = fa.attention_backward(q, k, v, o, lse, do, w.softmax_scale, causal, deterministic=True)
        fused = fa.attention_backward(q, k, v, o, lse, do, w.softmax_scale, causal)
        torch.cuda.synchronize()
        assert fa.fa_device_status(reset=True) == 0
        for name, a, b, c in zip(("dQ", "dK", "dV"), got, det, fused):
            assert torch.equal(a, b), (B, H, N, D, causal, name)
            err = rel_fro(a.cpu(), c.cpu())
            assert err <= TOL["grad_fro"], (B, H, N, D, causal, name, err)


def test_noalloc_rejects_problems_beyond_its_scratch():
    q = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    lib = fa.load_library()
    p = q.data_ptr()
    # B*H*N = 64 * 65536 padded rows need 32 MiB of statistics, four times the fixed array
    assert fa.fa_bwd_deterministic_workspace_size(1, 64, 65536, 128) > SCRATCH_BYTES
    st = lib.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 64, 65536, 128, 0.08, 1, None)
    assert st == 11
    assert fa.status_string(st).startswith("FA_ERR_NOALLOC_CAPACITY")
