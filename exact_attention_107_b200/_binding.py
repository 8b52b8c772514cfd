"""ctypes binding for libfa.so (argument marshalling only).

Every function here checks the torch tensors it is given (device, dtype, shape,
contiguity), passes raw device pointers and the current CUDA stream to the C
ABI declared in include/fa.h, and raises FAError on a non-zero status.  No
arithmetic of the attention itself happens in Python: if libfa.so is missing,
loading fails loudly instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import math
import pathlib

import torch

LIB_PATH = pathlib.Path(__file__).resolve().with_name("libfa.so")

# Exported C symbols (the full list declared in include/fa.h).
SYMBOLS = (
    "fa_fwd", "fa_fwd_f32", "fa_bwd_workspace_size", "fa_bwd", "fa_bwd_preprocess",
    "fa_bwd_dkdv", "fa_bwd_dq", "fa_status_string", "fa_device_status", "fa_version",
    "fa_bwd_noalloc", "fa_fwd_f16", "fa_bwd_f16", "fa_bwd_deterministic",
    "fa_bwd_deterministic_workspace_size", "fa_bwd_dkdvdq", "fa_bwd_dq_finish",
)

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load_library() -> ctypes.CDLL:
    """Loads libfa.so (built in-tree by exact_attention_107_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise RuntimeError(f"{LIB_PATH} is missing; build it with `python -m exact_attention_107_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd_f32.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_fwd_f16.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_workspace_size.restype = sz
    lib.fa_bwd_deterministic_workspace_size.argtypes = [i, i, i, i]
    lib.fa_bwd_deterministic_workspace_size.restype = sz
    lib.fa_bwd_deterministic.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
    lib.fa_bwd_dkdvdq.argtypes = [vp, vp, vp, vp, vp, sz, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_dq_finish.argtypes = [vp, sz, vp, i, i, i, i, f, vp]
    lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
    lib.fa_bwd_f16.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, vp]
    lib.fa_bwd_preprocess.argtypes = [vp, vp, vp, vp, sz, i, i, i, i, vp]
    lib.fa_bwd_dkdv.argtypes = [vp, vp, vp, vp, vp, sz, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_dq.argtypes = [vp, vp, vp, vp, vp, sz, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
    lib.fa_bwd_noalloc.restype = i
    lib.fa_status_string.argtypes = [i]
    lib.fa_status_string.restype = ctypes.c_char_p
    lib.fa_device_status.argtypes = [i]
    lib.fa_version.argtypes = []
    for name in ("fa_fwd", "fa_fwd_f32", "fa_fwd_f16", "fa_bwd", "fa_bwd_f16", "fa_bwd_preprocess", "fa_bwd_dkdv",
                 "fa_bwd_dq", "fa_device_status", "fa_version", "fa_bwd_deterministic", "fa_bwd_dkdvdq",
                 "fa_bwd_dq_finish"):
        getattr(lib, name).restype = i
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().fa_status_string(int(status)).decode()


def _p(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, shape) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _raise(st: int, where: str) -> None:
    if st != 0:
        raise FAError(st, where)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)


# ----------------------------------------------------------------------------- C-ABI calls
def fa_fwd(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> None:
    """O, lse <- attention(q, k, v); bf16 (B,H,N,D) tensors, lse (B,H,N) float32."""
    _fwd16("fa_fwd", torch.bfloat16, q, k, v, o, lse, scale, causal, stream)


def fa_fwd_f16(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> None:
    """O, lse <- attention(q, k, v); fp16 (B,H,N,D) tensors, lse (B,H,N) float32."""
    _fwd16("fa_fwd_f16", torch.float16, q, k, v, o, lse, scale, causal, stream)


def _fwd16(name, dtype, q, k, v, o, lse, scale, causal, stream) -> None:
    B, H, N, D = q.shape
    for tn, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, tn, dtype, (B, H, N, D))
    _check(lse, "lse", torch.float32, (B, H, N))
    _raise(getattr(load_library(), name)(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, N, D, float(scale),
                                         int(causal), _stream(stream)), name)


def fa_fwd_f32(q, k, v, o, lse, scale: float, causal: bool, stream=None) -> None:
    """fp32 forward: float32 (B,H,N,D) tensors, lse (B,H,N) float32."""
    B, H, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _check(t, name, torch.float32, (B, H, N, D))
    _check(lse, "lse", torch.float32, (B, H, N))
    _raise(load_library().fa_fwd_f32(_p(q), _p(k), _p(v), _p(o), _p(lse), B, H, N, D, float(scale), int(causal),
                                     _stream(stream)), "fa_fwd_f32")


def fa_bwd_workspace_size(B: int, H: int, N: int, D: int) -> int:
    return int(load_library().fa_bwd_workspace_size(B, H, N, D))


def fa_bwd_deterministic_workspace_size(B: int, H: int, N: int, D: int) -> int:
    return int(load_library().fa_bwd_deterministic_workspace_size(B, H, N, D))


def fa_bwd(q, k, v, o, do, lse, dq, dk, dv, workspace, scale: float, causal: bool, stream=None) -> None:
    """dq, dk, dv <- gradients of attention (bf16); workspace: uint8 CUDA tensor of
    fa_bwd_workspace_size bytes.  dQ is summed in fp32 in a run-dependent order."""
    _bwd16("fa_bwd", torch.bfloat16, q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal, stream)


def fa_bwd_deterministic(q, k, v, o, do, lse, dq, dk, dv, workspace, scale: float, causal: bool,
                         stream=None) -> None:
    """Bit-reproducible bf16 backward (three stages, no atomics); workspace of at least
    fa_bwd_deterministic_workspace_size bytes."""
    _bwd16("fa_bwd_deterministic", torch.bfloat16, q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal,
           stream)


def fa_bwd_f16(q, k, v, o, do, lse, dq, dk, dv, workspace, scale: float, causal: bool, stream=None) -> None:
    """fa_bwd with fp16 tensors (o and lse from fa_fwd_f16)."""
    _bwd16("fa_bwd_f16", torch.float16, q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal, stream)


def _bwd16(name, dtype, q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal, stream) -> None:
    B, H, N, D = q.shape
    for tn, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, tn, dtype, (B, H, N, D))
    _check(lse, "lse", torch.float32, (B, H, N))
    wp, wn = _ws(workspace)
    _raise(getattr(load_library(), name)(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
                                         wp, wn, B, H, N, D, float(scale), int(causal), _stream(stream)), name)


def fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, scale: float, causal: bool, stream=None) -> None:
    """Like fa_bwd_deterministic (bf16, same results bit for bit) but with no workspace:
    for callers that cannot allocate device memory (they are handed only input and
    output buffers).  Uses the library's fixed 8 MiB scratch array, so problems with
    B*H*ceil(N/128)*128 > 1,048,576 rows are rejected and calls that overlap on the GPU
    must not share it."""
    B, H, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)):
        _check(t, name, torch.bfloat16, (B, H, N, D))
    _check(lse, "lse", torch.float32, (B, H, N))
    _raise(load_library().fa_bwd_noalloc(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), _p(dq), _p(dk), _p(dv),
                                         B, H, N, D, float(scale), int(causal), _stream(stream)),
           "fa_bwd_noalloc")


def _ws(workspace):
    if not (isinstance(workspace, torch.Tensor) and workspace.is_cuda and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return _p(workspace), workspace.numel() * workspace.element_size()


def fa_bwd_preprocess(o, do, lse, workspace, stream=None) -> None:
    """Backward stage 1: fills the workspace with -lse*log2(e) and delta = rowsum(dO * O)."""
    B, H, N, D = o.shape
    _check(o, "o", torch.bfloat16, (B, H, N, D))
    _check(do, "do", torch.bfloat16, (B, H, N, D))
    _check(lse, "lse", torch.float32, (B, H, N))
    wp, wn = _ws(workspace)
    _raise(load_library().fa_bwd_preprocess(_p(o), _p(do), _p(lse), wp, wn, B, H, N, D, _stream(stream)),
           "fa_bwd_preprocess")


def fa_bwd_dkdv(q, k, v, do, workspace, dk, dv, scale: float, causal: bool, stream=None) -> None:
    """Backward stage 2: dK, dV from the workspace filled by fa_bwd_preprocess."""
    B, H, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("do", do), ("dk", dk), ("dv", dv)):
        _check(t, name, torch.bfloat16, (B, H, N, D))
    wp, wn = _ws(workspace)
    _raise(load_library().fa_bwd_dkdv(_p(q), _p(k), _p(v), _p(do), wp, wn, _p(dk), _p(dv),
                                      B, H, N, D, float(scale), int(causal), _stream(stream)), "fa_bwd_dkdv")


def fa_bwd_dq(q, k, v, do, workspace, dq, scale: float, causal: bool, stream=None) -> None:
    """Backward stage 3: dQ from the workspace filled by fa_bwd_preprocess."""
    B, H, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("do", do), ("dq", dq)):
        _check(t, name, torch.bfloat16, (B, H, N, D))
    wp, wn = _ws(workspace)
    _raise(load_library().fa_bwd_dq(_p(q), _p(k), _p(v), _p(do), wp, wn, _p(dq),
                                    B, H, N, D, float(scale), int(causal), _stream(stream)), "fa_bwd_dq")


def fa_bwd_dkdvdq(q, k, v, do, workspace, dk, dv, scale: float, causal: bool, stream=None) -> None:
    """Fused backward stage 2: dK, dV, and dQ added into the workspace's fp32 accumulator
    (zeroed by fa_bwd_preprocess on a workspace of fa_bwd_workspace_size bytes)."""
    B, H, N, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("do", do), ("dk", dk), ("dv", dv)):
        _check(t, name, torch.bfloat16, (B, H, N, D))
    wp, wn = _ws(workspace)
    _raise(load_library().fa_bwd_dkdvdq(_p(q), _p(k), _p(v), _p(do), wp, wn, _p(dk), _p(dv),
                                        B, H, N, D, float(scale), int(causal), _stream(stream)), "fa_bwd_dkdvdq")


def fa_bwd_dq_finish(workspace, dq, scale: float, stream=None) -> None:
    """Fused backward stage 3: dq <- scale * the workspace's fp32 dQ accumulator, as bf16."""
    B, H, N, D = dq.shape
    _check(dq, "dq", torch.bfloat16, (B, H, N, D))
    wp, wn = _ws(workspace)
    _raise(load_library().fa_bwd_dq_finish(wp, wn, _p(dq), B, H, N, D, float(scale), _stream(stream)),
           "fa_bwd_dq_finish")


def workspace_views(workspace, B: int, H: int, N: int):
    """(nl, delta) float32 views of a backward workspace, each (B, H, Npad)."""
    npad = (N + 127) // 128 * 128
    f = workspace.view(torch.float32)[: 2 * B * H * npad].view(2, B, H, npad)
    return f[0], f[1]


def fa_device_status(reset: bool = False) -> int:
    return int(load_library().fa_device_status(int(reset)))


def fa_version() -> int:
    return int(load_library().fa_version())


# ----------------------------------------------------------------------------- convenience API
def attention_forward(q, k, v, scale: float | None = None, causal: bool = False, stream=None):
    """Returns (O, lse).  bf16 and fp16 inputs use the tensor-core path, float32 inputs the fp32 path."""
    B, H, N, D = q.shape
    scale = default_scale(D) if scale is None else scale
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=q.device, dtype=torch.float32)
    if q.dtype == torch.float32:
        fa_fwd_f32(q, k, v, o, lse, scale, causal, stream)
    elif q.dtype == torch.float16:
        fa_fwd_f16(q, k, v, o, lse, scale, causal, stream)
    else:
        fa_fwd(q, k, v, o, lse, scale, causal, stream)
    return o, lse


def attention_backward(q, k, v, o, lse, do, scale: float | None = None, causal: bool = False, stream=None,
                       workspace=None, deterministic: bool = False):
    """Returns (dQ, dK, dV) for bf16 or fp16 inputs (deterministic: bf16 only, the
    bit-reproducible three-stage path)."""
    B, H, N, D = q.shape
    scale = default_scale(D) if scale is None else scale
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    size_fn = fa_bwd_deterministic_workspace_size if deterministic else fa_bwd_workspace_size
    if workspace is None:
        workspace = torch.empty(size_fn(B, H, N, D), device=q.device, dtype=torch.uint8)
    if deterministic:
        bwd = fa_bwd_deterministic
    else:
        bwd = fa_bwd_f16 if q.dtype == torch.float16 else fa_bwd
    bwd(q, k, v, o, do, lse, dq, dk, dv, workspace, scale, causal, stream)
    return dq, dk, dv


class FlashAttention(torch.autograd.Function):
    """autograd wrapper: forward saves (q, k, v, O, lse); backward recomputes P from lse."""

    @staticmethod
    def forward(ctx, q, k, v, scale, causal):
        o, lse = attention_forward(q, k, v, scale, causal)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.scale, ctx.causal = scale, causal
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = attention_backward(q, k, v, o, lse, do.contiguous(), ctx.scale, ctx.causal)
        return dq, dk, dv, None, None


def flash_attention(q, k, v, scale: float | None = None, causal: bool = False):
    """Differentiable exact attention on bf16 or fp16 (B,H,N,D) CUDA tensors."""
    return FlashAttention.apply(q, k, v, default_scale(q.shape[-1]) if scale is None else scale, causal)


def attention_fwd_bwd_from_host(q_h, k_h, v_h, do_h, scale: float, causal: bool, dev_bufs=None, out=None,
                                stream=None):
    """One full step from host memory: copy q, k, v, dO (pinned host tensors) to the
    device, run forward and backward, and copy O, lse, dQ, dK, dV back to `out`
    (pinned host tensors, allocated when None).  Returns (out, h2d_bytes, d2h_bytes)."""
    B, H, N, D = q_h.shape
    dtype = q_h.dtype
    if dtype not in (torch.bfloat16, torch.float16):
        raise TypeError(f"q must be bfloat16 or float16, got {dtype}")
    if dev_bufs is None:
        dev = torch.device("cuda")
        dev_bufs = {n: torch.empty(B, H, N, D, device=dev, dtype=dtype)
                    for n in ("q", "k", "v", "do", "o", "dq", "dk", "dv")}
        dev_bufs["lse"] = torch.empty(B, H, N, device=dev, dtype=torch.float32)
        dev_bufs["ws"] = torch.empty(fa_bwd_workspace_size(B, H, N, D), device=dev, dtype=torch.uint8)
    if out is None:
        out = {n: torch.empty(B, H, N, D, dtype=dtype).pin_memory() for n in ("o", "dq", "dk", "dv")}
        out["lse"] = torch.empty(B, H, N, dtype=torch.float32).pin_memory()
    d = dev_bufs
    for n, h in (("q", q_h), ("k", k_h), ("v", v_h), ("do", do_h)):
        if h.dtype != dtype or d[n].dtype != dtype:
            raise TypeError(f"{n}: every input and device buffer must be {dtype}")
        d[n].copy_(h, non_blocking=True)
    fwd, bwd = (fa_fwd_f16, fa_bwd_f16) if dtype == torch.float16 else (fa_fwd, fa_bwd)
    fwd(d["q"], d["k"], d["v"], d["o"], d["lse"], scale, causal, stream)
    bwd(d["q"], d["k"], d["v"], d["o"], d["do"], d["lse"], d["dq"], d["dk"], d["dv"], d["ws"], scale, causal, stream)
    for n in ("o", "lse", "dq", "dk", "dv"):
        out[n].copy_(d[n], non_blocking=True)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h, do_h))
    d2h = sum(t.numel() * t.element_size() for t in out.values())
    return out, h2d, d2h


class HostStepPipeline:
    """Attention steps whose inputs and results live in pinned host memory, pipelined over
    `depth` sets of device buffers and three CUDA streams: the upload of step i+1 and the
    download of step i-1 run on the copy engines while step i computes.

    submit(q, k, v, do, out, scale, causal) queues one step: copy q, k, v (and dO when
    `backward`) from pinned host tensors of shape (B,H,N,D) to the device, run the forward
    (fa_fwd, fa_fwd_f16 or fa_fwd_f32 by dtype) and, when `backward`, fa_bwd / fa_bwd_f16
    on the compute stream, then copy O, lse (and dQ, dK, dV) into `out` (a dict of pinned
    host tensors, as returned by host_outputs()).  Results of a step are in `out` once
    synchronize() has returned; a caller keeping several steps in flight gives each its
    own `out`.  The library's own kernels do all the arithmetic; this class only orders
    copies and launches."""

    def __init__(self, B: int, H: int, N: int, D: int, dtype=torch.bfloat16, depth: int = 2, device=None,
                 backward: bool = True):
        if backward and dtype == torch.float32:
            raise ValueError("the fp32 path has no backward")
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.shape, self.dtype, self.depth, self.backward = (B, H, N, D), dtype, depth, backward
        self.inputs = ("q", "k", "v", "do") if backward else ("q", "k", "v")
        self.outputs = ("o", "lse", "dq", "dk", "dv") if backward else ("o", "lse")
        self.bufs = []
        for _ in range(depth):
            b = {n: torch.empty(B, H, N, D, device=dev, dtype=dtype)
                 for n in self.inputs + tuple(n for n in self.outputs if n != "lse")}
            b["lse"] = torch.empty(B, H, N, device=dev, dtype=torch.float32)
            self.bufs.append(b)
        self.ws = (torch.empty(fa_bwd_workspace_size(B, H, N, D), device=dev, dtype=torch.uint8)
                   if backward else None)
        self.s_h2d, self.s_comp, self.s_d2h = (torch.cuda.Stream(dev) for _ in range(3))
        self.ev_loaded = [torch.cuda.Event() for _ in range(depth)]    # inputs of the slot on the device
        self.ev_computed = [torch.cuda.Event() for _ in range(depth)]  # slot's kernels done
        self.ev_fetched = [torch.cuda.Event() for _ in range(depth)]   # slot's results copied out
        self.used = [False] * depth
        self.i = 0

    def host_outputs(self):
        B, H, N, D = self.shape
        out = {n: torch.empty(B, H, N, D, dtype=self.dtype).pin_memory() for n in self.outputs if n != "lse"}
        out["lse"] = torch.empty(B, H, N, dtype=torch.float32).pin_memory()
        return out

    def submit(self, q_h, k_h, v_h, do_h, out, scale: float, causal: bool):
        """Queues one step (do_h is ignored without `backward`); returns (h2d_bytes, d2h_bytes)
        of its copies."""
        s = self.i % self.depth
        b = self.bufs[s]
        hosts = (q_h, k_h, v_h, do_h)[: len(self.inputs)]
        if self.used[s]:
            self.s_h2d.wait_event(self.ev_computed[s])     # the kernels of step i-depth read these inputs
        with torch.cuda.stream(self.s_h2d):
            for n, h in zip(self.inputs, hosts):
                b[n].copy_(h, non_blocking=True)
        self.ev_loaded[s].record(self.s_h2d)
        self.s_comp.wait_event(self.ev_loaded[s])
        if self.used[s]:
            self.s_comp.wait_event(self.ev_fetched[s])     # step i-depth's results have left these buffers
        fwd = {torch.float16: fa_fwd_f16, torch.float32: fa_fwd_f32}.get(self.dtype, fa_fwd)
        fwd(b["q"], b["k"], b["v"], b["o"], b["lse"], scale, causal, self.s_comp)
        if self.backward:
            bwd = fa_bwd_f16 if self.dtype == torch.float16 else fa_bwd
            bwd(b["q"], b["k"], b["v"], b["o"], b["do"], b["lse"], b["dq"], b["dk"], b["dv"], self.ws, scale, causal,
                self.s_comp)
        self.ev_computed[s].record(self.s_comp)
        self.s_d2h.wait_event(self.ev_computed[s])
        with torch.cuda.stream(self.s_d2h):
            for n in self.outputs:
                out[n].copy_(b[n], non_blocking=True)
        self.ev_fetched[s].record(self.s_d2h)
        self.used[s] = True
        self.i += 1
        h2d = sum(t.numel() * t.element_size() for t in hosts)
        d2h = sum(out[n].numel() * out[n].element_size() for n in self.outputs)
        return h2d, d2h

    def synchronize(self):
        """Waits until every queued step's results are in host memory."""
        for st in (self.s_h2d, self.s_comp, self.s_d2h):
            st.synchronize()
