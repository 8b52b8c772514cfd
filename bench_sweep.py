"""Sequence-length sweep and standard-attention comparison on one B200.

    python bench_sweep.py nsweep   [--H 8] [--D 128] [--causal 1] [--Ns 1024,2048,...] [--dtype fp16]
    python bench_sweep.py standard [--workload c3_bf16_fwdbwd]
    python bench_sweep.py fwd      [--B 1] [--H 16] [--N 16384] [--D 256] [--causal 1] [--dtype bf16]

nsweep: for each N, forward and backward time (CUDA events, median of 5 after 2
warm-up runs) and peak device memory of the fused path (fa_fwd + fa_bwd through
the C ABI), next to the same for standard attention written as separate PyTorch
operations -- S = scale*QK^T, causal mask, softmax, O = PV, with autograd for the
backward -- which materialises the N x N matrices (the "three lines of PyTorch" of
"CUDA-kernel-level optimisation: why Flash Attention is 5-10x faster than native
PyTorch", guanweilu.cn).  The standard path is skipped where its N x N tensors
would need more than --std-limit-gb of device memory.  Prints a markdown table.

standard: the same comparison on one named workload, printing one JSON line.

fwd: forward only (any supported head dim, 256 included), one JSON line with the median
time of 10 launches after 3 warm-up launches and the attention TFLOP/s.

Inputs are seeded N(0,1) draws rounded to bf16, or to fp16 with --dtype fp16 (the
recipe of workloads.py).
"""
from __future__ import annotations

import argparse
import json
import math
import statistics

import torch

import exact_attention_107_b200 as fa
import workloads


def _time(fn, warmup=2, reps=5):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def fused_step(q, k, v, do, scale, causal):
    B, H, N, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=q.device, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, D), device=q.device, dtype=torch.uint8)

    f16 = q.dtype == torch.float16
    fwd_call, bwd_call = (fa.fa_fwd_f16, fa.fa_bwd_f16) if f16 else (fa.fa_fwd, fa.fa_bwd)

    def fwd():
        fwd_call(q, k, v, o, lse, scale, causal)

    def bwd():
        bwd_call(q, k, v, o, do, lse, dq, dk, dv, ws, scale, causal)

    return fwd, bwd


def standard_step(q, k, v, do, scale, causal):
    N = q.shape[2]
    mask = torch.ones(N, N, device=q.device, dtype=torch.bool).triu(1) if causal else None
    qr, kr, vr = (t.detach().clone().requires_grad_(True) for t in (q, k, v))
    state = {}

    def fwd():
        s = torch.matmul(qr, kr.transpose(-1, -2)) * scale
        if mask is not None:
            s = s.masked_fill(mask, float("-inf"))
        p = torch.softmax(s, dim=-1)
        state["o"] = torch.matmul(p, vr)

    def bwd():
        qr.grad = kr.grad = vr.grad = None
        state["o"].backward(do, retain_graph=True)

    return fwd, bwd


def measure(make, q, k, v, do, scale, causal):
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats()
    base = torch.cuda.memory_allocated()
    fwd, bwd = make(q, k, v, do, scale, causal)
    t_f = _time(fwd)
    t_b = _time(bwd)
    peak = torch.cuda.max_memory_allocated() - base
    return t_f, t_b, peak


def inputs(B, H, N, D, causal, seed=77, dtype="bf16"):
    w = workloads.custom("sweep", B, H, N, D, causal, dtype=dtype, seed=seed)
    return w, [t.cuda() for t in workloads.make_inputs(w, with_grad_out=True)]


def nsweep(args):
    Ns = [int(x) for x in args.Ns.split(",")]
    print(f"| N | fused fwd (ms) | fused bwd (ms) | fused fwd+bwd TFLOP/s (2.5x) | fused peak extra memory (GiB) "
          f"| standard fwd (ms) | standard bwd (ms) | standard peak extra memory (GiB) | speedup fwd / bwd |")
    print("|---|---|---|---|---|---|---|---|---|")
    for N in Ns:
        w, (q, k, v, do) = inputs(args.B, args.H, N, args.D, bool(args.causal), dtype=args.dtype)
        scale = w.softmax_scale
        ff, fb, fm = measure(fused_step, q, k, v, do, scale, w.causal)
        tfl = 2.5 * w.fwd_flops() / ((ff + fb) * 1e-3) / 1e12
        # standard: S, P (bf16) and their gradients, ~4 live N x N bf16 tensors per head at the peak
        need_gb = 4 * args.B * args.H * N * N * 2 / 2**30 + (1 if w.causal else 0) * N * N / 2**30
        if need_gb <= args.std_limit_gb:
            try:
                sf, sb, sm = measure(standard_step, q, k, v, do, scale, w.causal)
                std = f"{sf:.3f} | {sb:.3f} | {sm / 2**30:.2f} | {sf / ff:.1f}x / {sb / fb:.1f}x"
            except torch.OutOfMemoryError:
                std = "OOM | OOM | - | -"
        else:
            std = f"not run (~{need_gb:.0f} GiB of N x N tensors) | - | - | -"
        print(f"| {N} | {ff:.3f} | {fb:.3f} | {tfl:.0f} | {fm / 2**30:.3f} | {std} |", flush=True)
        del q, k, v, do
        torch.cuda.empty_cache()


def standard(args):
    w = workloads.WORKLOADS[args.workload]
    q, k, v, do = (t.cuda() for t in workloads.make_inputs(w, with_grad_out=True))
    ff, fb, fm = measure(fused_step, q, k, v, do, w.softmax_scale, w.causal)
    sf, sb, sm = measure(standard_step, q, k, v, do, w.softmax_scale, w.causal)
    f = w.fwd_flops()
    print(json.dumps({"workload": w.describe(),
                      "fused": {"fwd_ms": ff, "bwd_ms": fb, "peak_extra_gib": fm / 2**30,
                                "fwd_tflops": f / ff / 1e9, "fwd_bwd_tflops_2_5x": 2.5 * f / (ff + fb) / 1e9},
                      "standard_3_kernel": {"fwd_ms": sf, "bwd_ms": sb, "peak_extra_gib": sm / 2**30,
                                            "fwd_tflops": f / sf / 1e9, "fwd_bwd_tflops_2_5x": 2.5 * f / (sf + sb) / 1e9},
                      "speedup": {"fwd": sf / ff, "bwd": sb / fb, "fwd_bwd": (sf + sb) / (ff + fb)}}))


def fwd_only(args):
    w, (q, k, v, do) = inputs(args.B, args.H, args.N, args.D, bool(args.causal), dtype=args.dtype)
    fwd, _ = fused_step(q, k, v, do, w.softmax_scale, w.causal)
    t = _time(fwd, warmup=3, reps=10)
    assert fa.fa_device_status(reset=True) == 0
    print(json.dumps({"workload": w.describe(), "fwd_ms": t, "fwd_tflops": w.fwd_flops() / t / 1e9}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("mode", choices=["nsweep", "standard", "fwd"])
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--H", type=int, default=8)
    ap.add_argument("--D", type=int, default=128)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--Ns", default="1024,2048,4096,8192,16384,32768,65536,131072")
    ap.add_argument("--N", type=int, default=16384)
    ap.add_argument("--std-limit-gb", type=float, default=80.0)
    ap.add_argument("--dtype", choices=["bf16", "fp16"], default="bf16")
    ap.add_argument("--workload", default="c3_bf16_fwdbwd")
    args = ap.parse_args()
    torch.cuda.set_device(0)
    {"nsweep": nsweep, "standard": standard, "fwd": fwd_only}[args.mode](args)


if __name__ == "__main__":
    main()
