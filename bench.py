"""Benchmark: attention TFLOPS, forward + backward, bf16, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the whole hot path on one batch: fa_fwd (forward, saves lse), then
the backward's three stages (delta preprocess, dK/dV kernel, dQ kernel), all
through the C ABI.  Default workload: long-context causal attention,
B1 H8 N65536 D128 (the spec D=128, N>=4096 configuration).

Throughput accounting (algorithmic, attention convention):
    F_fwd = 4 * B * H * N^2 * D, halved when causal
    value = 2.5 * F_fwd / (t_fwd + t_bwd)            ("metric-as-stated", the headline)
    detail.fwd_tflops = F_fwd / t_fwd, detail.bwd_tflops = 2.5 * F_fwd / t_bwd,
    detail.fwd_bwd_tflops_3_5x = 3.5 * F_fwd / (t_fwd + t_bwd)
Inputs (Q, K, V, dO: 4 x 128 MiB for the default workload) are larger than the
126 MB L2, so no flush is needed between steps.  With N GPUs (torchrun), every
rank runs its own copy of the workload (independent batch/head shards, no
collective on the data path): weak scaling, time = max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this method has:
the pages ship no code) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import workloads  # noqa: E402

PEAKS_FILE = ROOT / "MEASURED_PEAKS.json"
TRAFFIC_FILE = ROOT / "profiles" / "dram_traffic.md"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "fwd": "exact_attention_107_b200/csrc/fa_fwd_sm100.cu",
    "bwd_dkdv": "exact_attention_107_b200/csrc/fa_bwd_sm100.cu",
    "bwd_dq": "exact_attention_107_b200/csrc/fa_bwd_sm100.cu",
    "bwd_pre": "exact_attention_107_b200/csrc/fa_bwd_sm100.cu",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="c5_long_causal")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shape", default=None,
                    help="B,H,N,D,causal: a custom workload of the same recipe (profiling small cases)")
    a = ap.parse_args()
    if a.shape:
        B, H, N, D, c = (int(x) for x in a.shape.split(","))
        name = f"custom_B{B}_H{H}_N{N}_D{D}_{'causal' if c else 'full'}"
        workloads.WORKLOADS[name] = workloads.custom(name, B, H, N, D, bool(c), seed=1010)
        a.workload = name
    return a


def load_peaks():
    if PEAKS_FILE.exists():
        d = json.loads(PEAKS_FILE.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(rel: str) -> str:
    return hashlib.sha256((ROOT / rel).read_bytes()).hexdigest()[:12]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture, if the kernel source is unchanged since."""
    if not TRAFFIC_FILE.exists():
        return None
    for line in TRAFFIC_FILE.read_text().splitlines():
        m = re.match(r"\|\s*(\w+)\s*\|\s*(\w+)\s*\|\s*([0-9.eE+]+)\s*\|\s*([0-9a-f]{12})\s*\|", line)
        if m and m.group(1) == kernel and m.group(2) == workload:
            if m.group(4) == source_sha(KERNEL_SOURCES[kernel]):
                return float(m.group(3))
    return None


# ----------------------------------------------------------------------------- multi-rank helpers
def shard_seed(base_seed: int, rank: int) -> int:
    """Each rank holds its own batch/head shard of the same shape: its own input seed."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's value (timing is max over ranks); a no-op on one rank."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Aggregate throughput: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 200 ms) of one GPU while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        loaded = [s for s in sm if mx and s > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our implementation
def run_ours(args, rank, world, local_rank):
    import exact_attention_107_b200 as fa

    w = workloads.WORKLOADS[args.workload]
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # each rank holds its own shard of heads: same shapes, its own seed
    wr = workloads.custom(w.name, w.B, w.H, w.N, w.D, w.causal, dtype=w.dtype, seed=shard_seed(w.seed, rank),
                          qkv_std=w.qkv_std, scale=w.scale, backward=True)
    q_h, k_h, v_h, do_h = workloads.make_inputs(wr, with_grad_out=True)
    B, H, N, D = q_h.shape
    scale, causal = w.softmax_scale, w.causal
    q, k, v, do = (t.to(dev) for t in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, D), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    names = ("fwd", "bwd_pre", "bwd_dkdv", "bwd_dq")

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fa.fa_fwd(q, k, v, o, lse, scale, causal, stream)
        if ev is not None:
            ev[1].record(stream)
        fa.fa_bwd_preprocess(o, do, lse, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        fa.fa_bwd_dkdv(q, k, v, do, ws, dk, dv, scale, causal, stream)
        if ev is not None:
            ev[3].record(stream)
        fa.fa_bwd_dq(q, k, v, do, ws, dq, scale, causal, stream)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_device_status(reset=True) != 0:
        raise RuntimeError("device status error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    per = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)] for j, n in enumerate(names)}
    status = fa.fa_device_status(reset=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after timed region")

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)

    # ---------------------------------------------------------------- end-to-end from host buffers
    e2e = None
    if not args.no_e2e:
        # Every step uploads its inputs from pinned host memory and downloads O, lse, dQ,
        # dK, dV; HostStepPipeline overlaps step i's kernels with the copies of its
        # neighbours (two device buffer sets, separate copy streams).
        pinned = [t.pin_memory() for t in (q_h, k_h, v_h, do_h)]
        pipe = fa.HostStepPipeline(B, H, N, D, dtype=q.dtype, device=dev)
        outs = [pipe.host_outputs() for _ in range(pipe.depth)]
        for i in range(max(1, args.warmup)):
            pipe.submit(*pinned, outs[i % pipe.depth], scale, causal)
        pipe.synchronize()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(pipe.s_h2d)
        for i in range(args.steps):
            h2d, d2h = pipe.submit(*pinned, outs[i % pipe.depth], scale, causal)
        e1.record(pipe.s_d2h)
        pipe.synchronize()
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"ms_per_step": e2e_ms / args.steps, "h2d": h2d, "d2h": d2h}
    return w, per, elapsed_ms, clk.summary(), e2e


def cpu_baseline(w, rows: int = 8192, heads=None, repeats: int = 1):
    """The fp64 oracle, as it stands, on a bounded sample of the workload: the causal
    (or leading, if non-causal) rows x rows block of each sampled head, forward and
    backward.  Returns (TFLOPS by the metric's count, seconds, description)."""
    import oracle

    q, k, v, do = workloads.make_inputs(w, with_grad_out=True)
    n = min(rows, w.N)
    heads = list(range(w.B * w.H)) if heads is None else heads
    t0 = time.time()
    flops = 0.0
    for _ in range(repeats):
        for bh in heads:
            b, h = divmod(bh, w.H)
            sl = (slice(b, b + 1), slice(h, h + 1), slice(0, n))
            oracle.attention_backward(q[sl], k[sl], v[sl], do[sl], w.softmax_scale, w.causal)
            flops += 2.5 * 4.0 * n * n * w.D / (2.0 if w.causal else 1.0)
    dt = time.time() - t0
    desc = f"fp64 oracle fwd+bwd on the first {n} of {w.N} rows of {len(heads)} head(s), x{repeats}"
    return flops / dt / 1e12, dt, desc


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workloads.WORKLOADS[args.workload]
    metric = "attention TFLOPS fwd+bwd (bf16, 1 B200)"

    if args.impl == "reference":
        if rank != 0:
            return
        tflops_s = []
        for _ in range(args.warmup):
            cpu_baseline(w, heads=[0])
        t_all = 0.0
        for _ in range(args.steps):
            v, dt, desc = cpu_baseline(w, heads=[0])
            tflops_s.append(v)
            t_all += dt
        value = statistics.median(tflops_s)
        cores = torch.get_num_threads()
        print(json.dumps({
            "impl": "reference", "metric": metric, "value": value, "unit": "TFLOPS", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * t_all / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**w.describe(), "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    if world > 1:
        torch.cuda.set_device(local_rank)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    w, per, elapsed_ms, clocks, e2e = run_ours(args, rank, world, local_rank)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    f_fwd = w.fwd_flops()
    ms_step = elapsed_ms / args.steps
    value = whole_job_tflops(world, 2.5 * f_fwd, ms_step)
    mean = {n: statistics.mean(v) for n, v in per.items()}
    peaks, peak_kind = load_peaks()
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    # Algorithmic FLOPs per launch of each kernel (the backward's five GEMMs: the dK/dV
    # kernel does S, dP, dV, dK = 2 * F_fwd; the dQ kernel's algorithmic share is the
    # dQ GEMM = 0.5 * F_fwd, its recomputed S and dP are extra work).
    alg = {"fwd": f_fwd, "bwd_dkdv": 2.0 * f_fwd, "bwd_dq": 0.5 * f_fwd, "bwd_pre": 0.0}
    dom = max(("fwd", "bwd_dkdv", "bwd_dq"), key=lambda n: mean[n])
    achieved = alg[dom] / (mean[dom] * 1e-3) / 1e12
    detail = {
        "t_fwd_ms": mean["fwd"], "t_bwd_ms": mean["bwd_pre"] + mean["bwd_dkdv"] + mean["bwd_dq"],
        "t_kernels_ms": mean,
        "fwd_tflops": f_fwd / (mean["fwd"] * 1e-3) / 1e12,
        "bwd_tflops": 2.5 * f_fwd / ((mean["bwd_pre"] + mean["bwd_dkdv"] + mean["bwd_dq"]) * 1e-3) / 1e12,
        "fwd_bwd_tflops_3_5x": whole_job_tflops(world, 3.5 * f_fwd, ms_step),
    }
    detail["fwd_frac_of_burst_peak"] = detail["fwd_tflops"] / peak_burst
    detail["fwd_bwd_frac_of_burst_peak"] = value / world / peak_burst
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        v, dt, desc = cpu_baseline(w, repeats=3)
        cpu = {"value": v, "unit": "TFLOPS", "cores": torch.get_num_threads(), "kind": "oracle", "sample": desc,
               "seconds": dt}
    out = {
        "metric": metric, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**w.describe(), "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": "inputs (4 x %d MiB) larger than L2, no flush" % (w.B * w.H * w.N * w.D * 2 >> 20),
                   "flops": "F_fwd=4BHN^2D/(2 if causal); value=2.5*F_fwd/(t_fwd+t_bwd)"},
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak_sust, "unit": "TFLOP/s",
                     "frac": achieved / peak_sust,
                     "peak_kind": f"{peak_kind} bf16 sustained (kernel timed inside a long step loop)",
                     "frac_of_burst": achieved / peak_burst,
                     "traffic": recorded_traffic(dom, w.name)},
        "cpu_baseline": cpu,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "detail": detail,
    }
    if e2e is not None:
        out["e2e"] = {"value": whole_job_tflops(world, 2.5 * f_fwd, e2e["ms_per_step"]), "unit": "TFLOPS",
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                      "ms_per_step": e2e["ms_per_step"]}
    print(json.dumps(out))


if __name__ == "__main__":
    main()
