"""Benchmark: attention TFLOPS, forward and forward + backward, on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = the whole hot path on one batch, through the C ABI: the forward (fa_fwd,
or fa_fwd_f32 for the fp32 workload) and, for workloads with a backward, its three
kernels (row statistics + accumulator zeroing, the fused dK/dV/dQ kernel, dQ finish).
Default workload: long-context causal attention, B1 H8 N65536 D128 (the D=128,
N>=4096 configuration the metric is quoted on); the other four workloads (fp32
forward, bf16 forward, non-causal and GPT-2-style fwd+bwd) run with --workload.

Throughput accounting (algorithmic, attention convention):
    F_fwd = 4 * B * H * N^2 * D, halved when causal
    value = 2.5 * F_fwd / (t_fwd + t_bwd)   for workloads with a backward (the headline)
          = F_fwd / t_fwd                   for forward-only workloads
    detail: fwd_tflops, bwd_tflops = 2.5 F_fwd / t_bwd, fwd_bwd_tflops_3_5x = 3.5 F_fwd / (t_fwd + t_bwd)
Cold L2: when a workload's inputs are smaller than twice the 126 MB L2, a 256 MiB
buffer is written between steps (outside the timed spans); larger inputs evict L2
by themselves.  The `l2` field of `config` says which.  With N GPUs (torchrun),
every rank runs its own copy of the workload (independent batch/head shards, no
collective on the data path): weak scaling, time = max over ranks.

--impl reference times the fp64 CPU oracle (the only reference this method has: the
pages ship no code) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import workloads  # noqa: E402

METRIC = "attention TFLOPS fwd and fwd+bwd (bf16, 1 B200); % of dense BF16 tensor peak"
PEAKS_FILE = ROOT / "MEASURED_PEAKS.json"
TRAFFIC_FILE = ROOT / "profiles" / "dram_traffic.json"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's published dense BF16 tensor throughput of one B200 (the datasheet's 4.5 PFLOP/s
# is with 2:4 sparsity), reported as a third denominator.
DATASHEET_BF16_TFLOPS = 2250.0
# Plain fp32 FFMA peak, for the fp32 path: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz.
FP32_FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
L2_BYTES = 126e6
FLUSH_BYTES = 256 << 20
KERNEL_SOURCES = {
    "fwd": "exact_attention_107_b200/csrc/fa_fwd_sm100.cu",
    "fwd_f32": "exact_attention_107_b200/csrc/fa_fwd_f32.cu",
    "bwd_main": "exact_attention_107_b200/csrc/fa_bwd_fused_sm100.cu",
    "bwd_finish": "exact_attention_107_b200/csrc/fa_bwd_fused_sm100.cu",
    "bwd_pre": "exact_attention_107_b200/csrc/fa_bwd_sm100.cu",
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="c5_long_causal", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shape", default=None,
                    help="B,H,N,D,causal: a custom bf16 fwd+bwd workload of the same recipe (profiling small cases)")
    a = ap.parse_args(argv)
    if a.shape:
        B, H, N, D, c = (int(x) for x in a.shape.split(","))
        name = f"custom_B{B}_H{H}_N{N}_D{D}_{'causal' if c else 'full'}"
        workloads.WORKLOADS[name] = workloads.custom(name, B, H, N, D, bool(c), seed=1010)
        a.workload = name
    return a


def load_peaks():
    if PEAKS_FILE.exists():
        return json.loads(PEAKS_FILE.read_text()), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(rel: str) -> str:
    return hashlib.sha256((ROOT / rel).read_bytes()).hexdigest()[:12]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/dram_traffic.json), if the
    kernel source is unchanged since the capture; None otherwise."""
    if not TRAFFIC_FILE.exists():
        return None
    for e in json.loads(TRAFFIC_FILE.read_text()).get("entries", []):
        if e.get("kernel") == kernel and e.get("workload") == workload:
            if e.get("source_sha") == source_sha(KERNEL_SOURCES[kernel]):
                return float(e["bytes_per_launch"])
    return None


def input_bytes(w) -> int:
    elem = 4 if w.dtype == "fp32" else 2
    return (4 if w.backward else 3) * w.B * w.H * w.N * w.D * elem


def needs_flush(w) -> bool:
    """Inputs smaller than twice the L2 could stay cached between steps: flush."""
    return input_bytes(w) < 2 * L2_BYTES


def l2_label(w) -> str:
    mib = input_bytes(w) / 2**20
    if needs_flush(w):
        return f"inputs {mib:.0f} MiB < 2 x L2: a {FLUSH_BYTES >> 20} MiB buffer is written before every step (untimed)"
    return f"inputs {mib:.0f} MiB > 2 x L2 (126 MB): no flush needed"


def kernel_names(w):
    if not w.backward:
        return ("fwd_f32",) if w.dtype == "fp32" else ("fwd",)
    return ("fwd", "bwd_pre", "bwd_main", "bwd_finish")


def algorithmic_flops(w):
    """Algorithmic FLOPs per launch of each kernel: the forward's two GEMMs (F_fwd) and the
    backward's five (QK^T, dO V^T, P^T dO, dS^T Q, dS K: 2.5 F_fwd, all in the fused kernel)."""
    f = w.fwd_flops()
    return {"fwd": f, "fwd_f32": f, "bwd_pre": 0.0, "bwd_main": 2.5 * f, "bwd_finish": 0.0}


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


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


def step_flops(w) -> float:
    """FLOPs of one step by the metric's count."""
    return (2.5 if w.backward else 1.0) * w.fwd_flops()


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
                          qkv_std=w.qkv_std, scale=w.scale, backward=w.backward)
    q_h, k_h, v_h, do_h = workloads.make_inputs(wr, with_grad_out=w.backward)
    B, H, N, D = q_h.shape
    scale, causal = w.softmax_scale, w.causal
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty(B, H, N, device=dev, dtype=torch.float32)
    if w.backward:
        do = do_h.to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(fa.fa_bwd_workspace_size(B, H, N, D), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, device=dev, dtype=torch.uint8) if needs_flush(w) else None
    names = kernel_names(w)
    fwd = fa.fa_fwd_f32 if w.dtype == "fp32" else fa.fa_fwd

    def step(ev=None):
        if flush is not None:
            flush.fill_(1)                 # evict L2 (not timed: the spans start after it)
        if ev is not None:
            ev[0].record(stream)
        fwd(q, k, v, o, lse, scale, causal, stream)
        if ev is not None:
            ev[1].record(stream)
        if w.backward:
            fa.fa_bwd_preprocess(o, do, lse, ws, stream)
            if ev is not None:
                ev[2].record(stream)
            fa.fa_bwd_dkdvdq(q, k, v, do, ws, dk, dv, scale, causal, stream)
            if ev is not None:
                ev[3].record(stream)
            fa.fa_bwd_dq_finish(ws, dq, scale, stream)
            if ev is not None:
                ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if fa.fa_device_status(reset=True) != 0:
        raise RuntimeError("device status error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            step(evs[i])
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    per = {n: [evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps)] for j, n in enumerate(names)}
    spans = [evs[i][0].elapsed_time(evs[i][-1]) for i in range(args.steps)]
    status = fa.fa_device_status(reset=True)
    if status != 0:
        raise RuntimeError(f"device status {status} after timed region")
    elapsed_ms = max_over_ranks(sum(spans), world, dev)

    # ---------------------------------------------------------------- end-to-end from host buffers
    e2e = None
    if not args.no_e2e:
        # Every step uploads its inputs from pinned host memory and downloads its results
        # (O, lse and, with a backward, dQ, dK, dV); HostStepPipeline overlaps step i's
        # kernels with the copies of its neighbours (two device buffer sets, copy streams).
        pinned = [t.pin_memory() for t in (q_h, k_h, v_h)] + [do_h.pin_memory() if w.backward else None]
        pipe = fa.HostStepPipeline(B, H, N, D, dtype=q.dtype, device=dev, backward=w.backward)
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


def cpu_baseline(w, full: bool, rows: int = 8192, heads=None, repeats: int = 1):
    """The fp64 oracle, as it stands, on the host cores: the whole workload (full), or a
    bounded sample of it, the causal (or leading) rows x rows block of each sampled head.
    Forward and backward where the workload has a backward.  Returns (TFLOPS by the
    metric's count, seconds, description)."""
    import oracle

    q, k, v, do = workloads.make_inputs(w, with_grad_out=w.backward)
    n = w.N if full else min(rows, w.N)
    heads = list(range(w.B * w.H)) if heads is None else heads
    mult = 2.5 if w.backward else 1.0
    t0 = time.time()
    flops = 0.0
    for _ in range(repeats):
        if full and heads == list(range(w.B * w.H)):
            if w.backward:
                oracle.attention_backward(q, k, v, do, w.softmax_scale, w.causal)
            else:
                oracle.attention_forward(q, k, v, w.softmax_scale, w.causal)
            flops += mult * w.fwd_flops()
            continue
        for bh in heads:
            b, h = divmod(bh, w.H)
            sl = (slice(b, b + 1), slice(h, h + 1), slice(0, n))
            if w.backward:
                oracle.attention_backward(q[sl], k[sl], v[sl], do[sl], w.softmax_scale, w.causal)
            else:
                oracle.attention_forward(q[sl], k[sl], v[sl], w.softmax_scale, w.causal)
            flops += mult * 4.0 * n * n * w.D / (2.0 if w.causal else 1.0)
    dt = time.time() - t0
    what = "fwd+bwd" if w.backward else "fwd"
    if full:
        desc = f"fp64 oracle {what} on the whole workload"
    else:
        desc = f"fp64 oracle {what} on the first {n} of {w.N} rows of {len(heads)} head(s)"
    desc += f", x{repeats}; BLAS threads {torch.get_num_threads()}"
    return flops / dt / 1e12, dt, desc


def oracle_runs_full(w) -> bool:
    """The oracle is timed on the whole workload where that takes seconds (every workload but
    the long-context one, whose S matrix per head alone is 32 GiB in fp64)."""
    return w.N <= 8192


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = workloads.WORKLOADS[args.workload]
    dtype = "f32" if w.dtype == "fp32" else w.dtype

    if args.impl == "reference":
        if rank != 0:
            return
        full = oracle_runs_full(w)
        heads = None if full else [0]
        tflops_s = []
        for _ in range(args.warmup):
            cpu_baseline(w, full, heads=heads)
        t_all = 0.0
        desc = ""
        for _ in range(args.steps):
            v, dt, desc = cpu_baseline(w, full, heads=heads)
            tflops_s.append(v)
            t_all += dt
        value = statistics.median(tflops_s)
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * t_all / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**w.describe(), "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cpu_cores(), "kind": "oracle",
                             "sample": desc},
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
    value = whole_job_tflops(world, step_flops(w), ms_step)
    mean = {n: statistics.mean(v) for n, v in per.items()}
    peaks, peak_kind = load_peaks()
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    alg = algorithmic_flops(w)
    timed = [n for n in per if alg[n] > 0]
    dom = max(timed, key=lambda n: mean[n])
    achieved = alg[dom] / (mean[dom] * 1e-3) / 1e12
    t_fwd = mean[kernel_names(w)[0]]
    t_bwd = sum(mean[n] for n in ("bwd_pre", "bwd_main", "bwd_finish") if n in mean)
    detail = {"t_fwd_ms": t_fwd, "t_kernels_ms": mean, "fwd_tflops": f_fwd / (t_fwd * 1e-3) / 1e12}
    if w.backward:
        detail.update({"t_bwd_ms": t_bwd, "bwd_tflops": 2.5 * f_fwd / (t_bwd * 1e-3) / 1e12,
                       "fwd_bwd_tflops_3_5x": whole_job_tflops(world, 3.5 * f_fwd, ms_step)})
    if w.dtype != "fp32":
        detail["fwd_frac_of_burst_peak"] = detail["fwd_tflops"] / peak_burst
        detail["value_frac_of_burst_peak"] = value / world / peak_burst
        detail["value_frac_of_datasheet_peak"] = value / world / DATASHEET_BF16_TFLOPS
    if w.dtype == "fp32":
        roofline = {"bound": "alu", "kernel": dom, "achieved": achieved, "peak": FP32_FFMA_TFLOPS,
                    "unit": "TFLOP/s", "frac": achieved / FP32_FFMA_TFLOPS,
                    "peak_kind": "derived fp32 FFMA peak: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz",
                    "traffic": recorded_traffic(dom, w.name)}
    else:
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak_burst, "unit": "TFLOP/s",
                    "frac": achieved / peak_burst,
                    "peak_kind": f"{peak_kind} bf16 burst (kernel timed on its own launches)",
                    "frac_of_sustained": achieved / peak_sust,
                    "frac_of_datasheet": achieved / DATASHEET_BF16_TFLOPS,
                    "traffic": recorded_traffic(dom, w.name)}
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        full = oracle_runs_full(w)
        v, dt, desc = cpu_baseline(w, full, repeats=1 if full else 3)
        cpu = {"value": v, "unit": "TFLOPS", "cores": cpu_cores(), "blas_threads": torch.get_num_threads(),
               "kind": "oracle", "sample": desc, "seconds": dt}
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "value_kind": "fwd+bwd (2.5 x F_fwd per step)" if w.backward else "fwd (F_fwd per step)",
        "config": {**w.describe(), "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": l2_label(w),
                   "flops": "F_fwd=4BHN^2D/(2 if causal); value=2.5*F_fwd/(t_fwd+t_bwd) (fwd only: F_fwd/t_fwd)"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "gpu_launches": len(per) * args.steps,
        "clocks": clocks,
        "detail": detail,
    }
    if e2e is not None:
        out["e2e"] = {"value": whole_job_tflops(world, step_flops(w), e2e["ms_per_step"]), "unit": "TFLOPS",
                      "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                      "ms_per_step": e2e["ms_per_step"]}
    print(json.dumps(out))


if __name__ == "__main__":
    main()
