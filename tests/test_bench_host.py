"""bench.py's host-side logic, without a GPU: the DRAM-traffic table is used only while
the kernel source still has the recorded hash, clock samples are summarised the way
the timing rules read them, and the throughput arithmetic counts the metric's FLOPs."""
import json

import bench
import workloads


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    sha = bench.source_sha(bench.KERNEL_SOURCES["bwd_main"])
    table = tmp_path / "traffic.json"
    table.write_text(json.dumps({"entries": [
        {"kernel": "bwd_main", "workload": "c5_long_causal", "bytes_per_launch": 4.254e9, "source_sha": sha},
        {"kernel": "fwd", "workload": "c5_long_causal", "bytes_per_launch": 2.241e9, "source_sha": "000000000000"},
    ]}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", table)
    assert bench.recorded_traffic("bwd_main", "c5_long_causal") == 4.254e9
    assert bench.recorded_traffic("fwd", "c5_long_causal") is None          # stale hash
    assert bench.recorded_traffic("bwd_main", "c3_bf16_fwdbwd") is None     # other workload


def test_clock_summary_reads_load_and_reasons():
    s = bench.ClockSampler(0)
    rows = ["0, 1965, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle sample
            "0, 1710, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1690, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active",
            "0, 1720, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active"]
    s.out = "\n".join(rows) + "\n"
    summary = s.summary()
    assert summary["sm_max_mhz"] == 1965.0
    assert summary["reasons"] == ["sw_power_cap"]
    assert summary["samples"] == 4
    assert 1690.0 <= summary["sm_mhz"] <= 1965.0
    s.out = ""
    assert s.summary()["reasons"] == ["unsampled"]


def test_throughput_arithmetic():
    w = workloads.WORKLOADS["c5_long_causal"]
    f = w.fwd_flops()
    assert f == 4.0 * 1 * 8 * 65536 ** 2 * 128 / 2                           # causal halves the count
    # the headline counts forward + backward as 2.5 forward passes, over the slowest rank
    assert abs(bench.whole_job_tflops(1, 2.5 * f, 35.0) - 2.5 * f / 35e-3 / 1e12) < 1e-9
    assert abs(bench.whole_job_tflops(4, 2.5 * f, 35.0) - 4 * bench.whole_job_tflops(1, 2.5 * f, 35.0)) < 1e-6
    assert bench.shard_seed(1005, 0) == 1005                                  # one GPU: the workload itself
    assert bench.shard_seed(1005, 0) != bench.shard_seed(1005, 1)


def test_l2_policy_and_kernel_lists():
    w = workloads.WORKLOADS
    # long-context: 4 x 128 MiB of inputs evict L2 by themselves
    assert not bench.needs_flush(w["c5_long_causal"]) and "no flush" in bench.l2_label(w["c5_long_causal"])
    # the others fit (or nearly fit) in twice the 126 MB L2: flushed between steps
    for name in ("c1_fp32_fwd", "c2_bf16_fwd", "c4_gpt2_causal", "c3_bf16_fwdbwd"):
        assert bench.needs_flush(w[name]), name
        assert "written before every step" in bench.l2_label(w[name])
    assert bench.input_bytes(w["c3_bf16_fwdbwd"]) == 4 * 4 * 16 * 4096 * 64 * 2
    assert bench.input_bytes(w["c1_fp32_fwd"]) == 3 * 2 * 256 * 64 * 4
    assert bench.kernel_names(w["c1_fp32_fwd"]) == ("fwd_f32",)
    assert bench.kernel_names(w["c2_bf16_fwd"]) == ("fwd",)
    assert bench.kernel_names(w["c5_long_causal"]) == ("fwd", "bwd_pre", "bwd_main", "bwd_finish")


def test_flop_accounting_per_kernel():
    w = workloads.WORKLOADS["c3_bf16_fwdbwd"]
    f = w.fwd_flops()
    alg = bench.algorithmic_flops(w)
    # the backward's five GEMMs all run in the fused kernel: 2.5 forward passes
    assert alg["bwd_main"] == 2.5 * f and alg["fwd"] == f and alg["bwd_pre"] == 0 and alg["bwd_finish"] == 0
    assert bench.step_flops(w) == 2.5 * f
    assert bench.step_flops(workloads.WORKLOADS["c2_bf16_fwd"]) == workloads.WORKLOADS["c2_bf16_fwd"].fwd_flops()
    # the fp32 roofline denominator: 148 SMs x 128 FFMA lanes x 2 FLOP at 1.965 GHz
    assert abs(bench.FP32_FFMA_TFLOPS - 74.45) < 0.01


def test_oracle_timing_scope_and_cores():
    w = workloads.WORKLOADS
    assert all(bench.oracle_runs_full(w[n]) for n in ("c1_fp32_fwd", "c2_bf16_fwd", "c3_bf16_fwdbwd", "c4_gpt2_causal"))
    assert not bench.oracle_runs_full(w["c5_long_causal"])
    import os
    assert bench.cpu_cores() == len(os.sched_getaffinity(0))


def test_cli_accepts_every_workload():
    for name in workloads.WORKLOADS:
        assert bench.parse_args(["--workload", name]).workload == name
