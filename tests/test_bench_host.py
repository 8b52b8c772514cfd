"""bench.py's host-side logic, without a GPU: the DRAM-traffic table is used only while
the kernel source still has the recorded hash, clock samples are summarised the way
the timing rules read them, and the throughput arithmetic counts the metric's FLOPs."""
import bench
import workloads


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    sha = bench.source_sha(bench.KERNEL_SOURCES["bwd_dkdv"])
    table = tmp_path / "traffic.md"
    table.write_text("| kernel | workload | bytes_per_launch | source_sha |\n|---|---|---|---|\n"
                     f"| bwd_dkdv | c5_long_causal | 4.2540e+09 | {sha} |\n"
                     "| fwd | c5_long_causal | 2.2410e+09 | 000000000000 |\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", table)
    assert bench.recorded_traffic("bwd_dkdv", "c5_long_causal") == 4.254e9
    assert bench.recorded_traffic("fwd", "c5_long_causal") is None          # stale hash
    assert bench.recorded_traffic("bwd_dkdv", "c3_bf16_fwdbwd") is None     # other workload


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
