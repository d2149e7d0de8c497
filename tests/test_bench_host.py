"""Host logic of the bench without a GPU: clock-sample parsing, the peak table, the
whole-job rate and the DRAM-traffic figure's source check."""
import json
import os

import bench


class _Done:
    """Stands in for a sampler process that has already exited."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(tmp_path, text):
    s = bench.ClockSampler(0)
    f = tmp_path / "clocks.csv"
    f.write_text(text)
    s.tmp = open(f, "a")
    s.proc = _Done()
    return s


def test_clock_sampler_median_max_and_reasons(tmp_path):
    rows = [
        "0, 1350, 1965, 812.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1400, 1965, 790.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1300, 1965, 805.0, 0x0000000000000008, Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    r = _sampler_with(tmp_path, "\n".join(rows) + "\n").stop()
    assert r["sm_mhz"] == 1350.0                      # median of the three parsable samples
    assert r["sm_max_mhz"] == 1965.0 and r["samples"] == 3
    assert r["power_w_max"] == 812.5
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_sampler_without_samples(tmp_path):
    assert _sampler_with(tmp_path, "").stop()["reasons"] == ["no samples"]
    assert bench.ClockSampler(0).stop()["reasons"] == ["nvidia-smi unavailable"]


def test_peaks_measured_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    fb = bench.peaks()
    assert fb["source"] == "fallback" and fb["hbm"] == 6650.0 and fb["bf16"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6548.2, "bf16_tflops": 1652.2, "bf16_tflops_sustained": 1379.2}))
    m = bench.peaks()
    assert m["source"] == "measured" and m["bf16_sustained"] == 1379.2 and m["hbm"] == 6548.2


def test_whole_job_rate_counts_every_rank():
    # 2 ranks x 16384 tokens x 10 steps in 40 ms of the slowest rank
    assert bench.whole_job_rate(2, 16384, 10, 40.0) == 2 * 16384 * 10 / 0.040
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_traffic_figure_names_its_gemm_source():
    """profiles/gemm_dram_traffic.json carries the sha256 of the GEMM source its counters
    were taken from; the bench reports the figure only while that source is unchanged
    (null otherwise)."""
    with open(os.path.join(bench.ROOT, "profiles", "gemm_dram_traffic.json")) as fh:
        tr = json.load(fh)
    sha = tr["source_sha256"]
    assert len(sha) == 64 and all(c in "0123456789abcdef" for c in sha)
    assert tr["bytes_per_step"] > 0 and tr["workload"]


def test_tensor_peak_burst_only_at_full_clock():
    pk = dict(bf16=1652.2, bf16_sustained=1379.2, sm_max_mhz=1965.0, hbm=6548.2)
    # a short run at the maximum clock: the burst figure (a matmul timed alone)
    short = bench.tensor_peak(pk, "bf16", {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, 0.06)
    assert short["which"] == "burst" and short["peak"] == 1652.2
    assert short["sustained"] == 1379.2 and short["nominal"] == 2250.0
    # power-capped clocks, or a long timed region: the sustained figure
    capped = bench.tensor_peak(pk, "bf16", {"sm_mhz": 1327.0, "sm_max_mhz": 1965.0}, 0.06)
    assert capped["which"] == "sustained" and capped["peak"] == 1379.2
    long = bench.tensor_peak(pk, "bf16", {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, 30.0)
    assert long["which"] == "sustained"
    # no clock record: the sustained figure (the conservative one)
    assert bench.tensor_peak(pk, "bf16", {"sm_mhz": None, "sm_max_mhz": None}, 0.06)["which"] \
        == "sustained"
    # other precisions scale by the nominal ratio to bf16
    fp8 = bench.tensor_peak(pk, "fp8", {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}, 0.06)
    assert abs(fp8["peak"] - 1652.2 * 2) < 1e-9 and fp8["nominal"] == 4500.0
    tf32 = bench.tensor_peak(pk, "tf32", {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0}, 0.06)
    assert abs(tf32["peak"] - 1379.2 * 1.1 / 2.25) < 1e-9


def test_nvml_sampler_summary_and_absence(monkeypatch):
    """The in-region sampler reports the median and minimum SM clock and the power of its
    samples; without a usable device it reports nothing (the nvidia-smi record stands)."""
    s = bench.NvmlSampler.__new__(bench.NvmlSampler)
    s.h, s.thread, s.stop_flag = None, None, False
    s.samples = []
    assert s.stop() == {}
    s.thread = type("T", (), {"join": lambda self, timeout=None: None})()
    s.samples = [(1965, 400.0), (1400, 990.0), (1500, 1000.0), (1450, 995.0)]
    r = s.stop()
    assert r["sm_mhz"] == 1475 and r["sm_mhz_min"] == 1400 and r["samples"] == 4
    assert r["power_w_max"] == 1000.0 and r["power_w_median"] == 992.5


def test_stage_launch_counts_match_the_launch_lists():
    """The per-step launch counts of the bench's stages (the line's gpu_launches claim):
    13 for the headline bf16 step and 22 for the MXFP8 step with the weight codes kept,
    the totals the ncu launch lists of those commands show per step."""
    from routing_grouped_gemm_route_b200.inputs import WORKLOADS
    steps = ["route", "dispatch", "gemm_fwd", "combine", "combine_bwd", "gemm_bwd",
             "dispatch_bwd"]
    n = bench.stage_launches(WORKLOADS["e128_bf16"], False)
    assert sum(n[s] for s in steps) == 13
    n = bench.stage_launches(WORKLOADS["e128_mxfp8_large"], True)
    assert sum(n[s] for s in steps) == 22
    assert bench.stage_launches(WORKLOADS["e128_mxfp8_large"], False)["gemm_bwd"] == 12
    # the tiny fp32 workload runs the router: + 1 forward, + 2 backward; TF32 weight copies
    n = bench.stage_launches(WORKLOADS["tiny_fp32"], False)
    assert sum(n[s] for s in ["router"] + steps + ["router_bwd"]) == 20
