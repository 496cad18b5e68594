"""Host-side helpers of bench.py (no GPU): the algorithmic byte count, the
committed DRAM-traffic lookup, the clock-record parsing and its rejection
reasons, and the JSON of the reference arm's line."""

from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from lm_head_projection_b200.workloads import CE_WORKLOADS, WORKLOADS  # noqa: E402


def test_algorithmic_bytes_of_the_headline():
    w = WORKLOADS["bf16_bt1024_h4096_v128256"]
    X = 1024 * 4096 * 2
    Wb = 128256 * 4096 * 2
    Q = 1024 * 128256 * 2
    dX = X
    dW = 128256 * 4096 * 4  # fp32 head gradient
    assert bench.algorithmic_bytes(w) == float(X + Wb + Q + dX + dW)


def test_algorithmic_bytes_of_cross_entropy_counts_targets_not_q():
    w = CE_WORKLOADS["ce_bf16_bt1024_h4096_v128256"]
    assert bench.algorithmic_bytes(w) < bench.algorithmic_bytes(
        WORKLOADS["bf16_bt1024_h4096_v128256"])


def test_dram_traffic_lookup_follows_the_kernel_sources():
    v = bench.dram_traffic("bf16_bt1024_h4096_v128256", "chunk")
    path = os.path.join(ROOT, "profiles", "traffic_bf16_bt1024_h4096_v128256.md")
    text = open(path).read()
    if f"`{bench.kernel_source_hash()}`" in text:
        assert v is not None and v > 1e8
    else:
        assert v is None  # captured on other kernel sources: not reported
    assert bench.dram_traffic("no_such_workload", "chunk") is None


def test_kernel_hash_ignores_comments_but_not_code():
    src = ('int a = 1; // one\n/* two\n lines */ const char* s = "x // y /* z */";\n'
           "char q = '\"';  int b = 2;\n")
    assert bench.code_only(src) == ('int a = 1; const char* s = "x // y /* z */"; '
                                    "char q = '\"'; int b = 2;")
    assert bench.code_only(src.replace("// one", "// changed")) == bench.code_only(src)
    assert bench.code_only(src.replace("b = 2", "b = 3")) != bench.code_only(src)


def _sampler_with(tmp_path, lines, t0=None, t1=None):
    s = object.__new__(bench.ClockSampler)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.proc = object()  # a sampler that ran
    s.t0, s.t1 = t0, t1
    return s


def _ts(sec):
    import datetime
    return datetime.datetime.fromtimestamp(sec).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]


def test_clock_summary_keeps_the_timed_region_only(tmp_path):
    t = 1_700_000_000.0
    idle = [f"{_ts(t + 0.02 * i)}, 0, 1965, 1965, 300.0, 0x0, Not Active, Not Active, "
            "Not Active, Not Active" for i in range(10)]
    load = [f"{_ts(t + 0.2 + 0.02 * i)}, 0, 1400, 1965, 999.0, 0x4, Not Active, Not Active, "
            "Not Active, Active" for i in range(8)]
    after = [f"{_ts(t + 0.4 + 0.02 * i)}, 0, 1965, 1965, 300.0, 0x0, Not Active, Not Active, "
             "Not Active, Not Active" for i in range(5)]
    r = _sampler_with(tmp_path, idle + load + after, t0=t + 0.19, t1=t + 0.37).summary()
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert r["samples"] == 8 and r["window"] == "timed region"
    assert r["sm_mhz"] == 1400.0 and r["power_w_median"] == 999.0


def test_clock_summary_of_a_region_shorter_than_the_period(tmp_path):
    t = 1_700_000_000.0
    rows = [f"{_ts(t + 0.02 * i)}, 0, {1200 + i}, 1965, 800.0, 0x40, Not Active, Active, "
            "Not Active, Not Active" for i in range(6)]
    r = _sampler_with(tmp_path, rows, t0=t + 0.041, t1=t + 0.049).summary()
    assert r["samples"] == 1 and r["sm_mhz"] == 1203.0
    assert r["window"] == "first sample after the timed region"
    assert "hw_thermal_slowdown" in r["reasons"]


def test_clock_summary_without_samples(tmp_path):
    r = _sampler_with(tmp_path, ["garbage"]).summary()
    assert r["sm_mhz"] is None and r["reasons"] == ["no samples"]


def test_sm_clock_summary_from_a_trace():
    import torch

    # 1 ms apart, clock counter advancing 1500 cycles per microsecond
    t = [1_000_000 * i for i in range(11)]
    c = [1_500_000 * i for i in range(11)]
    buf = torch.tensor([v for pair in zip(t, c) for v in pair], dtype=torch.int64)
    r = bench.sm_clock_summary(buf, window_ms=5.5)
    assert r["median"] == 1500 and r["samples"] == 5


def test_kernel_roofline_counts_the_method_flops_against_the_burst_peak():
    w = WORKLOADS["bf16_bt1024_h4096_v128256"]
    g = 2.0 * w.BT * w.H * w.V
    steps = 2
    # per kind: [ms over all steps, launches, executed GEMM FLOPs]
    per_kind = {"stats": [2 * 0.8, 2, 2 * g], "grad": [2 * 0.1, 2, 2 * g / 8],
                "chunk": [2 * 2.4, 16, 2 * (g * 2 + g * 7 / 8)], "combine": [2 * 0.03, 2, 0.0]}
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    r = bench.kernel_roofline(w, per_kind, steps, peaks, "measured", 3.4)
    assert r["kernel_ms_per_step"] == pytest.approx(3.3)
    assert r["achieved"] == pytest.approx(round(3 * g / 3.3e-3 / 1e12, 1))
    assert r["peak"] == 1600.0 and r["frac"] == pytest.approx(r["achieved"] / 1600.0, abs=1e-4)
    assert r["executed_flops_per_step"] == pytest.approx(4 * g)
    assert r["frac_executed_of_burst"] > r["frac"]
    assert r["share_of_step"] == pytest.approx(3.3 / 3.4, abs=1e-4)


def test_step_roofline_cap_and_fractions():
    w = WORKLOADS["bf16_bt2048_h4096_v128256_frozen_ignore_t2_sum"]
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    ms = w.flops_counted() / 1600e12 * 1e3 * 2  # half of the burst roofline rate
    r = bench.step_roofline(w, ms, peaks, "measured")
    assert r["frac_of_burst"] == pytest.approx(0.5, abs=1e-4)
    assert r["cap_with_recompute"] == pytest.approx(2 / 3, abs=1e-4)
    # with the executed GEMM FLOPs of a call (first chunk not recomputed)
    executed = w.flops_counted() * 1.4
    r = bench.step_roofline(w, ms, peaks, "measured", executed=executed)
    assert r["cap_with_recompute"] == pytest.approx(1 / 1.4, abs=1e-4)


def test_max_over_ranks_without_a_group_is_the_value():
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
