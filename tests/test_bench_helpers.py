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


def _sampler_with(tmp_path, lines):
    s = object.__new__(bench.ClockSampler)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.proc = object()  # a sampler that ran
    return s


def test_clock_summary_median_under_load_and_reasons(tmp_path):
    rows = ["0, 1965, 1965, 300.0, 0x0, Not Active, Not Active, Not Active, Not Active"] * 4
    rows += ["0, 1400, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active"] * 8
    s = _sampler_with(tmp_path, rows)
    r = s.summary()
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    assert r["samples"] == 12
    assert 1400.0 <= r["sm_mhz"] <= 1965.0


def test_clock_summary_reports_thermal_slowdown(tmp_path):
    rows = ["0, 1200, 1965, 800.0, 0x40, Not Active, Active, Not Active, Not Active"] * 3
    r = _sampler_with(tmp_path, rows).summary()
    assert "hw_thermal_slowdown" in r["reasons"]


def test_clock_summary_without_samples(tmp_path):
    r = _sampler_with(tmp_path, ["garbage"]).summary()
    assert r["sm_mhz"] is None and r["reasons"] == ["no samples"]


def test_max_over_ranks_without_a_group_is_the_value():
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
