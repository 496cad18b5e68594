"""The input recipe (CPU): seeded generators give the same bytes on every
call, per-tensor streams are independent, and the stated structure holds —
teacher rows sum to 1, the peaked workload's exact zeros, the exact count of
dropped rows, targets in range, the norm inputs' shapes and offsets."""

from __future__ import annotations

import torch

from lm_head_projection_b200.workloads import (CE_WORKLOADS, NORM_SHAPES, WORKLOADS,
                                               make_inputs, make_norm_inputs, small_case)


def test_same_seed_same_bytes_and_streams_are_independent():
    w = small_case(dtype="bf16", BT=70, H=64, V=500, bias=True, ignore_frac=0.2, seed=3)
    a, b = make_inputs(w), make_inputs(w)
    for k in ("X", "W", "b", "Q", "shift_labels"):
        assert torch.equal(a[k], b[k]), k
    # a different dropped-row fraction draws the same X, W, Q (own streams)
    c = make_inputs(w.with_(ignore_frac=0.5))
    for k in ("X", "W", "b", "Q"):
        assert torch.equal(a[k], c[k]), k
    d = make_inputs(w.with_(seed=4))
    assert not torch.equal(a["X"], d["X"])


def test_teacher_rows_sum_to_one():
    w = small_case(dtype="fp32", BT=40, H=32, V=700, seed=1)
    Q = make_inputs(w)["Q"].double()
    assert torch.allclose(Q.sum(1), torch.ones(40, dtype=torch.float64), atol=1e-12)
    assert bool((Q > 0).all())


def test_peaked_workload_zeros_and_dropped_row_counts():
    w = WORKLOADS["bf16_bt4096_h4096_v128256_bias_mean_peaked"].with_(BT=8, H=64)
    Q = make_inputs(w)["Q"]
    zeros = (Q == 0).sum(1)
    assert bool((zeros >= round(0.05 * w.V)).all())  # 5 % set to exact 0 (bf16 may add more)
    w2 = WORKLOADS["bf16_bt2048_h4096_v128256_frozen_ignore_t2_sum"].with_(H=64, V=512)
    lab = make_inputs(w2)["shift_labels"]
    assert int((lab == -100).sum()) == round(0.1 * 2048) == 205
    kept = lab[lab != -100]
    assert bool(((kept >= 0) & (kept < w2.V)).all())


def test_cross_entropy_targets():
    w = CE_WORKLOADS["ce_bf16_bt1024_h4096_v128256"].with_(H=64, V=1000)
    inp = make_inputs(w)
    assert inp["Q"] is None and inp["target"].dtype == torch.int64
    t = inp["target"]
    assert int((t == -100).sum()) == round(0.1 * w.BT)
    kept = t[t != -100]
    assert bool(((kept >= 0) & (kept < w.V)).all())


def test_norm_inputs():
    assert (2048, 4096) in NORM_SHAPES and (8192, 8192) in NORM_SHAPES
    a = make_norm_inputs(64, 256, "bf16", 0)
    b = make_norm_inputs(64, 256, "bf16", 0)
    assert all(torch.equal(a[k], b[k]) for k in a)
    assert a["X"].shape == (64, 256) and a["W"].shape == (256,)
    # per-row offsets: row means spread well beyond the within-row noise / sqrt(H)
    assert float(a["X"].float().mean(1).std()) > 0.5
    assert abs(float(a["W"].float().mean()) - 1.0) < 0.05
