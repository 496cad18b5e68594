"""Parity of the fused linear cross-entropy path (one-hot teacher at an
integer target) with its fp64 oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import lm_head_projection_b200 as pkg
from lm_head_projection_b200.workloads import CE_WORKLOADS, make_inputs, small_case
from tests.parity_utils import assert_close, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

SMALL = [
    # dtype, BT, H, V, bias, reduction, T, ignore_frac, dW, db
    ("bf16", 133, 192, 1000, True, "batchmean", 1.0, 0.1, True, True),
    ("bf16", 300, 256, 4104, False, "sum", 2.0, 0.0, True, False),
    ("bf16", 1, 64, 8, False, "mean", 1.0, 0.0, True, False),
    ("bf16", 257, 320, 3000, True, "batchmean", 0.5, 0.3, False, False),
    ("fp32", 133, 72, 1000, True, "batchmean", 1.0, 0.1, True, True),
    ("fp32", 3, 64, 4104, False, "sum", 1.5, 0.0, True, False),
]


@pytest.mark.parametrize("case", SMALL, ids=[f"{c[0]}-{c[1]}x{c[2]}x{c[3]}-{c[5]}" for c in SMALL])
def test_small_ce_matches_oracle(case):
    dt, BT, H, V, bias, red, T, ig, dW, db = case
    w = small_case(dtype=dt, BT=BT, H=H, V=V, bias=bias, reduction=red, temperature=T,
                   ignore_frac=ig, compute_dW=dW, compute_db=db, seed=BT + 7 * V, ce=True)
    inp = make_inputs(w)
    assert_close(dt, run_gpu(inp), run_oracle(inp))


def test_ce_out_of_range_targets_contribute_nothing():
    w = small_case(dtype="bf16", BT=64, H=64, V=520, bias=False, ce=True)
    inp = make_inputs(w)
    inp["target"][[3, 9]] = torch.tensor([520, -7])
    got = run_gpu(inp)
    assert not torch.any(got["dX"][[3, 9]].cpu() != 0)
    assert_close("bf16", got, run_oracle(inp))


def test_ce_equals_kl_with_one_hot_teacher_on_gpu():
    """The cross-entropy entry and the KL entry with a materialised one-hot
    teacher agree (bf16 one-hot is exact)."""
    w = small_case(dtype="bf16", BT=200, H=128, V=2056, bias=True, ignore_frac=0.1, ce=True)
    inp = make_inputs(w)
    ce = run_gpu(inp)
    Q = torch.zeros((w.BT, w.V), dtype=torch.bfloat16)
    keep = inp["target"] != -100
    Q[keep.nonzero().flatten(), inp["target"][keep]] = 1.0
    kl_inp = dict(inp, Q=Q, target=None, shift_labels=inp["target"], eps=1e-10)
    kl = run_gpu(kl_inp)
    assert torch.equal(ce["loss"], kl["loss"])
    for k in ("dX", "dW", "db"):
        assert torch.equal(ce[k], kl[k]), k


def test_ce_module_autograd():
    w = small_case(dtype="bf16", BT=96, H=128, V=1000, bias=True, ce=True, ignore_frac=0.1)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    X = inp["X"].to(dev).requires_grad_(True)
    W = inp["W"].to(dev).requires_grad_(True)
    b = inp["b"].to(dev).requires_grad_(True)
    y = inp["target"].to(dev)
    loss = pkg.FusedLinearCrossEntropyLoss(accum_dtype=torch.float32)(W, X, y, bias=b)
    loss.backward()
    ref = run_oracle(inp)
    assert abs(float(loss.detach().cpu()) - ref["loss"]) <= 2e-2 * abs(ref["loss"])
    gx = X.grad.float().cpu().numpy()
    assert np.abs(gx - ref["dX"]).max() <= 2e-2 * np.abs(ref["dX"]).max()


def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    return sorted(set(int(x) for x in rng.choice(n, size=min(k, n), replace=False)) | {0, n - 1})


@pytest.mark.parametrize("name", list(CE_WORKLOADS))
def test_full_size_ce_workload(name):
    w = CE_WORKLOADS[name]
    inp = make_inputs(w)
    got = run_gpu(inp)
    dx_rows = _sample(w.BT, 24, 3)
    dw_rows = _sample(w.V, 24, 4) if w.compute_dW else None
    ref = run_oracle(inp, dX_rows=dx_rows, dW_rows=dw_rows)
    assert_close(w.dtype, got, ref, dX_rows=dx_rows, dW_rows=dw_rows)
