"""Fused linear JSD on the GPU against the fp64 oracle (generalized JSD,
student gradients only), through the C ABI and the module."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from lm_head_projection_b200.workloads import make_inputs, small_case
from oracle import jsd_forward_backward as oracle_jsd
from parity_utils import TOL, to_np

pytestmark = pytest.mark.gpu


def _teacher(w, Ht, seed):
    """Teacher hidden states and head of the same workload recipe."""
    t = make_inputs(small_case(dtype=w.dtype, BT=w.BT, H=Ht, V=w.V, bias=w.bias,
                               seed=seed + 1000, w_std=w.w_std * 1.3))
    return t["X"], t["W"], t["b"]


def _run(dtype, BT, H, Ht, V, bias, T, beta, reduction, ignore, seed, cw=True):
    import lm_head_projection_b200 as pkg

    w = small_case(dtype=dtype, BT=BT, H=H, V=V, bias=bias, reduction=reduction,
                   ignore_frac=ignore, temperature=T, seed=seed)
    inp = make_inputs(w)
    Xt, Wt, bt = _teacher(w, Ht, seed)
    dev = torch.device("cuda:0")
    g = lambda t: None if t is None else t.to(dev)
    r = pkg.jsd_forward_backward(g(inp["X"]), g(inp["W"]), g(inp["b"]), g(Xt), g(Wt), g(bt),
                                 g(inp["shift_labels"]), -100, T, beta, reduction,
                                 compute_dW=cw, compute_db=bias, check_status=True)
    torch.cuda.synchronize()
    lab = inp["shift_labels"]
    ref = oracle_jsd(to_np(inp["X"]), to_np(inp["W"]), to_np(inp["b"]), to_np(Xt), to_np(Wt),
                     to_np(bt), None if lab is None else lab.numpy(), -100, T, beta, reduction,
                     compute_dW=cw, compute_db=bias)
    return r, ref


def _check(dtype, r, ref):
    tol = TOL[dtype]
    loss = float(r["loss"].cpu())
    # the loss is a divergence (>= 0, can be small): relative bound plus a floor
    assert abs(loss - ref["loss"]) <= tol["loss_rel"] * abs(ref["loss"]) + (
        1e-6 if dtype == "fp32" else 1e-4), (loss, ref["loss"])
    for k in ("dX", "dW", "db"):
        if ref[k] is None:
            assert r[k] is None
            continue
        a, e = to_np(r[k]), ref[k]
        err = float(np.abs(a - e).max())
        assert err <= tol["grad_abs"] + tol["grad_rel_scale"] * float(np.abs(e).max()) + 1e-30, (
            k, err)


CASES = [
    ("fp32", 64, 256, 128, 1024, True, 1.0, 0.5, "batchmean", 0.0),
    ("fp32", 37, 64, 96, 200, False, 1.7, 0.3, "sum", 0.2),
    ("bf16", 300, 256, 192, 3000, True, 1.0, 0.5, "batchmean", 0.1),
    ("bf16", 129, 128, 256, 1000, False, 2.0, 0.8, "mean", 0.0),
    ("bf16", 8, 4096, 1024, 4104, True, 1.0, 0.5, "sum", 0.0),
]


@pytest.mark.parametrize("dtype,BT,H,Ht,V,bias,T,beta,reduction,ignore", CASES)
def test_small_cases(dtype, BT, H, Ht, V, bias, T, beta, reduction, ignore):
    r, ref = _run(dtype, BT, H, Ht, V, bias, T, beta, reduction, ignore, seed=BT + V)
    _check(dtype, r, ref)


def test_frozen_head_leaves_dx_and_loss_bitwise_unchanged():
    a, _ = _run("bf16", 200, 128, 128, 2000, False, 1.0, 0.5, "batchmean", 0.1, seed=3)
    b, _ = _run("bf16", 200, 128, 128, 2000, False, 1.0, 0.5, "batchmean", 0.1, seed=3,
                cw=False)
    assert b["dW"] is None
    assert torch.equal(a["dX"], b["dX"]) and torch.equal(a["loss"], b["loss"])


def test_teacher_equal_to_student_gives_zero():
    import lm_head_projection_b200 as pkg

    w = small_case(dtype="bf16", BT=96, H=128, V=1000, bias=True, seed=4)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    X, W, b = (inp[k].to(dev) for k in ("X", "W", "b"))
    r = pkg.jsd_forward_backward(X, W, b, X, W, b, compute_dW=True, compute_db=True)
    torch.cuda.synchronize()
    assert abs(float(r["loss"])) < 1e-6
    for k in ("dX", "dW", "db"):
        assert float(r[k].abs().max()) < 1e-6, k


def test_headline_head_shape_sampled_rows():
    import lm_head_projection_b200 as pkg

    w = small_case(dtype="bf16", BT=256, H=4096, V=128256, bias=False, seed=5, w_std=0.02)
    inp = make_inputs(w)
    Xt, Wt, _ = _teacher(w, 2048, 5)
    dev = torch.device("cuda:0")
    r = pkg.jsd_forward_backward(inp["X"].to(dev), inp["W"].to(dev), None, Xt.to(dev),
                                 Wt.to(dev), None, compute_dW=True, check_status=True)
    torch.cuda.synchronize()
    rows = np.linspace(0, w.BT - 1, 12).astype(np.int64)
    vrows = np.linspace(0, w.V - 1, 12).astype(np.int64)
    ref = oracle_jsd(to_np(inp["X"]), to_np(inp["W"]), None, to_np(Xt), to_np(Wt), None,
                     compute_dW=True, dX_rows=rows, dW_rows=vrows)
    got = {"loss": r["loss"], "dX": r["dX"][torch.as_tensor(rows, device=dev)],
           "dW": r["dW"][torch.as_tensor(vrows, device=dev)], "db": None}
    _check("bf16", got, {**ref, "db": None})


def test_module_autograd_student_only():
    from lm_head_projection_b200 import FusedLinearJSDLoss

    w = small_case(dtype="fp32", BT=48, H=64, V=500, bias=True, seed=6)
    inp = make_inputs(w)
    Xt, Wt, bt = _teacher(w, 32, 6)
    dev = torch.device("cuda:0")
    X = inp["X"].to(dev).requires_grad_(True)
    W = inp["W"].to(dev).requires_grad_(True)
    b = inp["b"].to(dev).requires_grad_(True)
    Wt_ = Wt.to(dev).requires_grad_(True)
    loss = FusedLinearJSDLoss(beta=0.4)(W, X, Xt.to(dev), Wt_, student_bias=b,
                                         teacher_bias=bt.to(dev))
    (2.0 * loss).backward()
    assert Wt_.grad is None
    ref = oracle_jsd(to_np(inp["X"]), to_np(inp["W"]), to_np(inp["b"]), to_np(Xt), to_np(Wt),
                     to_np(bt), None, -100, 1.0, 0.4, "batchmean", compute_dW=True,
                     compute_db=True)
    for k, g in (("dX", X.grad), ("dW", W.grad), ("db", b.grad)):
        assert float(np.abs(to_np(g) - 2.0 * ref[k]).max()) <= 2e-5, k
