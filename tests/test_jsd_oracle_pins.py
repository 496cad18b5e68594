"""Pins of the fused linear JSD oracle (generalized Jensen-Shannon
divergence, the reading stated in the oracle): identical distributions give
0, disjoint supports give the binary entropy of beta, the bound 0 <= l <=
H(beta), the student/teacher swap with beta -> 1 - beta, the small-beta
limit KL(P || Q) (scipy rel_entr), finite differences and torch fp64
autograd of the gradient, reductions and dropped rows.  CPU only."""

from __future__ import annotations

import numpy as np
import pytest
import torch
from scipy.special import rel_entr

from oracle import jsd_forward_backward


def _case(BT=6, H=4, V=9, Ht=5, seed=0):
    g = np.random.default_rng(seed)
    X, W, b = g.normal(size=(BT, H)), g.normal(size=(V, H)), g.normal(size=V) * 0.3
    Xt, Wt, bt = g.normal(size=(BT, Ht)), g.normal(size=(V, Ht)), g.normal(size=V) * 0.3
    lab = g.integers(0, V, size=BT)
    lab[2] = -100
    return X, W, b, Xt, Wt, bt, lab


def _H(beta):
    return -beta * np.log(beta) - (1 - beta) * np.log(1 - beta)


def test_identical_student_and_teacher_give_zero():
    X, W, b, _, _, _, lab = _case()
    r = jsd_forward_backward(X, W, b, X, W, b, lab, compute_dW=True, compute_db=True)
    assert abs(r["loss"]) < 1e-15
    for k in ("dX", "dW", "db"):
        assert np.abs(r[k]).max() < 1e-15


@pytest.mark.parametrize("beta", [0.5, 0.2, 0.9])
def test_disjoint_supports_give_the_binary_entropy(beta):
    # student mass on column 0, teacher mass on column 1 (one row, V = 3)
    X = np.array([[1.0]])
    W = np.array([[60.0], [0.0], [0.0]])
    Xt = np.array([[1.0]])
    Wt = np.array([[0.0], [60.0], [0.0]])
    r = jsd_forward_backward(X, W, None, Xt, Wt, None, beta=beta, reduction="sum",
                             compute_dW=False)
    assert abs(r["loss"] - _H(beta)) < 1e-12


@pytest.mark.parametrize("beta", [0.5, 0.3])
def test_bounded_by_the_binary_entropy(beta):
    for seed in range(5):
        X, W, b, Xt, Wt, bt, _ = _case(seed=seed)
        r = jsd_forward_backward(X, W, b, Xt, Wt, bt, beta=beta, reduction="sum",
                                 compute_dW=False)
        assert np.all(r["row_loss"] >= -1e-15) and np.all(r["row_loss"] <= _H(beta) + 1e-15)


def test_swapping_roles_and_beta():
    X, W, b, Xt, Wt, bt, _ = _case(seed=4)
    a = jsd_forward_backward(X, W, b, Xt, Wt, bt, beta=0.3, reduction="sum", compute_dW=False)
    c = jsd_forward_backward(Xt, Wt, bt, X, W, b, beta=0.7, reduction="sum", compute_dW=False)
    assert abs(a["loss"] - c["loss"]) < 1e-13


def test_small_beta_limit_is_kl_p_q():
    X, W, b, Xt, Wt, bt, _ = _case(seed=6)
    beta = 1e-7
    r = jsd_forward_backward(X, W, b, Xt, Wt, bt, beta=beta, reduction="sum", compute_dW=False)
    zs, zt = X @ W.T + b, Xt @ Wt.T + bt
    p = np.exp(zs - zs.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    q = np.exp(zt - zt.max(1, keepdims=True))
    q /= q.sum(1, keepdims=True)
    kl = rel_entr(p, q).sum()
    assert abs(r["loss"] / beta - kl) < 1e-5 * max(1.0, kl)


@pytest.mark.parametrize("T,beta", [(1.0, 0.5), (1.7, 0.25)])
def test_gradient_matches_torch_autograd(T, beta):
    X, W, b, Xt, Wt, bt, lab = _case(seed=2)
    r = jsd_forward_backward(X, W, b, Xt, Wt, bt, lab, temperature=T, beta=beta,
                             reduction="batchmean", compute_dW=True, compute_db=True)
    Xg, Wg, bg = (torch.tensor(a, requires_grad=True) for a in (X, W, b))
    logp = torch.log_softmax((Xg @ Wg.T + bg) / T, dim=1)
    logq = torch.log_softmax(torch.tensor(Xt @ Wt.T + bt) / T, dim=1)
    p, q = logp.exp(), logq.exp()
    logm = torch.log(beta * p + (1 - beta) * q)
    rows = beta * (p * (logp - logm)).sum(1) + (1 - beta) * (q * (logq - logm)).sum(1)
    keep = torch.tensor(lab != -100)
    loss = rows[keep].sum() / keep.sum()
    loss.backward()
    assert abs(float(loss.detach()) - r["loss"]) < 1e-13
    np.testing.assert_allclose(r["dX"], Xg.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["dW"], Wg.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["db"], bg.grad.numpy(), rtol=0, atol=1e-12)


def test_finite_differences():
    X, W, b, Xt, Wt, bt, lab = _case(BT=4, H=3, V=5, seed=9)
    T, beta = 1.3, 0.4
    f = lambda X_, W_, b_: jsd_forward_backward(X_, W_, b_, Xt, Wt, bt, lab, temperature=T,
                                                beta=beta, reduction="mean",
                                                compute_dW=False)["loss"]
    r = jsd_forward_backward(X, W, b, Xt, Wt, bt, lab, temperature=T, beta=beta,
                             reduction="mean", compute_dW=True, compute_db=True)
    h = 1e-6
    for k, arr, grad in ((0, X, r["dX"]), (1, W, r["dW"]), (2, b, r["db"])):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += h
            a2[idx] -= h
            args1, args2 = [X, W, b], [X, W, b]
            args1[k], args2[k] = a1, a2
            num[idx] = (f(*args1) - f(*args2)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-9)


def test_reductions_and_dropped_rows():
    X, W, b, Xt, Wt, bt, lab = _case(seed=3)
    V = W.shape[0]
    s = jsd_forward_backward(X, W, b, Xt, Wt, bt, lab, reduction="sum", compute_dW=True)
    bm = jsd_forward_backward(X, W, b, Xt, Wt, bt, lab, reduction="batchmean", compute_dW=True)
    mn = jsd_forward_backward(X, W, b, Xt, Wt, bt, lab, reduction="mean", compute_dW=True)
    n = int((lab != -100).sum())
    assert abs(s["loss"] - n * bm["loss"]) < 1e-12
    assert abs(s["loss"] - n * V * mn["loss"]) < 1e-12
    np.testing.assert_allclose(s["dW"], n * bm["dW"], rtol=1e-12, atol=1e-14)
    assert np.all(s["dX"][2] == 0.0)
    keep = lab != -100
    sub = jsd_forward_backward(X[keep], W, b, Xt[keep], Wt, bt, None, reduction="sum",
                               compute_dW=True)
    assert abs(sub["loss"] - s["loss"]) < 1e-12
    np.testing.assert_allclose(sub["dW"], s["dW"], rtol=0, atol=1e-12)


def test_temperature_scales_both_sides():
    X, W, b, Xt, Wt, bt, lab = _case(seed=12)
    T = 2.3
    a = jsd_forward_backward(X, W, b, Xt, Wt, bt, lab, temperature=T, reduction="sum",
                             compute_dW=False)
    c = jsd_forward_backward(X / T, W, b / T, Xt / T, Wt, bt / T, lab, temperature=1.0,
                             reduction="sum", compute_dW=False)
    assert abs(a["loss"] - c["loss"]) < 1e-13
    np.testing.assert_allclose(a["dX"], c["dX"] / T, rtol=0, atol=1e-13)
