"""Pins of the selective log-probability oracle (GRPO frozen-head page,
*Summary*): torch fp64 log_softmax / gather and autograd, central finite
differences, the cross-entropy special case, a closed form and an
invariant.  CPU only."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import ce_forward_backward, selective_logprob, selective_logprob_backward


def _case(BT=7, H=5, V=11, seed=0, bias=True):
    g = np.random.default_rng(seed)
    X = g.normal(size=(BT, H))
    W = g.normal(size=(V, H)) * 0.7
    b = g.normal(size=V) * 0.3 if bias else None
    tgt = g.integers(0, V, size=BT)
    tgt[1] = -100          # dropped
    tgt[4] = V + 3         # outside [0, V): no log-probability
    dl = g.normal(size=BT)
    return X, W, b, tgt, dl


def _torch_logp(X, W, b, tgt, T):
    Xt, Wt = torch.tensor(X), torch.tensor(W)
    bt = None if b is None else torch.tensor(b)
    z = torch.nn.functional.linear(Xt, Wt, bt) / T
    lp = torch.log_softmax(z, dim=1)
    y = torch.tensor(tgt)
    inside = (y != -100) & (y >= 0) & (y < W.shape[0])
    picked = lp.gather(1, y.clamp(0, W.shape[0] - 1)[:, None])[:, 0]
    return torch.where(inside, picked, torch.zeros_like(picked))


@pytest.mark.parametrize("T", [1.0, 0.7, 2.5])
def test_logp_matches_torch_log_softmax(T):
    X, W, b, tgt, _ = _case()
    got = selective_logprob(X, W, b, tgt, -100, T)
    ref = _torch_logp(X, W, b, tgt, T).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-13)
    assert got[1] == 0.0 and got[4] == 0.0


@pytest.mark.parametrize("T", [1.0, 1.7])
def test_backward_matches_torch_autograd(T):
    X, W, b, tgt, dl = _case(seed=3)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    z = torch.nn.functional.linear(Xt, Wt, bt) / T
    lp = torch.log_softmax(z, dim=1)
    y = torch.tensor(tgt)
    inside = (y != -100) & (y >= 0) & (y < W.shape[0])
    picked = lp.gather(1, y.clamp(0, W.shape[0] - 1)[:, None])[:, 0]
    (torch.where(inside, picked, torch.zeros_like(picked)) * torch.tensor(dl)).sum().backward()
    r = selective_logprob_backward(X, W, b, tgt, dl, -100, T, compute_dW=True, compute_db=True)
    np.testing.assert_allclose(r["dX"], Xt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["dW"], Wt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["db"], bt.grad.numpy(), rtol=0, atol=1e-12)


def test_finite_differences():
    X, W, b, tgt, dl = _case(BT=6, H=3, V=6, seed=5)
    T = 1.3
    f = lambda X_, W_, b_: float(np.dot(dl, selective_logprob(X_, W_, b_, tgt, -100, T)))
    r = selective_logprob_backward(X, W, b, tgt, dl, -100, T, compute_dW=True, compute_db=True)
    h = 1e-6
    for name, arr, grad in (("X", X, r["dX"]), ("W", W, r["dW"]), ("b", b, r["db"])):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += h
            a2[idx] -= h
            args1 = [X, W, b]
            args2 = [X, W, b]
            k = {"X": 0, "W": 1, "b": 2}[name]
            args1[k], args2[k] = a1, a2
            num[idx] = (f(*args1) - f(*args2)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_cross_entropy_is_the_mean_negative_logp():
    X, W, b, tgt, _ = _case(seed=8)
    tgt[4] = 2  # keep every non-dropped target in range for this identity
    T = 1.4
    kept = tgt != -100
    n = int(kept.sum())
    lp = selective_logprob(X, W, b, tgt, -100, T)
    ce = ce_forward_backward(X, W, b, tgt, -100, T, "batchmean", compute_dW=True,
                             compute_db=True)
    assert abs(-lp.sum() / n - ce["loss"]) < 1e-13
    r = selective_logprob_backward(X, W, b, tgt, np.where(kept, -1.0 / n, 0.0), -100, T,
                                   compute_dW=True, compute_db=True)
    for k in ("dX", "dW", "db"):
        np.testing.assert_allclose(r[k], ce[k], rtol=0, atol=1e-13, err_msg=k)


def test_zero_head_closed_form_and_zero_column_sums():
    X, W, b, tgt, dl = _case(seed=2)
    V = W.shape[0]
    T = 0.9
    Wz = np.zeros_like(W)
    lp = selective_logprob(X, Wz, None, tgt, -100, T)
    inside = (tgt != -100) & (tgt >= 0) & (tgt < V)
    np.testing.assert_allclose(lp, np.where(inside, -np.log(V), 0.0), rtol=0, atol=1e-14)
    r = selective_logprob_backward(X, Wz, np.zeros(V), tgt, dl, -100, T, compute_dW=False,
                                   compute_db=True)
    # dz_rv = dlogp_r ([v == y_r] - 1/V) / T on kept rows
    dz = -np.ones((len(tgt), V)) / V
    for r_, y in enumerate(tgt):
        if inside[r_]:
            dz[r_, y] += 1.0
    dz *= (np.where(inside, dl, 0.0) / T)[:, None]
    np.testing.assert_allclose(r["db"], dz.sum(axis=0), rtol=0, atol=1e-14)
    r2 = selective_logprob_backward(X, W, b, tgt, dl, -100, T, compute_dW=False,
                                    compute_db=True)
    assert abs(r2["db"].sum()) < 1e-12
