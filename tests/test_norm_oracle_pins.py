"""Pins of the norm-backward oracle: torch fp64 autograd of the forward
definitions (a library special case), finite differences, and the frozen
flags leaving dx unchanged (LoRA normalization page, *Test Validation*)."""

import numpy as np
import pytest
import torch

from oracle.norm_oracle import layer_norm_backward, rms_norm_backward


def _case(seed, N=6, H=10):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, H)), rng.standard_normal((N, H)) * 2.0 + 0.3,
            rng.standard_normal(H), rng.standard_normal(H))


def test_rms_norm_backward_matches_torch_autograd():
    dy, x, w, _ = _case(1)
    eps = 1e-6
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    y = wt * xt / torch.sqrt((xt * xt).mean(dim=1, keepdim=True) + eps)
    y.backward(torch.tensor(dy))
    dx, dW = rms_norm_backward(dy, x, w, eps)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dW, wt.grad.numpy(), rtol=1e-12, atol=1e-14)
    # torch's own rms_norm, a second library reference
    xt2 = torch.tensor(x, requires_grad=True)
    wt2 = torch.tensor(w, requires_grad=True)
    torch.nn.functional.rms_norm(xt2, (x.shape[1],), wt2, eps).backward(torch.tensor(dy))
    np.testing.assert_allclose(dx, xt2.grad.numpy(), rtol=1e-12, atol=1e-14)


def test_layer_norm_backward_matches_torch_layer_norm():
    dy, x, w, b = _case(2)
    eps = 1e-5
    xt = torch.tensor(x, requires_grad=True)
    wt = torch.tensor(w, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    torch.nn.functional.layer_norm(xt, (x.shape[1],), wt, bt, eps).backward(torch.tensor(dy))
    dx, dW, db = layer_norm_backward(dy, x, w, eps)
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(dW, wt.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("norm", ["rms", "layer"])
def test_finite_differences(norm):
    dy, x, w, b = _case(3, N=3, H=5)
    h = 1e-6

    def loss(x_, w_):
        if norm == "rms":
            y = w_ * x_ / np.sqrt((x_ * x_).mean(axis=1, keepdims=True) + 1e-6)
        else:
            c = x_ - x_.mean(axis=1, keepdims=True)
            y = w_ * c / np.sqrt((c * c).mean(axis=1, keepdims=True) + 1e-5) + b
        return float((dy * y).sum())

    if norm == "rms":
        dx, dW = rms_norm_backward(dy, x, w, 1e-6)
    else:
        dx, dW, _ = layer_norm_backward(dy, x, w, 1e-5)
    for arr, grad, is_x in ((x, dx, True), (w, dW, False)):
        num = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            p = arr.copy(); p[i] += h
            m = arr.copy(); m[i] -= h
            num[i] = ((loss(p, w) - loss(m, w)) if is_x else (loss(x, p) - loss(x, m))) / (2 * h)
        assert np.abs(num - grad).max() <= 1e-6 * np.abs(grad).max()


def test_frozen_flags_leave_dx_unchanged():
    dy, x, w, _ = _case(4)
    a = rms_norm_backward(dy, x, w, compute_dW=True)
    f = rms_norm_backward(dy, x, w, compute_dW=False)
    assert f[1] is None and np.array_equal(a[0], f[0])
    a = layer_norm_backward(dy, x, w, compute_dW=True, compute_db=True)
    f = layer_norm_backward(dy, x, w, compute_dW=False, compute_db=False)
    assert f[1] is None and f[2] is None and np.array_equal(a[0], f[0])
