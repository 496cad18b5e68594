"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test names what fixes the expected value: a hand-derived worked example,
a library special case (torch cross_entropy / kl_div in fp64 with autograd), a
closed form, an invariant of the mathematics, finite differences, or a
pure-Python loop version on tiny inputs.  A plausible slip in the oracle (a
dropped S_r factor, a missing 1/T, the wrong divisor, log q instead of
log max(q, eps), ignored rows leaking into dX) fails at least one of them.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import OracleError, forward_backward, forward_backward_loops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, BT=4, H=5, V=7, bias=True, q_std=1.0):
    X = rng.standard_normal((BT, H))
    W = rng.standard_normal((V, H)) * 0.7
    b = rng.standard_normal(V) * 0.3 if bias else None
    t = rng.standard_normal((BT, V)) * q_std
    Q = np.exp(t - t.max(1, keepdims=True))
    Q /= Q.sum(1, keepdims=True)
    return X, W, b, Q


def _golden():
    vals = {}
    with open(os.path.join(GOLDEN, "two_logit_worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            ex, name, val = line.split()
            vals[(ex, name)] = float(val)
    return vals


# ---------------------------------------------------------------- worked examples

def test_worked_example_two_logits():
    g = _golden()
    X = np.array([[1.0]])
    W = np.array([[1.0], [-1.0]])
    Q = np.array([[0.5, 0.5]])
    r = forward_backward(X, W, None, Q, reduction="batchmean")
    assert r["loss"] == pytest.approx(g[("A", "loss")], abs=1e-15)
    assert r["dX"][0, 0] == pytest.approx(g[("A", "dX")], abs=1e-15)
    assert r["dW"][0, 0] == pytest.approx(g[("A", "dW0")], abs=1e-15)
    assert r["dW"][1, 0] == pytest.approx(g[("A", "dW1")], abs=1e-15)


def test_worked_example_ignore_temperature_sum():
    g = _golden()
    X = np.array([[2.0], [5.0]])
    W = np.array([[1.0], [-1.0]])
    Q = np.array([[0.5, 0.5], [0.9, 0.1]])
    r = forward_backward(X, W, None, Q, shift_labels=np.array([0, -100]), ignore_index=-100,
                         temperature=2.0, reduction="sum")
    assert r["loss"] == pytest.approx(g[("B", "loss")], abs=1e-15)
    assert r["dX"][0, 0] == pytest.approx(g[("B", "dX0")], abs=1e-15)
    assert r["dX"][1, 0] == g[("B", "dX1")]
    assert r["dW"][0, 0] == pytest.approx(g[("B", "dW0")], abs=1e-15)
    assert r["dW"][1, 0] == pytest.approx(g[("B", "dW1")], abs=1e-15)


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("reduction", ["batchmean", "mean", "sum"])
@pytest.mark.parametrize("T", [0.5, 1.0, 2.0])
def test_matches_python_loops(reduction, T):
    rng = np.random.default_rng(1)
    X, W, b, Q = _rand_case(rng, BT=5, H=3, V=6)
    Q[1, 2] = 0.0
    Q[3, 0] = 1e-13
    labels = np.array([3, -100, 1, 2, -100])
    kw = dict(shift_labels=labels, ignore_index=-100, temperature=T, eps=1e-10,
              reduction=reduction, compute_dW=True, compute_db=True)
    a = forward_backward(X, W, b, Q, row_block=2, **kw)
    c = forward_backward_loops(X, W, b, Q, **kw)
    assert a["loss"] == pytest.approx(c["loss"], rel=1e-13, abs=1e-15)
    for k in ("dX", "dW", "db"):
        np.testing.assert_allclose(a[k], c[k], rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------- special cases

def test_teacher_equals_student_gives_zero():
    rng = np.random.default_rng(2)
    X, W, b, _ = _rand_case(rng, BT=6, H=8, V=11)
    T = 1.3
    u = (X @ W.T + b) / T
    Q = np.exp(u - u.max(1, keepdims=True))
    Q /= Q.sum(1, keepdims=True)
    r = forward_backward(X, W, b, Q, temperature=T, compute_db=True)
    assert abs(r["loss"]) < 1e-14
    assert np.abs(r["dX"]).max() < 1e-15
    assert np.abs(r["dW"]).max() < 1e-15
    assert np.abs(r["db"]).max() < 1e-15


@pytest.mark.parametrize("reduction", ["batchmean", "sum"])
def test_one_hot_teacher_is_cross_entropy(reduction):
    """With a one-hot teacher the sum q log q vanishes and KL is the
    cross-entropy of the student at the label; checked against torch's
    cross_entropy and its autograd in fp64."""
    rng = np.random.default_rng(3)
    X, W, b, _ = _rand_case(rng, BT=6, H=5, V=9)
    y = rng.integers(0, 9, size=6)
    Q = np.zeros((6, 9))
    Q[np.arange(6), y] = 1.0
    T = 0.7
    r = forward_backward(X, W, b, Q, temperature=T, reduction=reduction, compute_db=True)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    ce = F.cross_entropy(F.linear(Xt, Wt, bt) / T, torch.tensor(y),
                         reduction="mean" if reduction == "batchmean" else "sum")
    ce.backward()
    assert r["loss"] == pytest.approx(ce.item(), rel=1e-13)
    np.testing.assert_allclose(r["dX"], Xt.grad.numpy(), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(r["dW"], Wt.grad.numpy(), rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(r["db"], bt.grad.numpy(), rtol=1e-11, atol=1e-15)


# torch notes that its "mean" divides by batch x support; that is the
# reduction pinned here, so its deprecation notice is expected
@pytest.mark.filterwarnings("ignore:reduction.*mean.*divides:UserWarning")
@pytest.mark.parametrize("reduction", ["batchmean", "mean", "sum"])
def test_matches_torch_kl_div(reduction):
    """torch.nn.functional.kl_div on log_softmax(linear/T) with autograd, fp64.
    torch's reductions divide by BT (batchmean) and BT*V (mean); with no
    ignored rows these are the oracle's divisors."""
    rng = np.random.default_rng(4)
    X, W, b, Q = _rand_case(rng, BT=7, H=6, V=13, q_std=2.0)
    T = 1.9
    r = forward_backward(X, W, b, Q, temperature=T, reduction=reduction, compute_db=True)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    logp = F.log_softmax(F.linear(Xt, Wt, bt) / T, dim=-1)
    kl = F.kl_div(logp, torch.tensor(Q), reduction=reduction)
    kl.backward()
    assert r["loss"] == pytest.approx(kl.item(), rel=1e-12)
    np.testing.assert_allclose(r["dX"], Xt.grad.numpy(), rtol=1e-10, atol=1e-16)
    np.testing.assert_allclose(r["dW"], Wt.grad.numpy(), rtol=1e-10, atol=1e-16)
    np.testing.assert_allclose(r["db"], bt.grad.numpy(), rtol=1e-10, atol=1e-16)


def test_closed_form_zero_head():
    """W = 0, b = 0: the student is uniform, p = 1/V, so
    row loss = sum q log max(q,eps) + S log V and G = (S/V - q)/(T D)."""
    rng = np.random.default_rng(5)
    BT, H, V = 5, 4, 10
    X = rng.standard_normal((BT, H))
    W = np.zeros((V, H))
    b = np.zeros(V)
    Q = rng.random((BT, V))
    Q /= Q.sum(1, keepdims=True)
    Q[0, 3] = 0.0
    T = 3.0
    r = forward_backward(X, W, b, Q, temperature=T, reduction="batchmean", compute_db=True)
    S = Q.sum(1)
    with np.errstate(divide="ignore"):
        qlogq = np.where(Q > 0, Q * np.log(np.where(Q > 0, Q, 1.0)), 0.0).sum(1)
    expect = (qlogq + S * math.log(V)).sum() / BT
    assert r["loss"] == pytest.approx(expect, rel=1e-13)
    G = (S[:, None] / V - Q) / (T * BT)
    np.testing.assert_allclose(r["db"], G.sum(0), atol=1e-16)
    np.testing.assert_allclose(r["dW"], G.T @ X, atol=1e-15)
    np.testing.assert_allclose(r["dX"], 0.0, atol=0)


def test_eps_clamp_and_zero_entries():
    """An entry 0 < q < eps contributes q (log eps - log p) to the row loss;
    an entry q == 0 contributes nothing, also with eps = 0."""
    rng = np.random.default_rng(6)
    X, W, b, Q = _rand_case(rng, BT=3, H=4, V=8)
    Q[1, 5] = 0.0
    base = forward_backward(X, W, b, Q, eps=1e-10, reduction="sum", compute_dW=False)
    Q2 = Q.copy()
    Q2[1, 5] = 1e-13
    moved = forward_backward(X, W, b, Q2, eps=1e-10, reduction="sum", compute_dW=False)
    logp = base["lse"][1]  # lse of row 1
    u = (X[1] @ W.T + b)
    log_p5 = u[5] - logp
    assert moved["loss"] - base["loss"] == pytest.approx(1e-13 * (math.log(1e-10) - log_p5),
                                                         rel=1e-6)
    # eps = 0 with an exact zero: finite, and equal to the eps = 1e-10 result
    z0 = forward_backward(X, W, b, Q, eps=0.0, reduction="sum", compute_dW=False)
    assert np.isfinite(z0["loss"])
    assert z0["loss"] == base["loss"]


# ---------------------------------------------------------------- invariants

def test_gradient_rows_sum_to_zero_and_db_sums_to_zero():
    rng = np.random.default_rng(7)
    X, W, b, Q = _rand_case(rng, BT=9, H=6, V=15)
    r = forward_backward(X, W, b, Q, compute_db=True, temperature=0.8)
    assert abs(r["db"].sum()) < 1e-15
    # sum over v of dW[v, :] = (sum_v G[:, v])^T X = 0
    assert np.abs(r["dW"].sum(0)).max() < 1e-14


def test_bias_shift_invariance():
    rng = np.random.default_rng(8)
    X, W, b, Q = _rand_case(rng, BT=4, H=5, V=9)
    a = forward_backward(X, W, b, Q, temperature=1.5, compute_db=True)
    c = forward_backward(X, W, b + 3.25, Q, temperature=1.5, compute_db=True)
    assert a["loss"] == pytest.approx(c["loss"], rel=1e-12)
    for k in ("dX", "dW", "db"):
        np.testing.assert_allclose(a[k], c[k], rtol=1e-9, atol=1e-15)


def test_temperature_scaling():
    """loss(X, W, b, T) = loss(X/T, W, b/T, 1); dW is the same, dX and db
    scale by 1/T."""
    rng = np.random.default_rng(9)
    X, W, b, Q = _rand_case(rng, BT=4, H=5, V=9)
    T = 2.5
    a = forward_backward(X, W, b, Q, temperature=T, compute_db=True)
    c = forward_backward(X / T, W, b / T, Q, temperature=1.0, compute_db=True)
    assert a["loss"] == pytest.approx(c["loss"], rel=1e-12)
    np.testing.assert_allclose(a["dW"], c["dW"], rtol=1e-11, atol=1e-16)
    np.testing.assert_allclose(a["dX"], c["dX"] / T, rtol=1e-11, atol=1e-16)
    np.testing.assert_allclose(a["db"], c["db"] / T, rtol=1e-11, atol=1e-16)


def test_reduction_divisors():
    rng = np.random.default_rng(10)
    X, W, b, Q = _rand_case(rng, BT=6, H=4, V=7)
    labels = np.array([0, -100, 2, 3, -100, 1])
    kw = dict(shift_labels=labels, ignore_index=-100, compute_db=True)
    s = forward_backward(X, W, b, Q, reduction="sum", **kw)
    bm = forward_backward(X, W, b, Q, reduction="batchmean", **kw)
    mn = forward_backward(X, W, b, Q, reduction="mean", **kw)
    assert s["loss"] == pytest.approx(4 * bm["loss"], rel=1e-13)
    assert s["loss"] == pytest.approx(4 * 7 * mn["loss"], rel=1e-13)
    for k in ("dX", "dW", "db"):
        np.testing.assert_allclose(s[k], 4 * bm[k], rtol=1e-12, atol=1e-16)
        np.testing.assert_allclose(s[k], 28 * mn[k], rtol=1e-12, atol=1e-16)


def test_ignored_rows_drop_out():
    rng = np.random.default_rng(11)
    X, W, b, Q = _rand_case(rng, BT=6, H=4, V=7)
    labels = np.array([0, -100, 2, 3, -100, 1])
    keep = labels != -100
    r = forward_backward(X, W, b, Q, shift_labels=labels, ignore_index=-100, compute_db=True)
    assert np.all(r["dX"][~keep] == 0.0)
    k = forward_backward(X[keep], W, b, Q[keep], compute_db=True)
    assert r["loss"] == pytest.approx(k["loss"], rel=1e-13)
    np.testing.assert_allclose(r["dX"][keep], k["dX"], rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(r["dW"], k["dW"], rtol=1e-12, atol=1e-16)
    np.testing.assert_allclose(r["db"], k["db"], rtol=1e-12, atol=1e-16)
    # a label equal to another value than ignore_index keeps the row
    r2 = forward_backward(X, W, b, Q, shift_labels=labels, ignore_index=-7, compute_db=True)
    a = forward_backward(X, W, b, Q, compute_db=True)
    assert r2["loss"] == a["loss"]


def test_all_rows_ignored_gives_zeros():
    rng = np.random.default_rng(12)
    X, W, b, Q = _rand_case(rng, BT=3, H=4, V=5)
    r = forward_backward(X, W, b, Q, shift_labels=np.full(3, -100), compute_db=True)
    assert r["loss"] == 0.0
    assert not np.any(r["dX"]) and not np.any(r["dW"]) and not np.any(r["db"])


def test_frozen_head_leaves_loss_and_dX():
    rng = np.random.default_rng(13)
    X, W, b, Q = _rand_case(rng, BT=5, H=4, V=6)
    a = forward_backward(X, W, b, Q, compute_dW=True, compute_db=True)
    c = forward_backward(X, W, b, Q, compute_dW=False, compute_db=False)
    assert c["dW"] is None and c["db"] is None
    assert a["loss"] == c["loss"]
    assert np.array_equal(a["dX"], c["dX"])


def test_reduction_none_refused():
    rng = np.random.default_rng(14)
    X, W, b, Q = _rand_case(rng)
    with pytest.raises(OracleError):
        forward_backward(X, W, b, Q, reduction="none")


def test_sampled_rows_match_full():
    rng = np.random.default_rng(15)
    X, W, b, Q = _rand_case(rng, BT=10, H=4, V=9)
    full = forward_backward(X, W, b, Q, compute_db=True, row_block=3)
    part = forward_backward(X, W, b, Q, compute_db=True, dX_rows=[7, 2], dW_rows=[0, 8, 4],
                            row_block=4)
    np.testing.assert_allclose(part["dX"], full["dX"][[7, 2]], rtol=1e-13, atol=1e-16)
    np.testing.assert_allclose(part["dW"], full["dW"][[0, 8, 4]], rtol=1e-13, atol=1e-16)
    assert part["loss"] == pytest.approx(full["loss"], rel=1e-14)


# ---------------------------------------------------------------- finite differences

@pytest.mark.parametrize("reduction", ["batchmean", "mean", "sum"])
def test_finite_differences(reduction):
    rng = np.random.default_rng(16)
    X, W, b, Q = _rand_case(rng, BT=3, H=4, V=6, q_std=1.5)
    labels = np.array([1, -100, 4])
    T = 1.7
    kw = dict(shift_labels=labels, ignore_index=-100, temperature=T, reduction=reduction)
    r = forward_backward(X, W, b, Q, compute_db=True, **kw)

    def loss(X_, W_, b_):
        return forward_backward(X_, W_, b_, Q, compute_dW=False, **kw)["loss"]

    h = 1e-5
    for name, arr, grad in (("X", X, r["dX"]), ("W", W, r["dW"]), ("b", b, r["db"])):
        num = np.zeros_like(arr)
        it = np.nditer(arr, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            p = arr.copy(); p[i] += h
            m = arr.copy(); m[i] -= h
            args_p = {"X": X, "W": W, "b": b}
            args_m = {"X": X, "W": W, "b": b}
            args_p[name] = p
            args_m[name] = m
            num[i] = (loss(args_p["X"], args_p["W"], args_p["b"])
                      - loss(args_m["X"], args_m["W"], args_m["b"])) / (2 * h)
        scale = np.abs(grad).max()
        assert np.abs(num - grad).max() <= 1e-7 * scale + 1e-12, name


# ---------------------------------------------------------------- cross-entropy oracle

@pytest.mark.parametrize("reduction", ["batchmean", "sum"])
@pytest.mark.parametrize("T", [1.0, 1.7])
def test_ce_oracle_matches_torch_cross_entropy(reduction, T):
    """torch's cross_entropy with ignore_index (fp64, autograd): its 'mean'
    divides by the kept rows, which is batchmean here."""
    from oracle import ce_forward_backward
    rng = np.random.default_rng(20)
    X, W, b, _ = _rand_case(rng, BT=8, H=5, V=11)
    y = rng.integers(0, 11, size=8)
    y[[2, 5]] = -100
    r = ce_forward_backward(X, W, b, y, ignore_index=-100, temperature=T, reduction=reduction,
                            compute_db=True)
    Xt = torch.tensor(X, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    ce = F.cross_entropy(F.linear(Xt, Wt, bt) / T, torch.tensor(y), ignore_index=-100,
                         reduction="mean" if reduction == "batchmean" else "sum")
    ce.backward()
    assert r["loss"] == pytest.approx(ce.item(), rel=1e-13)
    np.testing.assert_allclose(r["dX"], Xt.grad.numpy(), rtol=1e-11, atol=1e-16)
    np.testing.assert_allclose(r["dW"], Wt.grad.numpy(), rtol=1e-11, atol=1e-16)
    np.testing.assert_allclose(r["db"], bt.grad.numpy(), rtol=1e-11, atol=1e-16)


@pytest.mark.parametrize("reduction", ["batchmean", "mean", "sum"])
def test_ce_oracle_is_kl_with_one_hot_teacher(reduction):
    from oracle import ce_forward_backward
    rng = np.random.default_rng(21)
    X, W, b, _ = _rand_case(rng, BT=7, H=4, V=9)
    y = rng.integers(0, 9, size=7)
    y[3] = -100
    Q = np.zeros((7, 9))
    Q[np.arange(7)[y >= 0], y[y >= 0]] = 1.0
    a = ce_forward_backward(X, W, b, y, temperature=0.6, reduction=reduction, compute_db=True,
                            row_block=3)
    k = forward_backward(X, W, b, Q, shift_labels=y, temperature=0.6, reduction=reduction,
                         compute_db=True)
    assert a["loss"] == pytest.approx(k["loss"], rel=1e-13)
    for key in ("dX", "dW", "db"):
        np.testing.assert_allclose(a[key], k[key], rtol=1e-12, atol=1e-16)


def test_ce_oracle_out_of_range_target_contributes_nothing():
    from oracle import ce_forward_backward
    rng = np.random.default_rng(22)
    X, W, b, _ = _rand_case(rng, BT=4, H=4, V=6)
    y = np.array([1, 9, 2, -5])
    r = ce_forward_backward(X, W, b, y, reduction="sum", compute_db=True)
    keep = ce_forward_backward(X[[0, 2]], W, b, y[[0, 2]], reduction="sum", compute_db=True)
    assert r["loss"] == pytest.approx(keep["loss"], rel=1e-13)
    assert np.all(r["dX"][[1, 3]] == 0.0)
    np.testing.assert_allclose(r["dW"], keep["dW"], rtol=1e-12, atol=1e-16)
