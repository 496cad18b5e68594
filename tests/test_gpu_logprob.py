"""Selective log-probability on the GPU (forward: per-row target
log-probabilities; backward: dX / dW / db for upstream per-row gradients)
against the fp64 oracle, through the C ABI and the autograd function."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from lm_head_projection_b200.workloads import make_inputs, small_case
from oracle import selective_logprob, selective_logprob_backward
from parity_utils import TOL, to_np

pytestmark = pytest.mark.gpu


def _inputs(dtype, BT, H, V, bias, T, seed):
    w = small_case(dtype=dtype, BT=BT, H=H, V=V, bias=bias, ignore_frac=0.15, temperature=T,
                   ce=True, seed=seed)
    inp = make_inputs(w)
    tgt = inp["target"].clone()
    if BT > 3:
        tgt[3] = V + 5  # outside [0, V)
    g = torch.Generator().manual_seed(seed + 1)
    dl = torch.randn(BT, generator=g, dtype=torch.float32)
    return inp, tgt, dl


def _gpu(pkg, inp, tgt, dl, dtype, T, cw, cb, accum_fp32=True):
    dev = torch.device("cuda:0")
    X, W = inp["X"].to(dev), inp["W"].to(dev)
    b = None if inp["b"] is None else inp["b"].to(dev)
    t = tgt.to(dev)
    BT, H = X.shape
    V = W.shape[0]
    dt = pkg.DTYPES[X.dtype]
    ws = torch.empty(pkg.flkl_workspace_size(BT, H, V, dt, cw, cb), dtype=torch.uint8,
                     device=dev)
    logp = torch.empty(BT, dtype=torch.float32, device=dev)
    p = lambda x: None if x is None else x.data_ptr()
    st = torch.cuda.current_stream().cuda_stream
    assert pkg.flkl_selective_logprob_forward(p(X), p(W), p(b), p(t), -100, BT, H, V, dt, T,
                                              cw, cb, p(logp), p(ws), ws.numel(), st) == 0
    pdt = torch.float32 if (accum_fp32 or dtype == "fp32") else X.dtype
    dX = torch.empty_like(X)
    dW = torch.empty((V, H), dtype=pdt, device=dev) if cw else None
    db = torch.empty(V, dtype=pdt, device=dev) if cb else None
    d = dl.to(dev)
    assert pkg.flkl_selective_logprob_backward(p(X), p(W), p(b), p(t), -100, BT, H, V, dt, T,
                                               p(d), cw, cb, accum_fp32, p(dX), p(dW), p(db),
                                               p(ws), ws.numel(), st) == 0
    torch.cuda.synchronize()
    assert pkg.flkl_device_status(p(ws), st) == 0
    return {"logp": logp, "dX": dX, "dW": dW, "db": db}


def _check(dtype, got, ref_lp, ref):
    tol = TOL[dtype]
    lp = to_np(got["logp"])
    scale = float(np.abs(ref_lp).max())
    bound = (tol["loss_rel"] if dtype == "fp32" else tol["loss_rel"]) * max(scale, 1.0)
    assert float(np.abs(lp - ref_lp).max()) <= bound
    for k in ("dX", "dW", "db"):
        if ref.get(k) is None:
            assert got[k] is None
            continue
        a, e = to_np(got[k]), ref[k]
        err = float(np.abs(a - e).max())
        assert err <= tol["grad_abs"] + tol["grad_rel_scale"] * float(np.abs(e).max()) + 1e-30, k


CASES = [("fp32", 64, 256, 1024, True, 1.0), ("fp32", 37, 64, 200, False, 0.7),
         ("bf16", 300, 256, 3000, True, 1.5), ("bf16", 129, 128, 1000, False, 1.0),
         ("bf16", 8, 4096, 4104, True, 2.0)]


@pytest.mark.parametrize("dtype,BT,H,V,bias,T", CASES)
@pytest.mark.parametrize("cw", [True, False])
def test_small_cases(dtype, BT, H, V, bias, T, cw):
    import lm_head_projection_b200 as pkg

    inp, tgt, dl = _inputs(dtype, BT, H, V, bias, T, seed=BT + V)
    got = _gpu(pkg, inp, tgt, dl, dtype, T, cw, bias)
    f = lambda t: None if t is None else to_np(t)
    ref_lp = selective_logprob(f(inp["X"]), f(inp["W"]), f(inp["b"]), tgt.numpy(), -100, T)
    ref = selective_logprob_backward(f(inp["X"]), f(inp["W"]), f(inp["b"]), tgt.numpy(),
                                     dl.numpy().astype(np.float64), -100, T, compute_dW=cw,
                                     compute_db=bias)
    _check(dtype, got, ref_lp, ref)
    assert float(got["logp"][3].cpu()) == 0.0  # target outside [0, V)


def test_headline_shape_sampled_rows():
    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.workloads import CE_WORKLOADS

    w = CE_WORKLOADS["ce_bf16_bt1024_h4096_v128256"]
    inp = make_inputs(w)
    tgt = inp["target"]
    dl = torch.randn(w.BT, generator=torch.Generator().manual_seed(7))
    got = _gpu(pkg, inp, tgt, dl, "bf16", w.temperature, True, False)
    rows = np.linspace(0, w.BT - 1, 26).astype(np.int64)
    vrows = np.linspace(0, w.V - 1, 26).astype(np.int64)
    f = lambda t: None if t is None else to_np(t)
    ref_lp = selective_logprob(f(inp["X"])[rows], f(inp["W"]), None, tgt.numpy()[rows], -100,
                               w.temperature)
    ref = selective_logprob_backward(f(inp["X"]), f(inp["W"]), None, tgt.numpy(),
                                     dl.numpy().astype(np.float64), -100, w.temperature,
                                     compute_dW=True, dX_rows=rows, dW_rows=vrows)
    sub = {"logp": got["logp"][torch.as_tensor(rows).cuda()],
           "dX": got["dX"][torch.as_tensor(rows).cuda()],
           "dW": got["dW"][torch.as_tensor(vrows).cuda()], "db": None}
    _check("bf16", sub, ref_lp, ref)


def test_autograd_follows_requires_grad_and_matches_the_oracle():
    import lm_head_projection_b200 as pkg

    inp, tgt, dl = _inputs("fp32", 96, 128, 1500, True, 1.3, seed=4)
    dev = torch.device("cuda:0")
    outs = {}
    for train in (True, False):
        X = inp["X"].to(dev).requires_grad_(True)
        W = inp["W"].to(dev).requires_grad_(train)
        b = inp["b"].to(dev).requires_grad_(train)
        logp = pkg.selective_logprob(X, W, b, tgt.to(dev), -100, 1.3)
        # a policy-gradient style objective of the per-token log-probabilities
        adv = dl.to(dev)
        loss = -(adv * torch.exp(logp - logp.detach())).sum()
        loss.backward()
        outs[train] = (X.grad.clone(), W.grad, b.grad)
    assert outs[False][1] is None and outs[False][2] is None
    assert torch.equal(outs[True][0], outs[False][0])  # dX the same either way
    f = lambda t: None if t is None else to_np(t)
    ref = selective_logprob_backward(f(inp["X"]), f(inp["W"]), f(inp["b"]), tgt.numpy(),
                                     -dl.numpy().astype(np.float64), -100, 1.3,
                                     compute_dW=True, compute_db=True)
    for k, g in zip(("dX", "dW", "db"), outs[True]):
        err = float(np.abs(to_np(g) - ref[k]).max())
        assert err <= 1e-5, (k, err)


def test_unit_upstream_gradient_gives_the_cross_entropy_gradients():
    import lm_head_projection_b200 as pkg

    inp, tgt, _ = _inputs("fp32", 80, 64, 700, True, 1.0, seed=9)
    tgt[3] = 5  # keep every non-dropped target in range
    kept = (tgt != -100)
    dl = torch.where(kept, -1.0 / float(kept.sum()), 0.0).to(torch.float32)
    got = _gpu(pkg, inp, tgt, dl, "fp32", 1.0, True, True)
    dev = torch.device("cuda:0")
    ce = pkg.cross_entropy_forward_backward(inp["X"].to(dev), inp["W"].to(dev),
                                            inp["b"].to(dev), tgt.to(dev), -100, 1.0,
                                            "batchmean", compute_dW=True, compute_db=True)
    torch.cuda.synchronize()
    for k in ("dX", "dW", "db"):
        assert float((got[k] - ce[k]).abs().max()) <= 1e-6, k
    assert abs(float(-got["logp"].sum() / kept.sum()) - float(ce["loss"])) <= 1e-5


def test_kept_first_chunk_gives_the_recomputed_gradients():
    """A whole cross-entropy call (sum reduction) forms the first vocabulary
    chunk's gradient block from the logits pass 1 kept; the selective
    log-probability backward call with upstream gradient -1 per row forms
    the same block by recomputing the logits.  Both are G = (p - onehot) / T
    on the kept rows, so dX, dW and db agree bit for bit."""
    import lm_head_projection_b200 as pkg

    T = 1.3
    inp, tgt, _ = _inputs("bf16", 300, 128, 4104, True, T, seed=21)
    dev = torch.device("cuda:0")
    X, W, b = inp["X"].to(dev), inp["W"].to(dev), inp["b"].to(dev)
    bounds = pkg.flkl_vocab_chunks(300, 128, 4104, 1, True, True)
    assert len(bounds) > 2  # several chunks: the first kept, the rest recomputed
    whole = pkg.cross_entropy_forward_backward(X, W, b, tgt.to(dev), -100, T, "sum",
                                               compute_dW=True, compute_db=True,
                                               accum_fp32=True, check_status=True)
    split = _gpu(pkg, inp, tgt, -torch.ones(300), "bf16", T, True, True)
    for k in ("dX", "dW", "db"):
        assert torch.equal(whole[k], split[k]), k
