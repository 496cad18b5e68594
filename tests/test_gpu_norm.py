"""Parity of the RMSNorm / LayerNorm backward (frozen-parameter flags) with
the fp64 oracle, on the CUDA library through the C ABI.

The LoRA normalization pull-request page (*Key Changes*, *Test Validation*):
with a frozen weight / bias no gradient is produced for it, and x.grad is
exactly the same as with the parameter trainable.

Tolerances (max-abs error against the oracle, relative to the largest oracle
value of that output): fp32 2e-5 (fp32 sums over up to 8192 terms); bf16
2e-2 (dX is rounded to bf16, i.e. 2^-8 relative, plus the bf16 inputs'
effect on the fp32 row statistics).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from lm_head_projection_b200.workloads import NORM_SHAPES, make_norm_inputs
from oracle.norm_oracle import layer_norm_backward as o_ln
from oracle.norm_oracle import rms_norm_backward as o_rms

pytestmark = pytest.mark.gpu

REL = {"fp32": 2e-5, "bf16": 2e-2}
EPS = {"rms": 1e-6, "layer": 1e-5}


def _np(t):
    return None if t is None else t.detach().float().cpu().numpy()


def run_pair(kind, rows, H, dtype, cw, cb=False, seed=0, accum_fp32=True):
    from lm_head_projection_b200 import norm

    inp = make_norm_inputs(rows, H, dtype, seed)
    g = {k: v.cuda() for k, v in inp.items()}
    if kind == "rms":
        got = norm.rms_norm_backward(g["dY"], g["X"], g["W"], EPS[kind], compute_dW=cw,
                                     accum_fp32=accum_fp32)
        dx, dw = o_rms(_np(inp["dY"]), _np(inp["X"]), _np(inp["W"]), EPS[kind], compute_dW=cw)
        ref = {"dX": dx, "dW": dw}
    else:
        got = norm.layer_norm_backward(g["dY"], g["X"], g["W"], EPS[kind], compute_dW=cw,
                                       compute_db=cb, accum_fp32=accum_fp32)
        dx, dw, db = o_ln(_np(inp["dY"]), _np(inp["X"]), _np(inp["W"]), EPS[kind],
                          compute_dW=cw, compute_db=cb)
        ref = {"dX": dx, "dW": dw, "db": db}
    torch.cuda.synchronize()
    return got, ref


def check(dtype, got, ref):
    for k, e in ref.items():
        if e is None:
            assert got[k] is None, k
            continue
        a = _np(got[k])
        assert a.shape == e.shape, (k, a.shape, e.shape)
        assert np.all(np.isfinite(a)), k
        if e.size == 0:
            continue
        err = float(np.abs(a - e).max())
        bound = REL[dtype] * max(float(np.abs(e).max()), 1e-30)
        assert err <= bound, (k, err, bound)


SMALL = [(1, 8), (37, 200), (300, 2056), (129, 4096), (70, 4104), (65, 8192), (1000, 64)]


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("rows,H", SMALL)
@pytest.mark.parametrize("cw", [True, False])
def test_rms_norm_small(dtype, rows, H, cw):
    got, ref = run_pair("rms", rows, H, dtype, cw, seed=rows + H)
    check(dtype, got, ref)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("rows,H", SMALL)
@pytest.mark.parametrize("cw,cb", [(True, True), (True, False), (False, True), (False, False)])
def test_layer_norm_small(dtype, rows, H, cw, cb):
    got, ref = run_pair("layer", rows, H, dtype, cw, cb, seed=rows * 7 + H)
    check(dtype, got, ref)


@pytest.mark.parametrize("kind", ["rms", "layer"])
def test_bf16_parameter_gradients_without_fp32_accumulation(kind):
    got, ref = run_pair(kind, 333, 1024, "bf16", True, True, accum_fp32=False)
    assert got["dW"].dtype == torch.bfloat16
    check("bf16", got, ref)


@pytest.mark.parametrize("kind", ["rms", "layer"])
@pytest.mark.parametrize("rows,H", NORM_SHAPES)
def test_page_shapes_bf16(kind, rows, H):
    got, ref = run_pair(kind, rows, H, "bf16", True, True, seed=1)
    check("bf16", got, ref)


@pytest.mark.parametrize("kind", ["rms", "layer"])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_frozen_parameters_leave_dx_bitwise_unchanged(kind, dtype):
    from lm_head_projection_b200 import norm

    inp = {k: v.cuda() for k, v in make_norm_inputs(2048, 4096, dtype, 5).items()}
    outs = []
    flags = [(True, True), (False, False), (True, False), (False, True)]
    for cw, cb in flags if kind == "layer" else [(True, False), (False, False)]:
        if kind == "rms":
            r = norm.rms_norm_backward(inp["dY"], inp["X"], inp["W"], compute_dW=cw)
        else:
            r = norm.layer_norm_backward(inp["dY"], inp["X"], inp["W"], compute_dW=cw,
                                         compute_db=cb)
        assert (r["dW"] is None) == (not cw)
        outs.append(r["dX"])
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_zero_rows_give_zero_parameter_gradients():
    from lm_head_projection_b200 import norm

    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    w = torch.ones(256, dtype=torch.bfloat16, device="cuda")
    r = norm.layer_norm_backward(x, x, w, compute_dW=True, compute_db=True)
    torch.cuda.synchronize()
    assert r["dX"].shape == (0, 256)
    assert torch.count_nonzero(r["dW"]) == 0 and torch.count_nonzero(r["db"]) == 0


def test_deterministic_parameter_gradients():
    from lm_head_projection_b200 import norm

    inp = {k: v.cuda() for k, v in make_norm_inputs(4096, 4096, "bf16", 9).items()}
    a = norm.layer_norm_backward(inp["dY"], inp["X"], inp["W"])
    b = norm.layer_norm_backward(inp["dY"], inp["X"], inp["W"])
    assert torch.equal(a["dW"], b["dW"]) and torch.equal(a["db"], b["db"])
    assert torch.equal(a["dX"], b["dX"])
    import lm_head_projection_b200 as pkg
    assert pkg.flkl_norm_device_status(torch.cuda.current_stream().cuda_stream) == 0


@pytest.mark.parametrize("freeze_w,freeze_b", [(False, False), (True, False), (True, True)])
def test_modules_follow_requires_grad(freeze_w, freeze_b):
    from lm_head_projection_b200.norm import LayerNorm, RMSNorm

    torch.manual_seed(0)
    x = torch.randn(64, 512, device="cuda", dtype=torch.float32)
    for mod in (RMSNorm(512, dtype=torch.float32, device="cuda"),
                LayerNorm(512, dtype=torch.float32, device="cuda")):
        mod.weight.requires_grad_(not freeze_w)
        if hasattr(mod, "bias"):
            mod.bias.requires_grad_(not freeze_b)
        xi = x.clone().requires_grad_(True)
        y = mod(xi)
        y.backward(torch.ones_like(y))
        assert (mod.weight.grad is None) == freeze_w
        if hasattr(mod, "bias"):
            assert (mod.bias.grad is None) == freeze_b
        assert xi.grad is not None and torch.isfinite(xi.grad).all()
