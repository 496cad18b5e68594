"""The device-side gradient scaling of the autograd wrappers
(flkl_scale_cast): every dtype pair, ragged lengths, a scale of 1 giving the
plain cast bitwise, other scales against torch, in place, and the autograd
backward with an incoming gradient other than 1 (no host synchronisation on
the way)."""

from __future__ import annotations

import pytest
import torch

pytestmark = pytest.mark.gpu

DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


@pytest.mark.parametrize("src,dst", [("fp32", "fp32"), ("fp32", "bf16"), ("bf16", "fp32"),
                                     ("bf16", "bf16")])
@pytest.mark.parametrize("n", [0, 7, 8, 65537, 3_000_001])
@pytest.mark.parametrize("scale", [None, 1.0, -2.5])
def test_scale_cast_matches_torch(src, dst, n, scale):
    import lm_head_projection_b200 as pkg

    g = torch.Generator(device="cuda").manual_seed(n)
    x = torch.randn(n, generator=g, device="cuda").to(DT[src])
    y = torch.full((n,), 7.0, device="cuda", dtype=DT[dst])
    s = None if scale is None else torch.tensor(scale, device="cuda", dtype=torch.float32)
    st = pkg.flkl_scale_cast(x.data_ptr() if n else None, pkg.DTYPES[x.dtype],
                             y.data_ptr() if n else None, pkg.DTYPES[y.dtype], n,
                             None if s is None else s.data_ptr(),
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    if scale is None or scale == 1.0:
        ref = x.to(DT[dst])  # a plain cast, bitwise
    else:
        ref = (x.float() * scale).to(DT[dst])
    assert torch.equal(y, ref)


def test_scale_cast_in_place_and_errors():
    import lm_head_projection_b200 as pkg

    x = torch.randn(1001, device="cuda")
    ref = x * 3.0
    s = torch.tensor(3.0, device="cuda")
    cs = torch.cuda.current_stream().cuda_stream
    assert pkg.flkl_scale_cast(x.data_ptr(), 0, x.data_ptr(), 0, x.numel(), s.data_ptr(), cs) == 0
    torch.cuda.synchronize()
    assert torch.equal(x, ref)
    # in place across dtypes, a negative length, an unknown dtype, misalignment
    assert pkg.flkl_scale_cast(x.data_ptr(), 0, x.data_ptr(), 1, 8, None, cs) == 1
    assert pkg.flkl_scale_cast(x.data_ptr(), 0, x.data_ptr(), 0, -1, None, cs) == 1
    assert pkg.flkl_scale_cast(x.data_ptr(), 5, x.data_ptr(), 0, 8, None, cs) == 1
    assert pkg.flkl_scale_cast(x.data_ptr() + 4, 0, x.data_ptr(), 0, 8, None, cs) == 2


def test_autograd_backward_applies_the_incoming_gradient_on_the_device():
    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.workloads import make_inputs, small_case

    w = small_case(dtype="bf16", BT=100, H=64, V=520, bias=True, seed=3)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in make_inputs(w).items()}
    direct = pkg.forward_backward(g["X"], g["W"], g["b"], g["Q"], compute_dW=True,
                                  compute_db=True, accum_fp32=True)
    mod = pkg.FusedLinearKLDivLoss(accum_dtype=torch.float32)
    for gscale in (1.0, -0.75):
        X = g["X"].clone().requires_grad_()
        W = g["W"].clone().requires_grad_()
        b = g["b"].clone().requires_grad_()
        loss = mod(W, X, g["Q"], bias=b)
        loss.backward(torch.tensor(gscale, device="cuda"))
        assert torch.equal(X.grad, (direct["dX"].float() * gscale).to(torch.bfloat16)
                           if gscale != 1.0 else direct["dX"])
        assert torch.equal(W.grad, (direct["dW"] * gscale).to(torch.bfloat16))
        assert torch.equal(b.grad, (direct["db"] * gscale).to(torch.bfloat16))
