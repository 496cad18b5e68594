"""RMSNorm / LayerNorm backward with frozen-parameter flags.

The LoRA normalization pull-request page (*Key Changes*): when a norm's
weight (bias) is frozen, its gradient is neither accumulated nor reduced;
the input gradient does not change.  ``rms_norm_backward`` and
``layer_norm_backward`` marshal torch tensors into the C entry points
``flkl_rms_norm_backward`` / ``flkl_layer_norm_backward``; the autograd
modules below take the flags from ``requires_grad`` of the parameters.
There is no PyTorch fallback: the CUDA library does every step.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import (DTYPES, FLKL_OK, FlklError, _check_dev, _ptr, flkl_layer_norm_backward,
               flkl_norm_workspace_size, flkl_rms_norm_backward)

__all__ = ["rms_norm_backward", "layer_norm_backward", "RMSNorm", "LayerNorm"]


def _prepare(dY, X, W, accum_fp32):
    if X.dtype not in DTYPES:
        raise ValueError(f"dtype {X.dtype} not supported (float32 or bfloat16)")
    if X.dim() < 1:
        raise ValueError("X needs a last (hidden) dimension")
    H = X.shape[-1]
    rows = X.numel() // H if H else 0
    dev, dt = X.device, X.dtype
    _check_dev("X", X, dt, X.shape, dev)
    _check_dev("dY", dY, dt, X.shape, dev)
    _check_dev("W", W, dt, (H,), dev)
    pdt = torch.float32 if (accum_fp32 or dt == torch.float32) else dt
    return rows, H, dev, dt, pdt


def rms_norm_backward(dY: torch.Tensor, X: torch.Tensor, W: torch.Tensor, eps: float = 1e-6,
                      compute_dW: bool = True, accum_fp32: bool = True,
                      stream: Optional[torch.cuda.Stream] = None) -> dict:
    """dX (and dW unless the weight is frozen) of ``y = W * X / rms(X)``
    over the last dimension; returns ``{"dX", "dW"}`` (dW None when frozen)."""
    rows, H, dev, dt, pdt = _prepare(dY, X, W, accum_fp32)
    dX = torch.empty_like(X)
    dW = torch.empty((H,), dtype=pdt, device=dev) if compute_dW else None
    need = flkl_norm_workspace_size(rows, H, compute_dW, False)
    ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    status = flkl_rms_norm_backward(_ptr(dY), _ptr(X), _ptr(W), rows, H, DTYPES[dt], eps,
                                    compute_dW, accum_fp32, _ptr(dX), _ptr(dW), _ptr(ws), need,
                                    st.cuda_stream)
    if status != FLKL_OK:
        raise FlklError(status, "flkl_rms_norm_backward")
    return {"dX": dX, "dW": dW}


def layer_norm_backward(dY: torch.Tensor, X: torch.Tensor, W: torch.Tensor, eps: float = 1e-5,
                        compute_dW: bool = True, compute_db: bool = True,
                        accum_fp32: bool = True,
                        stream: Optional[torch.cuda.Stream] = None) -> dict:
    """dX, dW and db (None when frozen) of ``y = W * (X - mean) / std + b``
    over the last dimension; returns ``{"dX", "dW", "db"}``."""
    rows, H, dev, dt, pdt = _prepare(dY, X, W, accum_fp32)
    dX = torch.empty_like(X)
    dW = torch.empty((H,), dtype=pdt, device=dev) if compute_dW else None
    db = torch.empty((H,), dtype=pdt, device=dev) if compute_db else None
    need = flkl_norm_workspace_size(rows, H, compute_dW, compute_db)
    ws = torch.empty(need, dtype=torch.uint8, device=dev) if need else None
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    status = flkl_layer_norm_backward(_ptr(dY), _ptr(X), _ptr(W), rows, H, DTYPES[dt], eps,
                                      compute_dW, compute_db, accum_fp32, _ptr(dX), _ptr(dW),
                                      _ptr(db), _ptr(ws), need, st.cuda_stream)
    if status != FLKL_OK:
        raise FlklError(status, "flkl_layer_norm_backward")
    return {"dX": dX, "dW": dW, "db": db}


class _RMSNormFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, eps):
        ctx.save_for_backward(X, W)
        ctx.eps = eps
        # forward in torch (not a hot path here; the backward is the kernel)
        Xf = X.float()
        r = torch.rsqrt(Xf.pow(2).mean(-1, keepdim=True) + eps)
        return (Xf * r * W.float()).to(X.dtype)

    @staticmethod
    def backward(ctx, dY):
        X, W = ctx.saved_tensors
        r = rms_norm_backward(dY.contiguous(), X, W, ctx.eps, compute_dW=ctx.needs_input_grad[1])
        dW = None if r["dW"] is None else r["dW"].to(W.dtype)
        return r["dX"], dW, None


class _LayerNormFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, b, eps):
        ctx.save_for_backward(X, W)
        ctx.eps = eps
        Xf = X.float()
        mu = Xf.mean(-1, keepdim=True)
        var = (Xf - mu).pow(2).mean(-1, keepdim=True)
        return ((Xf - mu) * torch.rsqrt(var + eps) * W.float() + b.float()).to(X.dtype)

    @staticmethod
    def backward(ctx, dY):
        X, W = ctx.saved_tensors
        r = layer_norm_backward(dY.contiguous(), X, W, ctx.eps,
                                compute_dW=ctx.needs_input_grad[1],
                                compute_db=ctx.needs_input_grad[2])
        dW = None if r["dW"] is None else r["dW"].to(W.dtype)
        db = None if r["db"] is None else r["db"].to(W.dtype)
        return r["dX"], dW, db, None


class RMSNorm(torch.nn.Module):
    """RMSNorm whose backward skips dW when ``weight.requires_grad`` is False."""

    def __init__(self, hidden: int, eps: float = 1e-6, dtype=torch.bfloat16, device=None):
        super().__init__()
        self.weight = torch.nn.Parameter(torch.ones(hidden, dtype=dtype, device=device))
        self.eps = eps

    def forward(self, x):
        return _RMSNormFunction.apply(x.contiguous(), self.weight, self.eps)


class LayerNorm(torch.nn.Module):
    """LayerNorm whose backward skips dW / db for frozen weight / bias."""

    def __init__(self, hidden: int, eps: float = 1e-5, dtype=torch.bfloat16, device=None):
        super().__init__()
        self.weight = torch.nn.Parameter(torch.ones(hidden, dtype=dtype, device=device))
        self.bias = torch.nn.Parameter(torch.zeros(hidden, dtype=dtype, device=device))
        self.eps = eps

    def forward(self, x):
        return _LayerNormFunction.apply(x.contiguous(), self.weight, self.bias, self.eps)
