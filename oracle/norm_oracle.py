"""fp64 CPU oracle of the RMSNorm / LayerNorm backward with frozen-parameter
flags.

TEST INFRASTRUCTURE (same rules as flkl_oracle: only the tests and the
benchmark's CPU leg use it; it imports nothing from the product package).

The LoRA normalization pull-request page (Liger-Kernel mirror), *Key
Changes*, adds COMPUTE_DW to the RMSNorm backward and COMPUTE_DW /
COMPUTE_DB to the LayerNorm backward: when the norm's weight (bias) is frozen
the weight (bias) gradient is not accumulated and not reduced, and the input
gradient is unchanged (*Test Validation*: exact x.grad equality).  The pages
do not print the norms; the plainest reading is the textbook forward

    RMSNorm:   y = w * x / r,         r = sqrt(mean(x^2) + eps)
    LayerNorm: y = w * (x - mu) / s + b,   mu = mean(x), s = sqrt(var(x) + eps)

(var the biased variance), with the backward of those definitions for an
incoming gradient dy; mean/var over the last (hidden) dimension, one row per
token.  The statistics are recomputed from x (the backward does not need the
forward's saved values).
"""

from __future__ import annotations

import numpy as np


def rms_norm_backward(dy, x, w, eps=1e-6, compute_dW=True):
    """dx [N,H] and dW [H] (None when frozen) of y = w * x / r."""
    dy = np.asarray(dy, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    H = x.shape[1]
    r = np.sqrt((x * x).mean(axis=1, keepdims=True) + eps)
    xhat = x / r
    g = dy * w                                   # d loss / d xhat
    # d xhat / d x: (I - xhat xhat^T / H) / r
    dx = (g - xhat * (g * xhat).sum(axis=1, keepdims=True) / H) / r
    dW = (dy * xhat).sum(axis=0) if compute_dW else None
    return dx, dW


def layer_norm_backward(dy, x, w, eps=1e-5, compute_dW=True, compute_db=True):
    """dx [N,H], dW [H] and db [H] (None when not asked for) of
    y = w * (x - mu) / s + b."""
    dy = np.asarray(dy, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    H = x.shape[1]
    mu = x.mean(axis=1, keepdims=True)
    xc = x - mu
    s = np.sqrt((xc * xc).mean(axis=1, keepdims=True) + eps)
    xhat = xc / s
    g = dy * w
    dx = (g - g.mean(axis=1, keepdims=True)
          - xhat * (g * xhat).sum(axis=1, keepdims=True) / H) / s
    dW = (dy * xhat).sum(axis=0) if compute_dW else None
    db = dy.sum(axis=0) if compute_db else None
    return dx, dW, db
