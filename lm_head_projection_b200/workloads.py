"""Seeded synthetic inputs for the fused linear-head + KL-divergence loss.

This module only draws inputs; it holds none of the loss arithmetic.  Both the
CUDA path (through the tests and the benchmark) and the fp64 oracle read the
tensors it returns, so that the two compute on identical bytes.

The workloads follow the distillation setting of the "Add FusedLinearKLDivLoss"
pull-request page (Liger-Kernel mirror), section *Details*: a llama-3 shaped
vocabulary head (H=4096, V=128256) and, for the largest case, the B=8, T=1024,
V=151936 head of the GRPO frozen-head page (section *Details*).  The pages use
no dataset, so every tensor is drawn from the distributions named per workload:

* X ~ N(0, x_std^2), W ~ N(0, w_std^2), b ~ N(0, b_std^2) (second argument of
  N(.,.) read as a standard deviation, except the small fp32 case whose W has
  variance 1/H, i.e. std 1/sqrt(H));
* teacher Q = softmax(teacher logits) per row, teacher logits ~ N(0, q_std^2),
  softmax taken in fp32 (fp64 for the fp32 workload) and then cast to the
  workload dtype;
* optionally a fraction of each row's entries set to exactly 0 (chosen
  uniformly without replacement) and the row renormalised before the cast;
* optionally a fraction of rows whose shift label equals ignore_index (-100),
  chosen by a seeded permutation; the other labels are uniform in [0, V).

Every tensor has its own counter-seeded torch.Generator so a tensor's bytes do
not depend on how the others were drawn; Q is drawn in row blocks, each with
its own generator, so the host never holds a BT x V fp32 array for more than one
block.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

IGNORE_INDEX = -100

# Stream ids used to derive the per-tensor seeds.
_S_X, _S_W, _S_B, _S_TEACHER, _S_ZEROS, _S_IGNORE, _S_LABELS = range(1, 8)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "fp32" | "bf16"
    BT: int
    H: int
    V: int
    bias: bool
    x_std: float
    w_std: float
    b_std: float
    q_std: float
    temperature: float
    eps: float
    reduction: str  # "batchmean" | "mean" | "sum"
    compute_dW: bool
    compute_db: bool
    accum_fp32: bool
    ignore_frac: float = 0.0
    zero_frac: float = 0.0
    seed: int = 0
    ce: bool = False  # cross-entropy: one-hot teacher at an integer target per row

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def flops_counted(self) -> float:
        """Counted FLOPs of one call: one logits GEMM, the dX GEMM and, when
        the head is trained, the dW GEMM (2*BT*H*V each)."""
        return 2.0 * self.BT * self.H * self.V * (2 + int(self.compute_dW))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: the small fp32 case, the headline bf16 case, the frozen
# head with ignored rows, the trained head with bias and a peaked teacher, and
# the B=8,T=1024 frozen head at V=151936.
WORKLOADS = {
    "fp32_bt64_h256_v1024": Workload(
        "fp32_bt64_h256_v1024", "fp32", 64, 256, 1024, False,
        x_std=1.0, w_std=1.0 / math.sqrt(256), b_std=0.0, q_std=2.0,
        temperature=1.0, eps=1e-10, reduction="batchmean",
        compute_dW=True, compute_db=False, accum_fp32=True),
    "bf16_bt1024_h4096_v128256": Workload(
        "bf16_bt1024_h4096_v128256", "bf16", 1024, 4096, 128256, False,
        x_std=1.0, w_std=0.02, b_std=0.0, q_std=2.0,
        temperature=1.0, eps=1e-10, reduction="batchmean",
        compute_dW=True, compute_db=False, accum_fp32=True),
    "bf16_bt2048_h4096_v128256_frozen_ignore_t2_sum": Workload(
        "bf16_bt2048_h4096_v128256_frozen_ignore_t2_sum", "bf16", 2048, 4096, 128256, False,
        x_std=1.0, w_std=0.02, b_std=0.0, q_std=2.0,
        temperature=2.0, eps=1e-10, reduction="sum",
        compute_dW=False, compute_db=False, accum_fp32=True, ignore_frac=0.1),
    "bf16_bt4096_h4096_v128256_bias_mean_peaked": Workload(
        "bf16_bt4096_h4096_v128256_bias_mean_peaked", "bf16", 4096, 4096, 128256, True,
        x_std=1.0, w_std=0.02, b_std=0.02, q_std=4.0,
        temperature=1.0, eps=1e-10, reduction="mean",
        compute_dW=True, compute_db=True, accum_fp32=True, zero_frac=0.05),
    "bf16_bt8192_h4096_v151936_frozen": Workload(
        "bf16_bt8192_h4096_v151936_frozen", "bf16", 8192, 4096, 151936, False,
        x_std=1.0, w_std=0.02, b_std=0.0, q_std=2.0,
        temperature=1.0, eps=1e-10, reduction="batchmean",
        compute_dW=False, compute_db=False, accum_fp32=True),
}

WORKLOAD_ORDER = list(WORKLOADS)
HEADLINE = "bf16_bt1024_h4096_v128256"


# Cross-entropy workloads (the one-hot-teacher case): the headline head shape
# with uniform targets, 10 % of rows dropped, and a small fp32 case.
CE_WORKLOADS = {
    "ce_bf16_bt1024_h4096_v128256": Workload(
        "ce_bf16_bt1024_h4096_v128256", "bf16", 1024, 4096, 128256, False,
        x_std=1.0, w_std=0.02, b_std=0.0, q_std=0.0,
        temperature=1.0, eps=0.0, reduction="batchmean",
        compute_dW=True, compute_db=False, accum_fp32=True, ignore_frac=0.1, ce=True),
    "ce_fp32_bt64_h256_v1024": Workload(
        "ce_fp32_bt64_h256_v1024", "fp32", 64, 256, 1024, True,
        x_std=1.0, w_std=1.0 / math.sqrt(256), b_std=0.02, q_std=0.0,
        temperature=1.0, eps=0.0, reduction="batchmean",
        compute_dW=True, compute_db=True, accum_fp32=True, ignore_frac=0.1, ce=True),
}


def _gen(device, seed: int, stream: int, block: int = 0) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(((seed * 1_000_003 + stream) * 1_000_033 + block) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _randn(shape, std, device, gen, dtype):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_inputs(w: Workload, device="cpu", q_block_rows: int = 256) -> dict:
    """Draw the inputs of workload ``w`` on ``device``.

    Returns a dict with X [BT,H], W [V,H], b [V] or None, Q [BT,V] (all in the
    workload dtype, contiguous), shift_labels [BT] int64 or None, and the scalar
    settings.  The same seed on the CPU always gives the same bytes.
    """
    dt = w.torch_dtype
    X = _randn((w.BT, w.H), w.x_std, device, _gen(device, w.seed, _S_X), dt)
    W = _randn((w.V, w.H), w.w_std, device, _gen(device, w.seed, _S_W), dt)
    b = _randn((w.V,), w.b_std, device, _gen(device, w.seed, _S_B), dt) if w.bias else None

    if w.ce:
        target = torch.randint(0, w.V, (w.BT,), generator=_gen(device, w.seed, _S_LABELS),
                               device=device, dtype=torch.int64)
        n_ign = int(round(w.ignore_frac * w.BT))
        if n_ign:
            perm = torch.randperm(w.BT, generator=_gen(device, w.seed, _S_IGNORE), device=device)
            target[perm[:n_ign]] = IGNORE_INDEX
        return dict(X=X, W=W, b=b, Q=None, target=target, shift_labels=None,
                    ignore_index=IGNORE_INDEX, temperature=w.temperature, eps=w.eps,
                    reduction=w.reduction, compute_dW=w.compute_dW,
                    compute_db=w.compute_db and w.bias, accum_fp32=w.accum_fp32)

    soft_dtype = torch.float64 if w.dtype == "fp32" else torch.float32
    Q = torch.empty((w.BT, w.V), dtype=dt, device=device)
    n_zero = int(round(w.zero_frac * w.V))
    for blk, r0 in enumerate(range(0, w.BT, q_block_rows)):
        r1 = min(w.BT, r0 + q_block_rows)
        g = _gen(device, w.seed, _S_TEACHER, blk)
        logits = torch.randn((r1 - r0, w.V), generator=g, device=device, dtype=torch.float32)
        logits = logits.to(soft_dtype).mul_(w.q_std)
        q = torch.softmax(logits, dim=1)
        if n_zero:
            gz = _gen(device, w.seed, _S_ZEROS, blk)
            # n_zero distinct columns per row: the first n_zero entries of a
            # uniformly random ordering of the row's columns.
            keys = torch.rand((r1 - r0, w.V), generator=gz, device=device)
            cols = torch.topk(keys, n_zero, dim=1, largest=False).indices
            q.scatter_(1, cols, 0.0)
            q.div_(q.sum(dim=1, keepdim=True))
        Q[r0:r1] = q.to(dt)
        del logits, q

    labels = None
    if w.ignore_frac > 0.0:
        labels = torch.randint(0, w.V, (w.BT,), generator=_gen(device, w.seed, _S_LABELS),
                               device=device, dtype=torch.int64)
        n_ign = int(round(w.ignore_frac * w.BT))
        perm = torch.randperm(w.BT, generator=_gen(device, w.seed, _S_IGNORE), device=device)
        labels[perm[:n_ign]] = IGNORE_INDEX

    return dict(X=X, W=W, b=b, Q=Q, shift_labels=labels, ignore_index=IGNORE_INDEX,
                temperature=w.temperature, eps=w.eps, reduction=w.reduction,
                compute_dW=w.compute_dW, compute_db=w.compute_db and w.bias,
                accum_fp32=w.accum_fp32)


def small_case(dtype="bf16", BT=133, H=192, V=1000, bias=True, reduction="batchmean",
               temperature=1.0, eps=1e-10, ignore_frac=0.0, zero_frac=0.0,
               compute_dW=True, compute_db=None, q_std=2.0, x_std=1.0, w_std=None,
               b_std=0.02, seed=0, ce=False) -> Workload:
    """A small workload for parity tests: several tiles and a ragged tail."""
    if w_std is None:
        w_std = 1.0 / math.sqrt(H)
    if compute_db is None:
        compute_db = bias
    return Workload(f"small_{'ce_' if ce else ''}{dtype}_{BT}x{H}x{V}", dtype, BT, H, V, bias,
                    x_std, w_std, b_std, q_std, temperature, eps, reduction, compute_dW,
                    compute_db, True, ignore_frac, zero_frac, seed, ce)


# ----------------------------------------------------------------- norm backward
# Shapes (rows, H) of the LoRA normalization pull-request page, *Benchmark
# Results* (bf16).  That page names no input distribution; the one below is a
# plain choice: hidden states with a per-row offset (so LayerNorm's centring
# matters), a unit-scale incoming gradient, and norm weights near 1.
NORM_SHAPES = [(2048, 4096), (4096, 4096), (4096, 8192), (8192, 4096), (8192, 8192)]
_S_NX, _S_NXM, _S_NDY, _S_NW = range(11, 15)


def make_norm_inputs(rows: int, H: int, dtype: str = "bf16", seed: int = 0,
                     device="cpu") -> dict:
    """dY, X [rows, H] and W [H]: X = m_row + N(0, 1) with m_row ~ N(0, 1),
    dY ~ N(0, 1), W = 1 + N(0, 0.1^2); cast to ``dtype`` ("fp32" | "bf16")."""
    dt = torch.float32 if dtype == "fp32" else torch.bfloat16
    x = torch.randn((rows, H), generator=_gen(device, seed, _S_NX), device=device)
    x += torch.randn((rows, 1), generator=_gen(device, seed, _S_NXM), device=device)
    dy = torch.randn((rows, H), generator=_gen(device, seed, _S_NDY), device=device)
    w = 1.0 + 0.1 * torch.randn((H,), generator=_gen(device, seed, _S_NW), device=device)
    return dict(dY=dy.to(dt), X=x.to(dt), W=w.to(dt))
