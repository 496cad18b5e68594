"""The allocation-free entry point, flkl_forward_backward_noalloc.

It serves callers that cannot allocate device memory or hand over a
workspace (a plugin interface that only passes tensors in, or a loop where
cudaMalloc's device synchronisation is not acceptable): it runs the same
computation in a fixed 128 MiB scratch array that the library carries on
every device.  These tests call it through the C ABI and check that it gives
what the workspace entry point gives, within the parity tolerances, on two
calls in a row (the scratch keeps the previous call's contents, which must
not leak into the next result), and that sizes beyond the scratch are
refused before anything runs (a size whose regular workspace does not fit
runs without the first chunk's kept logits, recomputing that chunk, as long
as the rest fits).  Both entry points run the same deterministic
kernels on the same bytes, so the results are also compared bitwise; a
sequence of different plans (a large one, then smaller ones of other dtypes
and flags, then the large one again) shows that no stale scratch contents
reach a result.  This file is collected last.
"""

import numpy as np
import pytest
import torch

import lm_head_projection_b200 as pkg
from lm_head_projection_b200.workloads import make_inputs, small_case
from tests.parity_utils import TOL, run_gpu

pytestmark = pytest.mark.gpu

TOO_LARGE = 6


def _call_noalloc(g, w, out):
    p = lambda t: None if t is None else t.data_ptr()
    return pkg.flkl_forward_backward_noalloc(
        p(g["X"]), p(g["W"]), p(g["b"]), p(g["Q"]), p(g["shift_labels"]), g["ignore_index"],
        w.BT, w.H, w.V, 0 if w.dtype == "fp32" else 1, g["temperature"], g["eps"],
        pkg.REDUCTIONS[g["reduction"]], g["compute_dW"], g["compute_db"], g["accum_fp32"],
        p(out["loss"]), p(out["dX"]), p(out["dW"]), p(out["db"]),
        torch.cuda.current_stream().cuda_stream)


def _close(dtype, got, ref):
    tol = TOL[dtype]
    gl, rl = float(got["loss"].cpu()), float(ref["loss"].cpu())
    assert abs(gl - rl) <= tol["loss_rel"] * abs(rl) + 1e-7, (gl, rl)
    for k in ("dX", "dW", "db"):
        if ref[k] is None:
            continue
        a = got[k].float().cpu().numpy()
        e = ref[k].float().cpu().numpy()
        bound = tol["grad_abs"] + tol["grad_rel_scale"] * float(np.abs(e).max())
        assert float(np.abs(a - e).max()) <= bound + 1e-30, k


CASES = [
    small_case(dtype="bf16", BT=300, H=256, V=4104, bias=True, reduction="mean",
               ignore_frac=0.1, zero_frac=0.05, seed=7),
    small_case(dtype="bf16", BT=1024, H=512, V=8192, bias=False, reduction="batchmean", seed=8),
    small_case(dtype="fp32", BT=133, H=72, V=1000, bias=True, reduction="sum", temperature=2.0,
               seed=9),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(w):
    inp = make_inputs(w)
    ref = run_gpu(inp)  # the entry point with a caller-owned workspace
    dev = torch.device("cuda:0")
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    for _ in range(2):
        out = {k: (None if ref[k] is None else torch.full_like(ref[k], float("nan")))
               for k in ("loss", "dX", "dW", "db")}
        assert _call_noalloc(g, w, out) == 0
        torch.cuda.synchronize()
        _close(w.dtype, out, ref)
        _same_bytes(out, ref)


def _same_bytes(got, ref):
    for k in ("loss", "dX", "dW", "db"):
        if ref[k] is None:
            assert got[k] is None, k
        else:
            assert torch.equal(got[k], ref[k]), k


# A large plan first (most of the scratch: a 1024-row, 16384-column head with
# dW), then smaller ones with other dtypes and flags, then the large one again.
SEQUENCE = [
    small_case(dtype="bf16", BT=1024, H=4096, V=16384, bias=False, reduction="batchmean",
               w_std=0.02, seed=21),
    small_case(dtype="bf16", BT=77, H=128, V=1032, bias=True, reduction="mean",
               ignore_frac=0.2, zero_frac=0.05, temperature=1.5, seed=22),
    small_case(dtype="fp32", BT=50, H=64, V=520, bias=True, reduction="sum", seed=23),
    small_case(dtype="bf16", BT=300, H=256, V=4104, bias=True, reduction="batchmean",
               compute_dW=False, seed=24),
]


def test_noalloc_interleaved_plans_give_the_workspace_entry_bytes():
    dev = torch.device("cuda:0")
    runs = []
    for w in SEQUENCE:
        inp = make_inputs(w)
        runs.append((w, {k: (v.to(dev) if isinstance(v, torch.Tensor) else v)
                         for k, v in inp.items()}, run_gpu(inp)))
    for w, g, ref in runs + runs[:1]:
        out = {k: (None if ref[k] is None else torch.full_like(ref[k], float("nan")))
               for k in ("loss", "dX", "dW", "db")}
        assert _call_noalloc(g, w, out) == 0
        torch.cuda.synchronize()
        _close(w.dtype, out, ref)
        _same_bytes(out, ref)


def test_noalloc_headline_recomputes_the_first_chunk_with_the_same_bytes():
    """At the headline size the regular workspace (with the first chunk's
    kept logits) exceeds the scratch; the allocation-free call runs without
    them, recomputing that chunk, and must give the regular call's bytes."""
    from lm_head_projection_b200.workloads import WORKLOADS

    w = WORKLOADS["bf16_bt1024_h4096_v128256"]
    assert pkg.flkl_workspace_size(w.BT, w.H, w.V, 1, 1, 0) > 128 * 2**20
    dev = torch.device("cuda:0")
    g = make_inputs(w, device=dev)
    ref = run_gpu(g)
    out = {k: (None if ref[k] is None else torch.full_like(ref[k], float("nan")))
           for k in ("loss", "dX", "dW", "db")}
    assert _call_noalloc(g, w, out) == 0
    torch.cuda.synchronize()
    _same_bytes(out, ref)


def test_noalloc_refuses_sizes_beyond_the_scratch():
    # BT=8192 rows over V=65536 need a 128 MiB gradient staging block alone
    w = small_case(dtype="bf16", BT=8192, H=64, V=65536, bias=False, seed=10)
    assert pkg.flkl_workspace_size(w.BT, w.H, w.V, 1, 1, 0) > 128 * 2**20
    dev = torch.device("cuda:0")
    g = dict(X=torch.zeros((w.BT, w.H), dtype=torch.bfloat16, device=dev),
             W=torch.zeros((w.V, w.H), dtype=torch.bfloat16, device=dev), b=None,
             Q=torch.zeros((w.BT, w.V), dtype=torch.bfloat16, device=dev), shift_labels=None,
             ignore_index=-100, temperature=1.0, eps=1e-10, reduction="batchmean",
             compute_dW=True, compute_db=False, accum_fp32=True)
    out = {"loss": torch.full((), 5.0, device=dev),
           "dX": torch.full((w.BT, w.H), 5.0, device=dev).to(torch.bfloat16),
           "dW": torch.full((w.V, w.H), 5.0, device=dev), "db": None}
    assert _call_noalloc(g, w, out) == TOO_LARGE
    torch.cuda.synchronize()
    assert float(out["loss"].cpu()) == 5.0
    assert bool((out["dW"] == 5.0).all()) and bool((out["dX"] == 5.0).all())
    assert "128 MiB" in pkg.flkl_status_string(TOO_LARGE)
