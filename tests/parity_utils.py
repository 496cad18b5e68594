"""Shared helpers of the parity tests: run the CUDA path and the fp64 oracle on
the same seeded inputs and compare with the tolerances of the workload dtype.

Tolerances: fp32 inputs -> loss relative error <= 1e-4 and gradient max-abs
error <= 1e-5; bf16 inputs -> loss relative error <= 2e-2 and gradient max-abs
error <= 2e-2 * max |oracle gradient|.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import forward_backward as oracle_fb

TOL = {
    "fp32": dict(loss_rel=1e-4, grad_abs=1e-5, grad_rel_scale=0.0),
    "bf16": dict(loss_rel=2e-2, grad_abs=0.0, grad_rel_scale=2e-2),
}


def to_np(t):
    return None if t is None else t.detach().float().cpu().numpy()


def run_gpu(inp: dict, compute_dW=None, compute_db=None, accum_fp32=None, device="cuda:0"):
    import lm_head_projection_b200 as pkg

    dev = torch.device(device)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    if g.get("target") is not None:  # cross-entropy workload
        r = pkg.cross_entropy_forward_backward(
            g["X"], g["W"], g["b"], g["target"], g["ignore_index"], g["temperature"],
            g["reduction"],
            compute_dW=inp["compute_dW"] if compute_dW is None else compute_dW,
            compute_db=inp["compute_db"] if compute_db is None else compute_db,
            accum_fp32=inp["accum_fp32"] if accum_fp32 is None else accum_fp32,
            check_status=True)
        torch.cuda.synchronize()
        return r
    r = pkg.forward_backward(
        g["X"], g["W"], g["b"], g["Q"], g["shift_labels"], g["ignore_index"], g["temperature"],
        g["eps"], g["reduction"],
        compute_dW=inp["compute_dW"] if compute_dW is None else compute_dW,
        compute_db=inp["compute_db"] if compute_db is None else compute_db,
        accum_fp32=inp["accum_fp32"] if accum_fp32 is None else accum_fp32,
        check_status=True)
    torch.cuda.synchronize()
    return r


def run_oracle(inp: dict, dX_rows=None, dW_rows=None, compute_dW=None, compute_db=None):
    if inp.get("target") is not None:
        from oracle import ce_forward_backward
        return ce_forward_backward(
            to_np(inp["X"]), to_np(inp["W"]), to_np(inp["b"]), inp["target"].cpu().numpy(),
            inp["ignore_index"], inp["temperature"], inp["reduction"],
            compute_dW=inp["compute_dW"] if compute_dW is None else compute_dW,
            compute_db=inp["compute_db"] if compute_db is None else compute_db,
            dX_rows=dX_rows, dW_rows=dW_rows)
    lab = inp["shift_labels"]
    return oracle_fb(
        to_np(inp["X"]), to_np(inp["W"]), to_np(inp["b"]), to_np(inp["Q"]),
        None if lab is None else lab.numpy(), inp["ignore_index"], inp["temperature"],
        inp["eps"], inp["reduction"],
        compute_dW=inp["compute_dW"] if compute_dW is None else compute_dW,
        compute_db=inp["compute_db"] if compute_db is None else compute_db,
        dX_rows=dX_rows, dW_rows=dW_rows)


def assert_close(dtype: str, got: dict, ref: dict, dX_rows=None, dW_rows=None):
    tol = TOL[dtype]
    loss = float(got["loss"].cpu())
    rl = ref["loss"]
    assert np.isfinite(loss), loss
    assert abs(loss - rl) <= tol["loss_rel"] * abs(rl) + 1e-7, (loss, rl)
    for k, rows in (("dX", dX_rows), ("dW", dW_rows), ("db", None)):
        if ref.get(k) is None:
            assert got.get(k) is None, k
            continue
        g = got[k]
        if rows is not None:
            g = g[torch.as_tensor(rows, device=g.device)]
        g = to_np(g)
        e = ref[k]
        assert g.shape == e.shape, (k, g.shape, e.shape)
        assert np.all(np.isfinite(g)), k
        err = float(np.abs(g - e).max()) if e.size else 0.0
        scale = float(np.abs(e).max()) if e.size else 0.0
        bound = tol["grad_abs"] + tol["grad_rel_scale"] * scale
        assert err <= bound + 1e-30, (k, err, bound, scale)
