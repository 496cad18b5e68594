"""Data-parallel form of the fused loss on one GPU: the kept-row count of the
CUDA library, the divisor taken from a whole-batch count (rows split in two
calls add up to the whole batch), and DataParallelFusedLinearLoss over a
one-rank NCCL group giving the direct call's bytes.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch

from lm_head_projection_b200.workloads import make_inputs, small_case
from parity_utils import TOL, assert_close, run_oracle

pytestmark = pytest.mark.gpu


def _call(pkg, g, rows=None, n_total=None):
    sl = (lambda t: t) if rows is None else (lambda t: None if t is None else t[rows])
    common = dict(compute_dW=True, compute_db=g["compute_db"], accum_fp32=True,
                  n_valid_total=n_total, check_status=True)
    if g.get("target") is not None:
        return pkg.cross_entropy_forward_backward(sl(g["X"]).contiguous(), g["W"], g["b"],
                                                  sl(g["target"]).contiguous(),
                                                  g["ignore_index"], g["temperature"],
                                                  g["reduction"], **common)
    lab = g["shift_labels"]
    return pkg.forward_backward(sl(g["X"]).contiguous(), g["W"], g["b"],
                                sl(g["Q"]).contiguous(),
                                None if lab is None else sl(lab).contiguous(), g["ignore_index"],
                                g["temperature"], g["eps"], g["reduction"], **common)


def test_count_valid():
    import lm_head_projection_b200 as pkg

    lab = torch.tensor([3, -100, 7, -100, -100, 0], dtype=torch.int64, device="cuda")
    assert int(pkg.count_valid(lab, 6)) == 3
    assert int(pkg.count_valid(None, 11, device="cuda")) == 11
    assert int(pkg.count_valid(lab[:0], 0)) == 0
    big = torch.full((100_000,), -100, dtype=torch.int64, device="cuda")
    big[::7] = 1
    assert int(pkg.count_valid(big, big.numel())) == int((big != -100).sum())


@pytest.mark.parametrize("dtype,reduction,ce", [("fp32", "batchmean", False),
                                               ("bf16", "mean", False),
                                               ("bf16", "sum", False),
                                               ("bf16", "batchmean", True),
                                               ("fp32", "mean", True)])
def test_split_rows_with_whole_batch_count_add_up(dtype, reduction, ce):
    import lm_head_projection_b200 as pkg

    w = small_case(dtype=dtype, BT=203, H=128 if dtype == "bf16" else 64, V=1000,
                   bias=True, reduction=reduction, ignore_frac=0.2, temperature=1.5, ce=ce,
                   seed=11)
    inp = make_inputs(w)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    whole = _call(pkg, g)
    mask = g["target"] if ce else g["shift_labels"]
    n_total = pkg.count_valid(mask, w.BT)
    halves = [torch.arange(0, 120, device="cuda"), torch.arange(120, w.BT, device="cuda")]
    parts = [_call(pkg, g, rows, n_total) for rows in halves]
    torch.cuda.synchronize()
    got = {"loss": parts[0]["loss"] + parts[1]["loss"],
           "dX": torch.cat([parts[0]["dX"], parts[1]["dX"]]),
           "dW": parts[0]["dW"] + parts[1]["dW"],
           "db": parts[0]["db"] + parts[1]["db"]}
    ref = run_oracle(inp, compute_dW=True, compute_db=True)
    assert_close(dtype, got, ref)
    # the split halves and the whole-batch call agree within the same bound
    assert_close(dtype, got, {k: (float(v.double().cpu()) if k == "loss" else
                                  v.double().cpu().numpy()) for k, v in whole.items()
                              if k in ("loss", "dX", "dW", "db")})


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("kind", ["kl", "ce"])
def test_one_rank_nccl_group_gives_the_direct_call(kind):
    import torch.distributed as dist

    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.dp import DataParallelFusedLinearLoss

    w = small_case(dtype="bf16", BT=300, H=256, V=2000, bias=True, ignore_frac=0.1,
                   ce=(kind == "ce"), seed=5)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
         for k, v in make_inputs(w).items()}
    direct = _call(pkg, g)
    torch.cuda.synchronize()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda:0"))
    try:
        loss = DataParallelFusedLinearLoss(kind, temperature=w.temperature, eps=w.eps)
        teacher = g["target"] if kind == "ce" else g["Q"]
        r = loss.step(g["X"], g["W"], g["b"], teacher, g["shift_labels"], compute_dW=True,
                      compute_db=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for k in ("loss", "dX", "dW", "db"):
        assert torch.equal(r[k], direct[k]), k


def test_steps_of_changing_batch_size_get_buffers_of_their_own_size():
    """A data-parallel loss object reused over steps of 96, 64 and 128 rows
    (a short batch, then a longer one) gives every step the direct call's
    bytes: outputs sized for another step are never reused."""
    import torch.distributed as dist

    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.dp import DataParallelFusedLinearLoss

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda:0"))
    try:
        loss = DataParallelFusedLinearLoss("kl", temperature=1.5)
        for i, (BT, flags) in enumerate([(96, (True, True)), (64, (True, True)),
                                         (128, (True, True)), (128, (False, True)),
                                         (128, (True, False))]):
            w = small_case(dtype="bf16", BT=BT, H=128, V=1000, bias=True, ignore_frac=0.1,
                           temperature=1.5, seed=30 + i)
            g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
                 for k, v in make_inputs(w).items()}
            cw, cb = flags
            r = loss.step(g["X"], g["W"], g["b"], g["Q"], g["shift_labels"], compute_dW=cw,
                          compute_db=cb)
            direct = pkg.forward_backward(g["X"], g["W"], g["b"], g["Q"], g["shift_labels"],
                                          g["ignore_index"], g["temperature"], g["eps"],
                                          g["reduction"], compute_dW=cw, compute_db=cb,
                                          accum_fp32=True, check_status=True)
            torch.cuda.synchronize()
            assert r["dX"].shape == (BT, 128)
            for k in ("loss", "dX", "dW", "db"):
                if direct[k] is None:
                    assert r[k] is None, k
                else:
                    assert torch.equal(r[k], direct[k]), (BT, k)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["kl", "ce"])
def test_chunk_events_and_overlapped_exchange_give_the_direct_call(kind):
    """The vocabulary chunks reported by the library tile [0, V); the call
    that records an event per chunk gives the plain call's bytes; and the
    one-rank NCCL step whose dW exchange runs chunk by chunk on a side stream
    (ordered by those events) gives the direct call's bytes."""
    import torch.distributed as dist

    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.dp import DataParallelFusedLinearLoss

    w = small_case(dtype="bf16", BT=300, H=256, V=4104, bias=True, ignore_frac=0.1,
                   ce=(kind == "ce"), seed=6)
    g = {k: (v.cuda() if isinstance(v, torch.Tensor) else v)
         for k, v in make_inputs(w).items()}
    bounds = pkg.flkl_vocab_chunks(w.BT, w.H, w.V, 1, True, True)
    assert bounds[0] == 0 and bounds[-1] == w.V and len(bounds) >= 3
    assert all(a < b for a, b in zip(bounds, bounds[1:]))
    assert pkg.flkl_vocab_chunks(0, w.H, w.V, 1, True, True) == []
    direct = _call(pkg, g)
    n_total = pkg.count_valid(g["target"] if kind == "ce" else g["shift_labels"], w.BT)
    events = [torch.cuda.Event() for _ in range(len(bounds) - 1)]
    common = dict(compute_dW=True, compute_db=True, accum_fp32=True, n_valid_total=n_total,
                  chunk_events=events, check_status=True)
    if kind == "ce":
        r = pkg.cross_entropy_forward_backward(g["X"], g["W"], g["b"], g["target"],
                                               g["ignore_index"], g["temperature"],
                                               g["reduction"], **common)
    else:
        r = pkg.forward_backward(g["X"], g["W"], g["b"], g["Q"], g["shift_labels"],
                                 g["ignore_index"], g["temperature"], g["eps"], g["reduction"],
                                 **common)
    torch.cuda.synchronize()
    for e in events:
        assert e.query()  # every chunk's event was recorded and has completed
    for k in ("loss", "dX", "dW", "db"):
        assert torch.equal(r[k], direct[k]), k
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda:0"))
    try:
        loss = DataParallelFusedLinearLoss(kind, temperature=w.temperature, eps=w.eps)
        assert loss._overlap_bounds(g["X"], g["W"], True, True) == bounds
        teacher = g["target"] if kind == "ce" else g["Q"]
        for _ in range(2):
            out = loss.step(g["X"], g["W"], g["b"], teacher, g["shift_labels"],
                            compute_dW=True, compute_db=True)
            torch.cuda.synchronize()
            for k in ("loss", "dX", "dW", "db"):
                assert torch.equal(out[k], direct[k]), k
    finally:
        dist.destroy_process_group()
