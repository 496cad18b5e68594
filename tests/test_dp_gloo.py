"""The data-parallel exchange of DataParallelFusedLinearLoss on 2 gloo ranks
(CPU): the kept-row count and the loss / dW / db are all-reduced so that each
rank's results equal the fp64 oracle on the whole batch (dX: the rank's own
rows).  The per-rank compute is the oracle here (the CUDA library needs a
GPU); the exchange logic under test is the module's own.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from lm_head_projection_b200.workloads import make_inputs, small_case
from oracle import ce_forward_backward, forward_backward


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _np(t):
    return None if t is None else t.detach().double().numpy()


def _make_oracle_loss(kind, reduction, V):
    from lm_head_projection_b200.dp import DataParallelFusedLinearLoss

    class OracleDP(DataParallelFusedLinearLoss):
        """Same exchange; the per-rank compute is the oracle with reduction
        "sum" divided by the whole batch's divisor."""

        def _count(self, mask, BT, device):
            if mask is None:
                return torch.tensor(BT, dtype=torch.int64)
            return (mask != self.ignore_index).sum().to(torch.int64)

        def _local(self, X, W, b, teacher, labels, n_total, compute_dW, compute_db):
            n = int(n_total)
            D = {"batchmean": n, "mean": n * V, "sum": 1}[self.reduction]
            if self.kind == "ce":
                r = ce_forward_backward(_np(X), _np(W), _np(b), teacher.numpy(),
                                        self.ignore_index, self.temperature, "sum",
                                        compute_dW=compute_dW, compute_db=compute_db)
            else:
                r = forward_backward(_np(X), _np(W), _np(b), _np(teacher),
                                     None if labels is None else labels.numpy(),
                                     self.ignore_index, self.temperature, self.eps, "sum",
                                     compute_dW=compute_dW, compute_db=compute_db)
            s = 1.0 / D if n > 0 else 0.0
            t = lambda a: None if a is None else torch.from_numpy(np.asarray(a) * s)
            return {"loss": torch.tensor(r["loss"] * s, dtype=torch.float64), "dX": t(r["dX"]),
                    "dW": t(r["dW"]), "db": t(r["db"])}

    return OracleDP(kind, reduction=reduction, temperature=1.5)


def _rank(rank, world, port, kind, reduction, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = small_case(dtype="fp32", BT=37, H=16, V=24, bias=True, reduction=reduction,
                       ignore_frac=0.3, temperature=1.5, ce=(kind == "ce"), seed=3)
        inp = make_inputs(w)
        rows = np.array_split(np.arange(w.BT), world)[rank]
        sl = lambda t: None if t is None else t[torch.as_tensor(rows)]
        teacher = inp["target"] if kind == "ce" else inp["Q"]
        loss = _make_oracle_loss(kind, reduction, w.V)
        r = loss.step(sl(inp["X"]), inp["W"], inp["b"], sl(teacher), sl(inp["shift_labels"]),
                      compute_dW=True, compute_db=True)
        q.put((rank, rows, float(r["loss"]), r["dX"].numpy(), r["dW"].numpy(),
               r["db"].numpy(), int(r["n_valid_total"])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["kl", "ce"])
@pytest.mark.parametrize("reduction", ["batchmean", "mean", "sum"])
def test_two_gloo_ranks_match_the_whole_batch(kind, reduction):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, kind, reduction, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = small_case(dtype="fp32", BT=37, H=16, V=24, bias=True, reduction=reduction,
                   ignore_frac=0.3, temperature=1.5, ce=(kind == "ce"), seed=3)
    inp = make_inputs(w)
    if kind == "ce":
        ref = ce_forward_backward(_np(inp["X"]), _np(inp["W"]), _np(inp["b"]),
                                  inp["target"].numpy(), inp["ignore_index"], 1.5, reduction,
                                  compute_dW=True, compute_db=True)
        kept = int((inp["target"] != inp["ignore_index"]).sum())
    else:
        ref = forward_backward(_np(inp["X"]), _np(inp["W"]), _np(inp["b"]), _np(inp["Q"]),
                               inp["shift_labels"].numpy(), inp["ignore_index"], 1.5, w.eps,
                               reduction, compute_dW=True, compute_db=True)
        kept = int((inp["shift_labels"] != inp["ignore_index"]).sum())
    for rank, rows, loss, dX, dW, db, n in res:
        assert n == kept
        assert abs(loss - ref["loss"]) <= 1e-12 * max(1.0, abs(ref["loss"]))
        np.testing.assert_allclose(dW, ref["dW"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(db, ref["db"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dX, ref["dX"][rows], rtol=0, atol=1e-12)
