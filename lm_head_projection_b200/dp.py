"""Data-parallel fused linear KL-divergence / cross-entropy loss.

Rows of the batch are split over the ranks of a ``torch.distributed`` group
(NCCL on GPUs); every rank holds the whole head W, b.  The rows are
independent except for the divisor of the reduction and the parameter
gradients, so one step is:

1. count the kept rows of the local batch (CUDA library) and all-reduce the
   count (sum), so that every rank divides by the whole batch's kept rows;
2. run the fused loss on the local rows with that divisor (CUDA library);
3. all-reduce the loss, dW and db (sum).  dX needs no exchange: each rank's
   dX rows are the whole batch's dX rows for its shard.

With NCCL and a trained head, step 3 overlaps the call: the library records
an event as each vocabulary chunk's dW rows become final, and those rows are
all-reduced on a side stream while the later chunks run; the loss and db
follow once the call ends, and the caller's stream waits for the exchange.

The library itself runs no collective; the exchange is torch.distributed's.
Every rank takes the same collective steps in the same order.
"""

from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import (DTYPES, count_valid, cross_entropy_forward_backward, flkl_vocab_chunks,
               forward_backward)

__all__ = ["DataParallelFusedLinearLoss"]


class DataParallelFusedLinearLoss:
    """One data-parallel loss step per :meth:`step` call.

    ``kind`` "kl" (teacher distribution Q [BT, V] and optional shift labels)
    or "ce" (integer targets [BT], which are also the row mask).  Options are
    those of :func:`forward_backward` / :func:`cross_entropy_forward_backward`.
    ``group`` is the process group (default: the world).  Outputs are reused
    from step to step while the shapes and flags stay the same (``out`` and
    the workspace stay allocated), so a step's results are overwritten by
    the next step's.
    """

    def __init__(self, kind: str = "kl", group=None, ignore_index: int = -100,
                 temperature: float = 1.0, eps: float = 1e-10, reduction: str = "batchmean",
                 accum_fp32: bool = True):
        if kind not in ("kl", "ce"):
            raise ValueError("kind must be 'kl' or 'ce'")
        self.kind, self.group = kind, group
        self.ignore_index, self.temperature, self.eps = ignore_index, temperature, eps
        self.reduction, self.accum_fp32 = reduction, accum_fp32
        self.out: Optional[dict] = None
        self.workspace: Optional[torch.Tensor] = None

    # -- the three pieces (overridable, e.g. by tests of the exchange logic)
    def _count(self, mask_labels: Optional[torch.Tensor], BT: int, device) -> torch.Tensor:
        return count_valid(mask_labels, BT, self.ignore_index, device=device)

    def _reusable_out(self, X, W, b, compute_dW, compute_db) -> Optional[dict]:
        """The previous step's outputs when this step writes the same shapes,
        dtypes and gradients (else None, and the call allocates new ones): a
        short last batch, or a change of the flags, must not reuse buffers
        sized for another step."""
        key = (tuple(X.shape), tuple(W.shape), X.dtype, X.device, bool(compute_dW),
               bool(compute_db and b is not None), bool(self.accum_fp32))
        if key != getattr(self, "_out_key", None):
            self.out = None
            self._out_key = key
        return self.out

    def _local(self, X, W, b, teacher, labels, n_total, compute_dW, compute_db,
               chunk_events=None) -> dict:
        out = self._reusable_out(X, W, b, compute_dW, compute_db)
        common = dict(compute_dW=compute_dW, compute_db=compute_db, accum_fp32=self.accum_fp32,
                      out=out, workspace=self.workspace, n_valid_total=n_total)
        if chunk_events is not None:
            common["chunk_events"] = chunk_events
        if self.kind == "ce":
            r = cross_entropy_forward_backward(X, W, b, teacher, self.ignore_index,
                                               self.temperature, self.reduction, **common)
        else:
            r = forward_backward(X, W, b, teacher, labels, self.ignore_index, self.temperature,
                                 self.eps, self.reduction, **common)
        self.workspace = r.get("workspace", self.workspace)
        self.out = {k: r[k] for k in ("loss", "dX", "dW", "db")}
        return r

    def _all_reduce(self, tensors) -> None:
        for t in tensors:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)

    # -- one step
    def step(self, X: torch.Tensor, W: torch.Tensor, b: Optional[torch.Tensor],
             teacher: torch.Tensor, shift_labels: Optional[torch.Tensor] = None,
             compute_dW: bool = True, compute_db: bool = False) -> dict:
        """``teacher`` is Q for "kl" and the targets for "ce".  Returns the
        whole batch's loss, dW and db (identical on every rank) and this
        rank's dX rows."""
        mask = teacher if self.kind == "ce" else shift_labels
        n_total = self._count(mask, X.shape[0], X.device)
        self._all_reduce([n_total])
        bounds = self._overlap_bounds(X, W, compute_dW, compute_db)
        if not bounds:
            r = self._local(X, W, b, teacher, shift_labels, n_total, compute_dW, compute_db)
            self._all_reduce([r[k] for k in ("loss", "dW", "db") if r[k] is not None])
        else:
            r = self._overlapped(X, W, b, teacher, shift_labels, n_total, compute_dW,
                                 compute_db, bounds)
        return {"loss": r["loss"], "dX": r["dX"], "dW": r["dW"], "db": r["db"],
                "n_valid_total": n_total}

    # -- overlap of the dW exchange with the call (NCCL, trained head)
    def _overlap_bounds(self, X, W, compute_dW, compute_db) -> list:
        if not (compute_dW and X.is_cuda and dist.is_initialized()
                and dist.get_backend(self.group) == "nccl"):
            return []
        return flkl_vocab_chunks(X.shape[0], X.shape[1], W.shape[0], DTYPES[X.dtype],
                                 compute_dW, compute_db)

    def _overlapped(self, X, W, b, teacher, labels, n_total, compute_dW, compute_db,
                    bounds) -> dict:
        main = torch.cuda.current_stream(X.device)
        side = getattr(self, "_side", None)
        if side is None or side.device != X.device:
            side = self._side = torch.cuda.Stream(X.device)
        events = [torch.cuda.Event() for _ in range(len(bounds) - 1)]
        r = self._local(X, W, b, teacher, labels, n_total, compute_dW, compute_db,
                        chunk_events=events)
        done = torch.cuda.Event()
        done.record(main)
        with torch.cuda.stream(side):
            for c, ev in enumerate(events):
                side.wait_event(ev)
                self._all_reduce([r["dW"][bounds[c]:bounds[c + 1]]])
            side.wait_event(done)
            self._all_reduce([r[k] for k in ("loss", "db") if r[k] is not None])
        main.wait_stream(side)
        return r
