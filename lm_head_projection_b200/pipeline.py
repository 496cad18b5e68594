"""Streaming host batches through the fused loss with copies overlapped.

A training loop that keeps its batches (hidden states X, teacher
distribution Q or targets, shift labels) in pinned host memory pays one
host-to-device copy per step.  ``BatchPipeline`` hides it: the copy of batch
i+1 runs on its own stream into the second of two device buffers while the
fused loss of batch i runs on the compute stream.  The head (W, b) stays on
the device.  Every computation still runs in the CUDA library; torch only
provides the buffers, streams and events.
"""

from __future__ import annotations

from typing import Optional, Sequence

import torch

from . import cross_entropy_forward_backward, forward_backward


class BatchPipeline:
    """Double-buffered host-to-device input pipeline around one loss.

    ``W``/``b`` are device tensors.  ``kind`` is "kl" (batches are
    ``(X, Q, shift_labels or None)``) or "ce" (batches are ``(X, target)``).
    ``options`` are the keyword arguments of :func:`forward_backward` /
    :func:`cross_entropy_forward_backward` (ignore_index, temperature, eps,
    reduction, compute_dW, compute_db, accum_fp32).

    ``submit(host_batch)`` enqueues the copy of a pinned host batch and the
    loss of the previously submitted batch; ``finish()`` runs the last one.
    The loss of step i is copied into slot i of a pinned host buffer of
    ``max_steps`` entries (``losses()`` after ``torch.cuda.synchronize()``).
    Outputs (dX, dW, db) are the device tensors of the most recent step.
    """

    def __init__(self, W: torch.Tensor, b: Optional[torch.Tensor], kind: str = "kl",
                 options: Optional[dict] = None, compute_stream=None, max_steps: int = 4096):
        if kind not in ("kl", "ce"):
            raise ValueError("kind must be 'kl' or 'ce'")
        self.W, self.b, self.kind = W, b, kind
        self.options = dict(options or {})
        self.dev = W.device
        self.compute = compute_stream or torch.cuda.current_stream(self.dev)
        self.copy = torch.cuda.Stream(self.dev)
        self.buffers: list = [None, None]
        self.copied = [torch.cuda.Event(), torch.cuda.Event()]
        self.consumed = [torch.cuda.Event(), torch.cuda.Event()]
        self.pending: Optional[int] = None
        self.n = 0
        self.out: Optional[dict] = None
        self.workspace: Optional[torch.Tensor] = None
        self.loss_host = torch.empty((max_steps,), dtype=torch.float32, pin_memory=True)
        self.done = 0

    def _device_like(self, hosts: Sequence[Optional[torch.Tensor]]):
        return [None if h is None else torch.empty(h.shape, dtype=h.dtype, device=self.dev)
                for h in hosts]

    def submit(self, host_batch: Sequence[Optional[torch.Tensor]]) -> None:
        slot = self.n % 2
        if self.buffers[slot] is None:
            self.buffers[slot] = self._device_like(host_batch)
        with torch.cuda.stream(self.copy):
            # the buffer was last read by the step two submissions ago
            self.copy.wait_event(self.consumed[slot])
            for d, h in zip(self.buffers[slot], host_batch):
                if d is not None:
                    d.copy_(h, non_blocking=True)
            self.copied[slot].record(self.copy)
        if self.pending is not None:
            self._run(self.pending)
        self.pending = slot
        self.n += 1

    def finish(self) -> None:
        if self.pending is not None:
            self._run(self.pending)
            self.pending = None

    def _run(self, slot: int) -> None:
        self.compute.wait_event(self.copied[slot])
        buf = self.buffers[slot]
        with torch.cuda.stream(self.compute):
            if self.kind == "ce":
                X, target = buf[0], buf[1]
                r = cross_entropy_forward_backward(X, self.W, self.b, target, out=self.out,
                                                   workspace=self.workspace,
                                                   stream=self.compute, **self.options)
            else:
                X, Q, labels = buf[0], buf[1], buf[2] if len(buf) > 2 else None
                r = forward_backward(X, self.W, self.b, Q, labels, out=self.out,
                                     workspace=self.workspace, stream=self.compute,
                                     **self.options)
            self.consumed[slot].record(self.compute)
            if self.done < self.loss_host.numel():
                self.loss_host[self.done].copy_(r["loss"], non_blocking=True)
        self.done += 1
        self.out = {k: r[k] for k in ("loss", "dX", "dW", "db")}
        self.workspace = r["workspace"]

    def losses(self) -> torch.Tensor:
        """Host losses of the completed steps (valid after a synchronize)."""
        return self.loss_host[:min(self.done, self.loss_host.numel())]
