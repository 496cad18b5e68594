"""B200-native fused linear-head + KL-divergence loss (FusedLinearKLDivLoss).

Python binding of the C ABI in ``include/flkl.h``.  It only marshals
arguments: torch supplies device memory and the current stream, and every
step of the computation runs in the CUDA library ``_flkl.so`` built from
``csrc/`` (``python -m lm_head_projection_b200.build``).  There is no CPU or
PyTorch fallback: without the built library every call raises.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "FLKL_OK", "FlklError", "flkl_abi_version", "flkl_workspace_size", "flkl_forward_backward",
    "flkl_forward_backward_profiled", "LAUNCH_KINDS", "flkl_forward_backward_noalloc",
    "flkl_device_status", "flkl_set_wait_limit_ms", "flkl_wait_selftest", "flkl_status_string",
    "forward_backward", "FusedLinearKLDivLoss", "library_path", "REDUCTIONS",
    "flkl_ce_forward_backward", "cross_entropy_forward_backward", "FusedLinearCrossEntropyLoss",
    "flkl_norm_workspace_size", "flkl_rms_norm_backward", "flkl_layer_norm_backward",
    "flkl_norm_device_status", "flkl_count_valid", "flkl_forward_backward_dp",
    "flkl_ce_forward_backward_dp", "count_valid", "flkl_selective_logprob_forward",
    "flkl_selective_logprob_backward", "selective_logprob", "SelectiveLogProb",
    "flkl_jsd_workspace_size", "flkl_jsd_forward_backward", "jsd_forward_backward",
    "FusedLinearJSDLoss", "flkl_scale_cast", "flkl_clock_trace", "flkl_gemm_ctas", "flkl_vocab_chunks",
    "flkl_forward_backward_dp_events", "flkl_ce_forward_backward_dp_events",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "_flkl.so")
_LIB = None

FLKL_OK = 0
REDUCTIONS = {"batchmean": 0, "mean": 1, "sum": 2, "none": 3}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}


class FlklError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {flkl_status_string(status)} (status {status})")


def library_path() -> str:
    return _LIB_PATH


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"CUDA library {_LIB_PATH} is not built; run "
                "`python -m lm_head_projection_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(_LIB_PATH)
        c = ctypes
        lib.flkl_abi_version.restype = c.c_int
        lib.flkl_abi_version.argtypes = []
        lib.flkl_workspace_size.restype = c.c_size_t
        lib.flkl_workspace_size.argtypes = [c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_int,
                                            c.c_int]
        lib.flkl_forward_backward.restype = c.c_int
        lib.flkl_forward_backward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,      # X W b Q
            c.c_void_p, c.c_int64,                               # labels ignore_index
            c.c_int64, c.c_int64, c.c_int64, c.c_int,            # BT H V dtype
            c.c_float, c.c_float, c.c_int,                       # T eps reduction
            c.c_int, c.c_int, c.c_int,                           # dW db accum_fp32
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,      # loss dX dW db
            c.c_void_p, c.c_size_t, c.c_void_p]                  # ws bytes stream
        lib.flkl_forward_backward_profiled.restype = c.c_int
        lib.flkl_forward_backward_profiled.argtypes = list(lib.flkl_forward_backward.argtypes) + [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_int, c.c_void_p, c.c_void_p]
        lib.flkl_ce_forward_backward.restype = c.c_int
        lib.flkl_ce_forward_backward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p,                  # X W b
            c.c_void_p, c.c_int64,                               # target ignore_index
            c.c_int64, c.c_int64, c.c_int64, c.c_int,            # BT H V dtype
            c.c_float, c.c_int,                                  # T reduction
            c.c_int, c.c_int, c.c_int,                           # dW db accum_fp32
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,      # loss dX dW db
            c.c_void_p, c.c_size_t, c.c_void_p]                  # ws bytes stream
        lib.flkl_forward_backward_dp.restype = c.c_int
        lib.flkl_forward_backward_dp.argtypes = list(lib.flkl_forward_backward.argtypes) + [
            c.c_void_p]
        lib.flkl_ce_forward_backward_dp.restype = c.c_int
        lib.flkl_ce_forward_backward_dp.argtypes = list(
            lib.flkl_ce_forward_backward.argtypes) + [c.c_void_p]
        lib.flkl_selective_logprob_forward.restype = c.c_int
        lib.flkl_selective_logprob_forward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64, c.c_int64, c.c_int64,
            c.c_int64, c.c_int, c.c_float, c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_size_t,
            c.c_void_p]
        lib.flkl_selective_logprob_backward.restype = c.c_int
        lib.flkl_selective_logprob_backward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64, c.c_int64, c.c_int64,
            c.c_int64, c.c_int, c.c_float, c.c_void_p, c.c_int, c.c_int, c.c_int, c.c_void_p,
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_size_t, c.c_void_p]
        lib.flkl_jsd_workspace_size.restype = c.c_size_t
        lib.flkl_jsd_workspace_size.argtypes = [c.c_int64, c.c_int64, c.c_int64, c.c_int64,
                                                c.c_int, c.c_int, c.c_int]
        lib.flkl_jsd_forward_backward.restype = c.c_int
        lib.flkl_jsd_forward_backward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
            c.c_int64, c.c_int64, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_float,
            c.c_float, c.c_int, c.c_int, c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_void_p,
            c.c_void_p, c.c_void_p, c.c_size_t, c.c_void_p]
        lib.flkl_scale_cast.restype = c.c_int
        lib.flkl_scale_cast.argtypes = [c.c_void_p, c.c_int, c.c_void_p, c.c_int, c.c_int64,
                                        c.c_void_p, c.c_void_p]
        lib.flkl_gemm_ctas.restype = c.c_int
        lib.flkl_gemm_ctas.argtypes = []
        lib.flkl_clock_trace.restype = c.c_int
        lib.flkl_clock_trace.argtypes = [c.c_void_p, c.c_int, c.c_uint, c.c_void_p]
        lib.flkl_vocab_chunks.restype = c.c_int
        lib.flkl_vocab_chunks.argtypes = [c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_int,
                                          c.c_int, c.c_void_p, c.c_int]
        lib.flkl_forward_backward_dp_events.restype = c.c_int
        lib.flkl_forward_backward_dp_events.argtypes = list(
            lib.flkl_forward_backward.argtypes) + [c.c_void_p, c.c_void_p, c.c_int]
        lib.flkl_ce_forward_backward_dp_events.restype = c.c_int
        lib.flkl_ce_forward_backward_dp_events.argtypes = list(
            lib.flkl_ce_forward_backward.argtypes) + [c.c_void_p, c.c_void_p, c.c_int]
        lib.flkl_count_valid.restype = c.c_int
        lib.flkl_count_valid.argtypes = [c.c_void_p, c.c_int64, c.c_int64, c.c_void_p, c.c_void_p]
        lib.flkl_forward_backward_noalloc.restype = c.c_int
        lib.flkl_forward_backward_noalloc.argtypes = (
            list(lib.flkl_forward_backward.argtypes[:20]) + [c.c_void_p])
        lib.flkl_device_status.restype = c.c_int
        lib.flkl_device_status.argtypes = [c.c_void_p, c.c_void_p]
        lib.flkl_set_wait_limit_ms.restype = None
        lib.flkl_set_wait_limit_ms.argtypes = [c.c_uint]
        lib.flkl_wait_selftest.restype = c.c_int
        lib.flkl_wait_selftest.argtypes = [c.c_void_p, c.c_uint, c.c_void_p]
        lib.flkl_status_string.restype = c.c_char_p
        lib.flkl_status_string.argtypes = [c.c_int]
        lib.flkl_norm_workspace_size.restype = c.c_size_t
        lib.flkl_norm_workspace_size.argtypes = [c.c_int64, c.c_int64, c.c_int, c.c_int]
        lib.flkl_rms_norm_backward.restype = c.c_int
        lib.flkl_rms_norm_backward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64, c.c_int64, c.c_int, c.c_float,
            c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_void_p, c.c_size_t, c.c_void_p]
        lib.flkl_norm_device_status.restype = c.c_int
        lib.flkl_norm_device_status.argtypes = [c.c_void_p]
        lib.flkl_layer_norm_backward.restype = c.c_int
        lib.flkl_layer_norm_backward.argtypes = [
            c.c_void_p, c.c_void_p, c.c_void_p, c.c_int64, c.c_int64, c.c_int, c.c_float,
            c.c_int, c.c_int, c.c_int, c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
            c.c_size_t, c.c_void_p]
        _LIB = lib
    return _LIB


# ------------------------------------------------------------------ raw C ABI

def flkl_abi_version() -> int:
    return _lib().flkl_abi_version()


def flkl_status_string(status: int) -> str:
    return _lib().flkl_status_string(int(status)).decode()


def flkl_workspace_size(BT, H, V, dtype, compute_dW, compute_db) -> int:
    return _lib().flkl_workspace_size(int(BT), int(H), int(V), int(dtype), int(bool(compute_dW)),
                                      int(bool(compute_db)))


def flkl_forward_backward(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype, temperature,
                          eps, reduction, compute_dW, compute_db, accum_fp32, loss, dX, dW, db,
                          workspace, workspace_bytes, stream) -> int:
    """The C entry point with raw integer pointers (0 = NULL); returns the status."""
    return _lib().flkl_forward_backward(
        X, W, b, Q, shift_labels, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), float(eps), int(reduction), int(bool(compute_dW)),
        int(bool(compute_db)), int(bool(accum_fp32)), loss, dX, dW, db, workspace,
        int(workspace_bytes), stream)


def flkl_ce_forward_backward(X, W, b, target, ignore_index, BT, H, V, dtype, temperature,
                             reduction, compute_dW, compute_db, accum_fp32, loss, dX, dW, db,
                             workspace, workspace_bytes, stream) -> int:
    """The cross-entropy C entry point (one-hot teacher at target[r]) with raw
    integer pointers; returns the status."""
    return _lib().flkl_ce_forward_backward(
        X, W, b, target, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), int(reduction), int(bool(compute_dW)), int(bool(compute_db)),
        int(bool(accum_fp32)), loss, dX, dW, db, workspace, int(workspace_bytes), stream)


def flkl_count_valid(labels, BT, ignore_index, count, stream) -> int:
    """Kept rows of a batch into the device int64 at ``count``; returns the status."""
    return _lib().flkl_count_valid(labels, int(BT), int(ignore_index), count, stream)


def flkl_forward_backward_dp(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                             temperature, eps, reduction, compute_dW, compute_db, accum_fp32, loss,
                             dX, dW, db, workspace, workspace_bytes, stream,
                             n_valid_total) -> int:
    """flkl_forward_backward with the divisor taken from the device int64 at
    ``n_valid_total`` (the kept rows of every rank's batch)."""
    return _lib().flkl_forward_backward_dp(
        X, W, b, Q, shift_labels, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), float(eps), int(reduction), int(bool(compute_dW)),
        int(bool(compute_db)), int(bool(accum_fp32)), loss, dX, dW, db, workspace,
        int(workspace_bytes), stream, n_valid_total)


def flkl_ce_forward_backward_dp(X, W, b, target, ignore_index, BT, H, V, dtype, temperature,
                                reduction, compute_dW, compute_db, accum_fp32, loss, dX, dW, db,
                                workspace, workspace_bytes, stream, n_valid_total) -> int:
    """flkl_ce_forward_backward with the divisor from ``n_valid_total``."""
    return _lib().flkl_ce_forward_backward_dp(
        X, W, b, target, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), int(reduction), int(bool(compute_dW)), int(bool(compute_db)),
        int(bool(accum_fp32)), loss, dX, dW, db, workspace, int(workspace_bytes), stream,
        n_valid_total)


def flkl_selective_logprob_forward(X, W, b, target, ignore_index, BT, H, V, dtype, temperature,
                                   compute_dW, compute_db, logp, workspace, workspace_bytes,
                                   stream) -> int:
    """Per-row target log-probabilities (raw pointers); returns the status."""
    return _lib().flkl_selective_logprob_forward(
        X, W, b, target, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), int(bool(compute_dW)), int(bool(compute_db)), logp, workspace,
        int(workspace_bytes), stream)


def flkl_selective_logprob_backward(X, W, b, target, ignore_index, BT, H, V, dtype, temperature,
                                    dlogp, compute_dW, compute_db, accum_fp32, dX, dW, db,
                                    workspace, workspace_bytes, stream) -> int:
    """Gradients for upstream per-row gradients ``dlogp`` (raw pointers)."""
    return _lib().flkl_selective_logprob_backward(
        X, W, b, target, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), dlogp, int(bool(compute_dW)), int(bool(compute_db)),
        int(bool(accum_fp32)), dX, dW, db, workspace, int(workspace_bytes), stream)


def flkl_jsd_workspace_size(BT, H, Ht, V, dtype, compute_dW, compute_db) -> int:
    return _lib().flkl_jsd_workspace_size(int(BT), int(H), int(Ht), int(V), int(dtype),
                                          int(bool(compute_dW)), int(bool(compute_db)))


def flkl_jsd_forward_backward(X, W, b, Xt, Wt, bt, shift_labels, ignore_index, BT, H, Ht, V,
                              dtype, temperature, beta, reduction, compute_dW, compute_db,
                              accum_fp32, loss, dX, dW, db, workspace, workspace_bytes,
                              stream) -> int:
    """The fused linear JSD entry point with raw pointers; returns the status."""
    return _lib().flkl_jsd_forward_backward(
        X, W, b, Xt, Wt, bt, shift_labels, int(ignore_index), int(BT), int(H), int(Ht), int(V),
        int(dtype), float(temperature), float(beta), int(reduction), int(bool(compute_dW)),
        int(bool(compute_db)), int(bool(accum_fp32)), loss, dX, dW, db, workspace,
        int(workspace_bytes), stream)


def flkl_norm_workspace_size(rows, H, compute_dW, compute_db) -> int:
    return _lib().flkl_norm_workspace_size(int(rows), int(H), int(bool(compute_dW)),
                                           int(bool(compute_db)))


def flkl_rms_norm_backward(dY, X, W, rows, H, dtype, eps, compute_dW, accum_fp32, dX, dW,
                           workspace, workspace_bytes, stream) -> int:
    """The RMSNorm-backward C entry point with raw pointers; returns the status."""
    return _lib().flkl_rms_norm_backward(
        dY, X, W, int(rows), int(H), int(dtype), float(eps), int(bool(compute_dW)),
        int(bool(accum_fp32)), dX, dW, workspace, int(workspace_bytes), stream)


def flkl_layer_norm_backward(dY, X, W, rows, H, dtype, eps, compute_dW, compute_db, accum_fp32,
                             dX, dW, db, workspace, workspace_bytes, stream) -> int:
    """The LayerNorm-backward C entry point with raw pointers; returns the status."""
    return _lib().flkl_layer_norm_backward(
        dY, X, W, int(rows), int(H), int(dtype), float(eps), int(bool(compute_dW)),
        int(bool(compute_db)), int(bool(accum_fp32)), dX, dW, db, workspace,
        int(workspace_bytes), stream)


def flkl_norm_device_status(stream=None) -> int:
    """Synchronise ``stream``; status of the norm kernels since the last call."""
    return _lib().flkl_norm_device_status(stream)


def flkl_forward_backward_noalloc(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                                  temperature, eps, reduction, compute_dW, compute_db, accum_fp32,
                                  loss, dX, dW, db, stream) -> int:
    """The allocation-free C entry point (raw pointers, no workspace): it
    uses the library's fixed 128 MiB device scratch, for callers that cannot
    allocate device memory.  Returns the status (6 = sizes too large)."""
    return _lib().flkl_forward_backward_noalloc(
        X, W, b, Q, shift_labels, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), float(eps), int(reduction), int(bool(compute_dW)),
        int(bool(compute_db)), int(bool(accum_fp32)), loss, dX, dW, db, stream)


LAUNCH_KINDS = ("prepare", "stats", "combine", "loss", "grad", "dW", "dX", "db", "zero",
                "chunk")


def flkl_forward_backward_profiled(X, W, b, Q, shift_labels, ignore_index, BT, H, V, dtype,
                                   temperature, eps, reduction, compute_dW, compute_db,
                                   accum_fp32, loss, dX, dW, db, workspace, workspace_bytes,
                                   stream, events, capacity, ce_target=None):
    """The profiled C entry point.  ``events`` is a list of 2*capacity
    torch.cuda.Event(enable_timing=True), each recorded once beforehand (torch
    creates the CUDA event lazily).  Returns (status, kinds, flops, n) with the
    launch kind and GEMM FLOPs of each recorded launch and the launch count."""
    c = ctypes
    ev = (c.c_void_p * (2 * capacity))(*[e.cuda_event for e in events[:2 * capacity]])
    kinds = (c.c_int * max(capacity, 1))()
    flops = (c.c_double * max(capacity, 1))()
    n = c.c_int(0)
    st = _lib().flkl_forward_backward_profiled(
        X, W, b, Q, shift_labels, int(ignore_index), int(BT), int(H), int(V), int(dtype),
        float(temperature), float(eps), int(reduction), int(bool(compute_dW)),
        int(bool(compute_db)), int(bool(accum_fp32)), loss, dX, dW, db, workspace,
        int(workspace_bytes), stream, ev, kinds, flops, int(capacity), c.byref(n), ce_target)
    k = min(n.value, capacity)
    return st, [kinds[i] for i in range(k)], [flops[i] for i in range(k)], n.value


def flkl_scale_cast(src, src_dtype, dst, dst_dtype, n, scale, stream=None) -> int:
    return _lib().flkl_scale_cast(src, int(src_dtype), dst, int(dst_dtype), int(n), scale,
                                  stream)


def flkl_gemm_ctas() -> int:
    return _lib().flkl_gemm_ctas()


def flkl_clock_trace(out_ptr, n_samples, interval_ns, stream=None) -> int:
    return _lib().flkl_clock_trace(out_ptr, int(n_samples), int(interval_ns), stream)


def flkl_vocab_chunks(BT, H, V, dtype, compute_dW, compute_db) -> list:
    """Row bounds of the vocabulary chunks of a call: [b0=0, b1, ..., bn=V]
    (chunk c covers dW rows [b_c, b_{c+1})); [] for BT = 0."""
    n = _lib().flkl_vocab_chunks(int(BT), int(H), int(V), int(dtype), int(bool(compute_dW)),
                                 int(bool(compute_db)), None, 0)
    if n <= 0:
        return []
    b = (ctypes.c_int64 * (n + 1))()
    _lib().flkl_vocab_chunks(int(BT), int(H), int(V), int(dtype), int(bool(compute_dW)),
                             int(bool(compute_db)), b, n)
    return [int(b[i]) for i in range(n + 1)]


def _event_array(events):
    """cudaEvent_t handles of torch.cuda.Event objects; torch creates the CUDA
    event on its first record, so an event never recorded is recorded once
    here (on the current stream) first."""
    for e in events:
        if not e.cuda_event:
            e.record()
    return (ctypes.c_void_p * max(1, len(events)))(*[e.cuda_event for e in events])


def flkl_forward_backward_dp_events(*args_and_events):
    """flkl_forward_backward_dp's arguments, then n_valid_total, then a list of
    recorded-once torch.cuda.Event (chunk_done[c])."""
    *args, n_total, events = args_and_events
    return _lib().flkl_forward_backward_dp_events(*args, n_total, _event_array(events),
                                                  len(events))


def flkl_ce_forward_backward_dp_events(*args_and_events):
    *args, n_total, events = args_and_events
    return _lib().flkl_ce_forward_backward_dp_events(*args, n_total, _event_array(events),
                                                     len(events))


def flkl_device_status(workspace_ptr, stream=None) -> int:
    return _lib().flkl_device_status(workspace_ptr, stream)


def flkl_set_wait_limit_ms(ms: int) -> None:
    _lib().flkl_set_wait_limit_ms(int(ms))


def flkl_wait_selftest(status_ptr, limit_ms, stream=None) -> int:
    return _lib().flkl_wait_selftest(status_ptr, int(limit_ms), stream)


# ------------------------------------------------------------------ torch-facing wrapper

def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _check_dev(name, t, dtype, shape, device):
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _outputs(out: Optional[dict], dev, BT: int, H: int, V: int, dt, pdt, compute_dW: bool,
             compute_db: bool) -> tuple:
    """loss, dX, dW, db for one call: each caller-supplied tensor of ``out``
    is checked against the shape, dtype and device this call writes (the
    kernels write BT*H, V*H and V elements, so a smaller buffer would be
    written past its end); missing ones are allocated."""
    out = {} if out is None else out
    specs = {"loss": (torch.float32, ()), "dX": (dt, (BT, H)),
             "dW": (pdt, (V, H)) if compute_dW else None,
             "db": (pdt, (V,)) if compute_db else None}
    res = []
    for name, spec in specs.items():
        if spec is None:
            res.append(None)
            continue
        t = out.get(name)
        if t is None:
            t = torch.empty(spec[1], dtype=spec[0], device=dev)
        else:
            _check_dev(f"out[{name!r}]", t, spec[0], spec[1], dev)
        res.append(t)
    return tuple(res)


def _workspace(workspace: Optional[torch.Tensor], need: int, dev) -> torch.Tensor:
    """The caller's workspace when it is a large enough contiguous uint8
    buffer on ``dev``, else a new one."""
    if workspace is not None:
        if workspace.device != dev or workspace.dtype != torch.uint8 or \
                not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous uint8 tensor on " + str(dev))
        if workspace.numel() >= need:
            return workspace
    return torch.empty(need, dtype=torch.uint8, device=dev)


def _scaled(t: Optional[torch.Tensor], grad_out: torch.Tensor, dtype) -> Optional[torch.Tensor]:
    """``t * grad_out`` in ``dtype`` as a new tensor, by the CUDA library:
    the incoming gradient is read on the device (no host synchronisation)
    and the product is skipped when it is 1."""
    if t is None:
        return None
    out = torch.empty(t.shape, dtype=dtype, device=t.device)
    g = grad_out.detach().to(device=t.device, dtype=torch.float32).reshape(()).contiguous()
    st = torch.cuda.current_stream(t.device)
    s = flkl_scale_cast(_ptr(t), DTYPES[t.dtype], _ptr(out), DTYPES[dtype], t.numel(), _ptr(g),
                        st.cuda_stream)
    if s != FLKL_OK:
        raise FlklError(s, "flkl_scale_cast")
    return out


def forward_backward(X: torch.Tensor, W: torch.Tensor, b: Optional[torch.Tensor], Q: torch.Tensor,
                     shift_labels: Optional[torch.Tensor] = None, ignore_index: int = -100,
                     temperature: float = 1.0, eps: float = 1e-10, reduction: str = "batchmean",
                     compute_dW: bool = True, compute_db: bool = False, accum_fp32: bool = True,
                     out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None, check_status: bool = False,
                     n_valid_total: Optional[torch.Tensor] = None,
                     chunk_events: Optional[list] = None) -> dict:
    """Loss and gradients in one call on the current CUDA stream.

    Allocates outputs (and the workspace) with torch unless given in ``out`` /
    ``workspace``; returns ``{"loss", "dX", "dW", "db"}`` (None for the ones
    not asked for).  Raises FlklError on a non-OK status.  ``n_valid_total``
    (a device int64 scalar) replaces the batch's kept-row count in the
    divisor: the data-parallel form (see :mod:`.dp`); with it,
    ``chunk_events`` (torch.cuda.Event, one per vocabulary chunk, see
    :func:`flkl_vocab_chunks`) are recorded as each chunk's dW rows become
    final.
    """
    if reduction not in REDUCTIONS:
        raise ValueError(f"unknown reduction {reduction!r}")
    if X.dtype not in DTYPES:
        raise ValueError(f"dtype {X.dtype} not supported (float32 or bfloat16)")
    dev = X.device
    BT, H = X.shape
    V = W.shape[0]
    dt = X.dtype
    _check_dev("X", X, dt, (BT, H), dev)
    _check_dev("W", W, dt, (V, H), dev)
    _check_dev("Q", Q, dt, (BT, V), dev)
    if b is not None:
        _check_dev("b", b, dt, (V,), dev)
    if shift_labels is not None:
        _check_dev("shift_labels", shift_labels, torch.int64, (BT,), dev)
    compute_db = bool(compute_db and b is not None)
    pdt = torch.float32 if (accum_fp32 or dt == torch.float32) else dt
    loss, dX, dW, db = _outputs(out, dev, BT, H, V, dt, pdt, compute_dW, compute_db)
    need = flkl_workspace_size(BT, H, V, DTYPES[dt], compute_dW, compute_db)
    if need == 0:
        raise FlklError(1, "flkl_workspace_size")
    workspace = _workspace(workspace, need, dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    args = (_ptr(X), _ptr(W), _ptr(b), _ptr(Q), _ptr(shift_labels), ignore_index, BT, H, V,
            DTYPES[dt], temperature, eps, REDUCTIONS[reduction], compute_dW, compute_db,
            accum_fp32, _ptr(loss), _ptr(dX), _ptr(dW), _ptr(db), _ptr(workspace),
            workspace.numel(), st.cuda_stream)
    if n_valid_total is not None:
        _check_dev("n_valid_total", n_valid_total, torch.int64, (), dev)
        if chunk_events is not None:
            status = flkl_forward_backward_dp_events(*args, _ptr(n_valid_total), chunk_events)
        else:
            status = flkl_forward_backward_dp(*args, _ptr(n_valid_total))
    else:
        status = flkl_forward_backward(*args)
    if status != FLKL_OK:
        raise FlklError(status, "flkl_forward_backward")
    if check_status:
        s = flkl_device_status(_ptr(workspace), st.cuda_stream)
        if s != FLKL_OK:
            raise FlklError(s, "flkl_forward_backward (device)")
    return {"loss": loss, "dX": dX, "dW": dW, "db": db, "workspace": workspace}


class _FusedLinearKLDivFunction(torch.autograd.Function):
    """Gradient-in-forward: the forward call produces every gradient; the
    backward only scales them by the incoming gradient of the loss."""

    @staticmethod
    def forward(ctx, X, W, b, Q, shift_labels, ignore_index, temperature, eps, reduction,
                accum_fp32):
        need_dW = ctx.needs_input_grad[1]
        need_db = b is not None and ctx.needs_input_grad[2]
        r = forward_backward(X.contiguous(), W.contiguous(),
                             None if b is None else b.contiguous(), Q.contiguous(),
                             shift_labels, ignore_index, temperature, eps, reduction,
                             compute_dW=need_dW, compute_db=need_db, accum_fp32=accum_fp32)
        ctx.save_for_backward(r["dX"], r["dW"], r["db"])
        ctx.w_dtype = W.dtype
        return r["loss"]

    @staticmethod
    def backward(ctx, grad_out):
        dX, dW, db = ctx.saved_tensors
        # one pass each: scale by the incoming gradient and cast to the
        # parameter dtype, on the device
        dX = _scaled(dX, grad_out, dX.dtype)
        dW = _scaled(dW, grad_out, ctx.w_dtype)
        db = _scaled(db, grad_out, ctx.w_dtype)
        return dX, dW, db, None, None, None, None, None, None, None


class FusedLinearKLDivLoss(torch.nn.Module):
    """Module form with the options of the pull-request page (*Details*):
    ``reduction`` ("batchmean" / "mean" / "sum"; "none" is refused),
    ``ignore_index`` applied through ``shift_labels``, ``temperature``, ``eps``
    and ``accum_dtype`` (torch.float32 keeps the head gradient in fp32).

    ``forward(lin_weight, _input, target_probs, bias=None, shift_labels=None)``
    """

    def __init__(self, ignore_index: int = -100, reduction: str = "batchmean",
                 temperature: float = 1.0, eps: float = 1e-10,
                 accum_dtype: Optional[torch.dtype] = None):
        super().__init__()
        if reduction == "none":
            raise ValueError("reduction='none' is not supported: the gradient is computed with "
                             "the loss and needs a scalar loss; use an element-wise KL loss")
        if reduction not in ("batchmean", "mean", "sum"):
            raise ValueError(f"unknown reduction {reduction!r}")
        self.ignore_index = ignore_index
        self.reduction = reduction
        self.temperature = temperature
        self.eps = eps
        self.accum_fp32 = accum_dtype == torch.float32

    def forward(self, lin_weight, _input, target_probs, bias=None, shift_labels=None):
        return _FusedLinearKLDivFunction.apply(_input, lin_weight, bias, target_probs,
                                               shift_labels, self.ignore_index, self.temperature,
                                               self.eps, self.reduction, self.accum_fp32)


def cross_entropy_forward_backward(X: torch.Tensor, W: torch.Tensor, b: Optional[torch.Tensor],
                                   target: torch.Tensor, ignore_index: int = -100,
                                   temperature: float = 1.0, reduction: str = "batchmean",
                                   compute_dW: bool = True, compute_db: bool = False,
                                   accum_fp32: bool = True, out: Optional[dict] = None,
                                   workspace: Optional[torch.Tensor] = None,
                                   stream: Optional[torch.cuda.Stream] = None,
                                   check_status: bool = False,
                                   n_valid_total: Optional[torch.Tensor] = None,
                                   chunk_events: Optional[list] = None) -> dict:
    """Fused linear + cross-entropy (one-hot teacher at ``target``) in one call.
    ``reduction="batchmean"`` divides by the kept rows (torch's cross_entropy
    "mean").  Same outputs and conventions as :func:`forward_backward`."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"unknown reduction {reduction!r}")
    if X.dtype not in DTYPES:
        raise ValueError(f"dtype {X.dtype} not supported (float32 or bfloat16)")
    dev = X.device
    BT, H = X.shape
    V = W.shape[0]
    dt = X.dtype
    _check_dev("X", X, dt, (BT, H), dev)
    _check_dev("W", W, dt, (V, H), dev)
    _check_dev("target", target, torch.int64, (BT,), dev)
    if b is not None:
        _check_dev("b", b, dt, (V,), dev)
    compute_db = bool(compute_db and b is not None)
    pdt = torch.float32 if (accum_fp32 or dt == torch.float32) else dt
    loss, dX, dW, db = _outputs(out, dev, BT, H, V, dt, pdt, compute_dW, compute_db)
    need = flkl_workspace_size(BT, H, V, DTYPES[dt], compute_dW, compute_db)
    if need == 0:
        raise FlklError(1, "flkl_workspace_size")
    workspace = _workspace(workspace, need, dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    args = (_ptr(X), _ptr(W), _ptr(b), _ptr(target), ignore_index, BT, H, V, DTYPES[dt],
            temperature, REDUCTIONS[reduction], compute_dW, compute_db, accum_fp32, _ptr(loss),
            _ptr(dX), _ptr(dW), _ptr(db), _ptr(workspace), workspace.numel(), st.cuda_stream)
    if n_valid_total is not None:
        _check_dev("n_valid_total", n_valid_total, torch.int64, (), dev)
        if chunk_events is not None:
            status = flkl_ce_forward_backward_dp_events(*args, _ptr(n_valid_total),
                                                        chunk_events)
        else:
            status = flkl_ce_forward_backward_dp(*args, _ptr(n_valid_total))
    else:
        status = flkl_ce_forward_backward(*args)
    if status != FLKL_OK:
        raise FlklError(status, "flkl_ce_forward_backward")
    if check_status:
        s = flkl_device_status(_ptr(workspace), st.cuda_stream)
        if s != FLKL_OK:
            raise FlklError(s, "flkl_ce_forward_backward (device)")
    return {"loss": loss, "dX": dX, "dW": dW, "db": db, "workspace": workspace}


def jsd_forward_backward(X: torch.Tensor, W: torch.Tensor, b: Optional[torch.Tensor],
                         Xt: torch.Tensor, Wt: torch.Tensor, bt: Optional[torch.Tensor] = None,
                         shift_labels: Optional[torch.Tensor] = None, ignore_index: int = -100,
                         temperature: float = 1.0, beta: float = 0.5,
                         reduction: str = "batchmean", compute_dW: bool = True,
                         compute_db: bool = False, accum_fp32: bool = True,
                         workspace: Optional[torch.Tensor] = None,
                         stream: Optional[torch.cuda.Stream] = None,
                         check_status: bool = False) -> dict:
    """Fused linear Jensen-Shannon divergence between the student head
    (X, W, b) and the teacher head (Xt, Wt, bt) in one call: the generalized
    JSD with weight ``beta`` (M = beta P + (1 - beta) Q), loss and student
    gradients; returns ``{"loss", "dX", "dW", "db", "workspace"}``."""
    if reduction not in REDUCTIONS:
        raise ValueError(f"unknown reduction {reduction!r}")
    if X.dtype not in DTYPES:
        raise ValueError(f"dtype {X.dtype} not supported (float32 or bfloat16)")
    dev, dt = X.device, X.dtype
    BT, H = X.shape
    V = W.shape[0]
    Ht = Xt.shape[1]
    _check_dev("X", X, dt, (BT, H), dev)
    _check_dev("W", W, dt, (V, H), dev)
    _check_dev("Xt", Xt, dt, (BT, Ht), dev)
    _check_dev("Wt", Wt, dt, (V, Ht), dev)
    if b is not None:
        _check_dev("b", b, dt, (V,), dev)
    if bt is not None:
        _check_dev("bt", bt, dt, (V,), dev)
    if shift_labels is not None:
        _check_dev("shift_labels", shift_labels, torch.int64, (BT,), dev)
    compute_db = bool(compute_db and b is not None)
    pdt = torch.float32 if (accum_fp32 or dt == torch.float32) else dt
    loss = torch.empty((), dtype=torch.float32, device=dev)
    dX = torch.empty_like(X)
    dW = torch.empty((V, H), dtype=pdt, device=dev) if compute_dW else None
    db = torch.empty((V,), dtype=pdt, device=dev) if compute_db else None
    need = flkl_jsd_workspace_size(BT, H, Ht, V, DTYPES[dt], compute_dW, compute_db)
    if need == 0:
        raise FlklError(1, "flkl_jsd_workspace_size")
    workspace = _workspace(workspace, need, dev)
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    status = flkl_jsd_forward_backward(
        _ptr(X), _ptr(W), _ptr(b), _ptr(Xt), _ptr(Wt), _ptr(bt), _ptr(shift_labels),
        ignore_index, BT, H, Ht, V, DTYPES[dt], temperature, beta, REDUCTIONS[reduction],
        compute_dW, compute_db, accum_fp32, _ptr(loss), _ptr(dX), _ptr(dW), _ptr(db),
        _ptr(workspace), workspace.numel(), st.cuda_stream)
    if status != FLKL_OK:
        raise FlklError(status, "flkl_jsd_forward_backward")
    if check_status:
        s = flkl_device_status(_ptr(workspace), st.cuda_stream)
        if s != FLKL_OK:
            raise FlklError(s, "flkl_jsd_forward_backward (device)")
    return {"loss": loss, "dX": dX, "dW": dW, "db": db, "workspace": workspace}


class _FusedLinearJSDFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, b, Xt, Wt, bt, shift_labels, ignore_index, temperature, beta,
                reduction, accum_fp32):
        r = jsd_forward_backward(
            X.contiguous(), W.contiguous(), None if b is None else b.contiguous(),
            Xt.contiguous(), Wt.contiguous(), None if bt is None else bt.contiguous(),
            None if shift_labels is None else shift_labels.contiguous(), ignore_index,
            temperature, beta, reduction, compute_dW=ctx.needs_input_grad[1],
            compute_db=b is not None and ctx.needs_input_grad[2], accum_fp32=accum_fp32)
        ctx.save_for_backward(r["dX"], r["dW"], r["db"])
        ctx.w_dtype = W.dtype
        return r["loss"]

    @staticmethod
    def backward(ctx, grad_out):
        dX, dW, db = ctx.saved_tensors
        # one pass each: scale by the incoming gradient and cast to the
        # parameter dtype, on the device
        dX = _scaled(dX, grad_out, dX.dtype)
        dW = _scaled(dW, grad_out, ctx.w_dtype)
        db = _scaled(db, grad_out, ctx.w_dtype)
        return dX, dW, db, None, None, None, None, None, None, None, None, None


class FusedLinearJSDLoss(torch.nn.Module):
    """Fused linear generalized Jensen-Shannon divergence between a student
    head and a teacher head (the teacher gets no gradient), gradient in
    forward: ``forward(student_weight, student_input, teacher_input,
    teacher_weight, shift_labels=None, student_bias=None, teacher_bias=None)``.
    """

    def __init__(self, beta: float = 0.5, ignore_index: int = -100,
                 temperature: float = 1.0, reduction: str = "batchmean",
                 accum_dtype: Optional[torch.dtype] = None):
        super().__init__()
        if not 0.0 < beta < 1.0:
            raise ValueError("beta must lie in (0, 1)")
        if reduction not in ("batchmean", "mean", "sum"):
            raise ValueError(f"reduction {reduction!r} is not supported")
        self.beta, self.ignore_index, self.temperature = beta, ignore_index, temperature
        self.reduction = reduction
        self.accum_fp32 = accum_dtype == torch.float32

    def forward(self, student_weight, student_input, teacher_input, teacher_weight,
                shift_labels=None, student_bias=None, teacher_bias=None):
        return _FusedLinearJSDFunction.apply(student_input, student_weight, student_bias,
                                             teacher_input.detach(), teacher_weight.detach(),
                                             None if teacher_bias is None
                                             else teacher_bias.detach(),
                                             shift_labels, self.ignore_index, self.temperature,
                                             self.beta, self.reduction, self.accum_fp32)


def count_valid(labels: Optional[torch.Tensor], BT: int, ignore_index: int = -100,
                device=None, out: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Kept rows of a batch (labels != ignore_index; all BT rows when labels is
    None) as a device int64 scalar, counted by the CUDA library."""
    dev = labels.device if labels is not None else torch.device(device or "cuda")
    if labels is not None:
        _check_dev("labels", labels, torch.int64, (BT,), dev)
    count = torch.empty((), dtype=torch.int64, device=dev) if out is None else out
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    status = flkl_count_valid(_ptr(labels), BT, ignore_index, _ptr(count), st.cuda_stream)
    if status != FLKL_OK:
        raise FlklError(status, "flkl_count_valid")
    return count


class _SelectiveLogProbFunction(torch.autograd.Function):
    """Per-row target log-probabilities with a true backward: the forward
    keeps the row statistics in its workspace, the backward runs pass 2 and
    the dX / dW / db GEMMs for the incoming gradients, computing dW and db
    only when autograd asks for them."""

    @staticmethod
    def forward(ctx, X, W, b, target, ignore_index, temperature, accum_fp32):
        X, W = X.contiguous(), W.contiguous()
        b = None if b is None else b.contiguous()
        target = target.contiguous()
        dev, dt = X.device, X.dtype
        if dt not in DTYPES:
            raise ValueError(f"dtype {dt} not supported (float32 or bfloat16)")
        BT, H = X.shape
        V = W.shape[0]
        _check_dev("W", W, dt, (V, H), dev)
        _check_dev("target", target, torch.int64, (BT,), dev)
        if b is not None:
            _check_dev("b", b, dt, (V,), dev)
        cw = bool(ctx.needs_input_grad[1])
        cb = bool(b is not None and ctx.needs_input_grad[2])
        need = flkl_workspace_size(BT, H, V, DTYPES[dt], cw, cb)
        if need == 0:
            raise FlklError(1, "flkl_workspace_size")
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        logp = torch.empty((BT,), dtype=torch.float32, device=dev)
        st = torch.cuda.current_stream(dev)
        s = flkl_selective_logprob_forward(_ptr(X), _ptr(W), _ptr(b), _ptr(target),
                                           ignore_index, BT, H, V, DTYPES[dt], temperature, cw,
                                           cb, _ptr(logp), _ptr(ws), ws.numel(), st.cuda_stream)
        if s != FLKL_OK:
            raise FlklError(s, "flkl_selective_logprob_forward")
        ctx.save_for_backward(X, W, b, target)
        ctx.ws, ctx.cw, ctx.cb = ws, cw, cb
        ctx.opts = (ignore_index, temperature, accum_fp32)
        return logp

    @staticmethod
    def backward(ctx, dlogp):
        X, W, b, target = ctx.saved_tensors
        ignore_index, temperature, accum_fp32 = ctx.opts
        dev, dt = X.device, X.dtype
        BT, H = X.shape
        V = W.shape[0]
        dlogp = dlogp.contiguous().to(torch.float32)
        pdt = torch.float32 if (accum_fp32 or dt == torch.float32) else dt
        dX = torch.empty_like(X)
        dW = torch.empty((V, H), dtype=pdt, device=dev) if ctx.cw else None
        db = torch.empty((V,), dtype=pdt, device=dev) if ctx.cb else None
        st = torch.cuda.current_stream(dev)
        s = flkl_selective_logprob_backward(
            _ptr(X), _ptr(W), _ptr(b), _ptr(target), ignore_index, BT, H, V, DTYPES[dt],
            temperature, _ptr(dlogp), ctx.cw, ctx.cb, accum_fp32, _ptr(dX), _ptr(dW), _ptr(db),
            _ptr(ctx.ws), ctx.ws.numel(), st.cuda_stream)
        if s != FLKL_OK:
            raise FlklError(s, "flkl_selective_logprob_backward")
        if dW is not None:
            dW = dW.to(W.dtype)
        if db is not None:
            db = db.to(W.dtype)
        return dX, dW, db, None, None, None, None


def selective_logprob(X: torch.Tensor, W: torch.Tensor, b: Optional[torch.Tensor],
                      target: torch.Tensor, ignore_index: int = -100,
                      temperature: float = 1.0, accum_fp32: bool = True) -> torch.Tensor:
    """Per-row log-probability of ``target`` under softmax((X Wᵀ + b)/T), as
    an autograd function (any loss of the per-token log-probabilities can
    follow, e.g. a policy-gradient objective); rows whose target is
    ``ignore_index`` or outside [0, V) give 0 and no gradient.  dW / db are
    computed only when W / b require grad."""
    return _SelectiveLogProbFunction.apply(X, W, b, target, ignore_index, temperature,
                                           accum_fp32)


class SelectiveLogProb(torch.nn.Module):
    """Module form of :func:`selective_logprob`:
    ``forward(lin_weight, _input, target, bias=None) -> logp [BT]``."""

    def __init__(self, ignore_index: int = -100, temperature: float = 1.0,
                 accum_dtype: Optional[torch.dtype] = torch.float32):
        super().__init__()
        self.ignore_index = ignore_index
        self.temperature = temperature
        self.accum_fp32 = accum_dtype == torch.float32

    def forward(self, lin_weight, _input, target, bias=None):
        return selective_logprob(_input, lin_weight, bias, target, self.ignore_index,
                                 self.temperature, self.accum_fp32)


class _FusedLinearCEFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, X, W, b, target, ignore_index, temperature, reduction, accum_fp32):
        r = cross_entropy_forward_backward(
            X.contiguous(), W.contiguous(), None if b is None else b.contiguous(),
            target.contiguous(), ignore_index, temperature, reduction,
            compute_dW=ctx.needs_input_grad[1],
            compute_db=b is not None and ctx.needs_input_grad[2], accum_fp32=accum_fp32)
        ctx.save_for_backward(r["dX"], r["dW"], r["db"])
        ctx.w_dtype = W.dtype
        return r["loss"]

    @staticmethod
    def backward(ctx, grad_out):
        dX, dW, db = ctx.saved_tensors
        # one pass each: scale by the incoming gradient and cast to the
        # parameter dtype, on the device
        dX = _scaled(dX, grad_out, dX.dtype)
        dW = _scaled(dW, grad_out, ctx.w_dtype)
        db = _scaled(db, grad_out, ctx.w_dtype)
        return dX, dW, db, None, None, None, None, None


class FusedLinearCrossEntropyLoss(torch.nn.Module):
    """Fused vocabulary-head projection + cross-entropy with gradient in
    forward (the one-hot-teacher case of FusedLinearKLDivLoss).

    ``forward(lin_weight, _input, target, bias=None)``; rows whose target
    equals ``ignore_index`` are dropped; ``reduction`` "batchmean" (kept-row
    mean, torch's "mean"), "mean" (per element) or "sum".
    """

    def __init__(self, ignore_index: int = -100, reduction: str = "batchmean",
                 temperature: float = 1.0, accum_dtype: Optional[torch.dtype] = None):
        super().__init__()
        if reduction not in ("batchmean", "mean", "sum"):
            raise ValueError(f"reduction {reduction!r} is not supported")
        self.ignore_index = ignore_index
        self.reduction = reduction
        self.temperature = temperature
        self.accum_fp32 = accum_dtype == torch.float32

    def forward(self, lin_weight, _input, target, bias=None):
        return _FusedLinearCEFunction.apply(_input, lin_weight, bias, target, self.ignore_index,
                                            self.temperature, self.reduction, self.accum_fp32)
