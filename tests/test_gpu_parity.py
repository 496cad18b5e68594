"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases compare every output element; they span several tiles, ragged
tails in BT, H and V, several vocabulary chunks, and the degenerate cases
(one row, all rows dropped, no rows, exact zeros and sub-eps entries in Q).
The full-size workloads run in the same launch configuration as the
benchmark and compare the loss, db, and sampled rows of dX and dW.
"""

import numpy as np
import pytest
import torch

import lm_head_projection_b200 as pkg
from lm_head_projection_b200.workloads import WORKLOADS, make_inputs, small_case
from tests.parity_utils import assert_close, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

SMALL = [
    # dtype, BT, H, V, bias, reduction, T, ignore_frac, zero_frac, dW, db
    ("bf16", 133, 192, 1000, True, "batchmean", 1.0, 0.0, 0.0, True, True),
    ("bf16", 1, 64, 8, False, "sum", 1.0, 0.0, 0.0, True, False),
    ("bf16", 129, 72, 1032, True, "batchmean", 1.0, 0.0, 0.05, True, True),
    ("bf16", 300, 256, 4104, True, "mean", 2.0, 0.1, 0.05, True, True),
    ("bf16", 127, 128, 2056, False, "batchmean", 0.5, 0.2, 0.0, False, False),
    ("bf16", 257, 320, 3000, False, "sum", 1.0, 0.0, 0.0, True, False),
    ("bf16", 3, 4096, 1024, True, "batchmean", 1.0, 0.0, 0.0, True, True),
    ("fp32", 64, 256, 1024, False, "batchmean", 1.0, 0.0, 0.0, True, False),
    ("fp32", 133, 72, 1000, True, "mean", 2.0, 0.1, 0.05, True, True),
    ("fp32", 3, 64, 4104, True, "sum", 0.5, 0.0, 0.0, True, True),
    ("fp32", 1, 4, 4, False, "batchmean", 1.0, 0.0, 0.0, True, False),
]


def _ids(c):
    return f"{c[0]}-{c[1]}x{c[2]}x{c[3]}-{'b' if c[4] else 'nob'}-{c[5]}-T{c[6]}-ig{c[7]}-z{c[8]}"


@pytest.mark.parametrize("case", SMALL, ids=[_ids(c) for c in SMALL])
def test_small_case_matches_oracle(case):
    dt, BT, H, V, bias, red, T, ig, zf, dW, db = case
    w = small_case(dtype=dt, BT=BT, H=H, V=V, bias=bias, reduction=red, temperature=T,
                   ignore_frac=ig, zero_frac=zf, compute_dW=dW, compute_db=db, seed=BT + V)
    inp = make_inputs(w)
    got = run_gpu(inp)
    ref = run_oracle(inp)
    assert_close(dt, got, ref)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_all_rows_dropped_gives_zeros(dt):
    w = small_case(dtype=dt, BT=70, H=64, V=520, bias=True, ignore_frac=1.0)
    inp = make_inputs(w)
    got = run_gpu(inp)
    assert float(got["loss"].cpu()) == 0.0
    for k in ("dX", "dW", "db"):
        assert not torch.any(got[k] != 0), k


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_no_rows(dt):
    tdt = torch.float32 if dt == "fp32" else torch.bfloat16
    dev = torch.device("cuda:0")
    X = torch.empty((0, 64), dtype=tdt, device=dev)
    W = torch.randn((40, 64), device=dev).to(tdt)
    b = torch.zeros(40, device=dev).to(tdt)
    Q = torch.empty((0, 40), dtype=tdt, device=dev)
    out = {"dW": torch.full((40, 64), 7.0, device=dev), "db": torch.full((40,), 7.0, device=dev),
           "loss": torch.full((), 7.0, device=dev)}
    r = pkg.forward_backward(X, W, b, Q, compute_dW=True, compute_db=True, out=out,
                             check_status=True)
    torch.cuda.synchronize()
    assert float(r["loss"].cpu()) == 0.0
    assert not torch.any(r["dW"] != 0) and not torch.any(r["db"] != 0)


@pytest.mark.parametrize("dt", ["bf16", "fp32"])
def test_frozen_head_gives_identical_loss_and_dX(dt):
    """compute_dW / compute_db change nothing in the loss and dX, bit for bit
    (frozen-head pages: the loss and the input gradients are unchanged)."""
    w = small_case(dtype=dt, BT=200, H=128, V=2056, bias=True, ignore_frac=0.1)
    inp = make_inputs(w)
    a = run_gpu(inp, compute_dW=True, compute_db=True)
    b = run_gpu(inp, compute_dW=False, compute_db=False)
    c = run_gpu(inp, compute_dW=True, compute_db=False)
    assert b["dW"] is None and b["db"] is None and c["db"] is None
    assert torch.equal(a["loss"], b["loss"]) and torch.equal(a["loss"], c["loss"])
    assert torch.equal(a["dX"], b["dX"]) and torch.equal(a["dX"], c["dX"])
    assert torch.equal(a["dW"], c["dW"])


def test_frozen_call_leaves_foreign_buffers_alone():
    """A frozen call must not be handed a dW buffer: the host rejects it and
    nothing is launched (the canary buffers keep their values)."""
    w = small_case(dtype="bf16", BT=64, H=64, V=256, bias=False)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    loss = torch.full((), 3.0, device=dev)
    dX = torch.full_like(g["X"], 5.0)
    dW = torch.full((256, 64), 9.0, device=dev)
    ws = torch.empty(pkg.flkl_workspace_size(64, 64, 256, 1, 0, 0), dtype=torch.uint8, device=dev)
    st = pkg.flkl_forward_backward(
        g["X"].data_ptr(), g["W"].data_ptr(), None, g["Q"].data_ptr(), None, -100, 64, 64, 256, 1,
        1.0, 1e-10, 0, 0, 0, 1, loss.data_ptr(), dX.data_ptr(), dW.data_ptr(), None,
        ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 1
    assert float(loss.cpu()) == 3.0 and bool((dX == 5.0).all()) and bool((dW == 9.0).all())


def test_repeated_calls_are_bitwise_deterministic():
    w = small_case(dtype="bf16", BT=300, H=256, V=4104, bias=True, ignore_frac=0.1)
    inp = make_inputs(w)
    a = run_gpu(inp)
    b = run_gpu(inp)
    for k in ("loss", "dX", "dW", "db"):
        assert torch.equal(a[k], b[k]), k


def test_bf16_param_grads_without_fp32_accumulation():
    w = small_case(dtype="bf16", BT=100, H=128, V=1000, bias=True)
    inp = make_inputs(w)
    got = run_gpu(inp, accum_fp32=False)
    assert got["dW"].dtype == torch.bfloat16 and got["db"].dtype == torch.bfloat16
    assert_close("bf16", got, run_oracle(inp))


def test_teacher_equal_to_student_gives_small_loss():
    """Q = softmax of the student's own logits (fp64, from the bf16 inputs):
    the loss is the KL of the bf16-rounded teacher against the student, so it
    must sit near 0 on both sides, and the oracle decides the value."""
    w = small_case(dtype="bf16", BT=64, H=128, V=1024, bias=False, temperature=1.3)
    inp = make_inputs(w)
    X = inp["X"].double()
    W = inp["W"].double()
    u = (X @ W.T) / 1.3
    inp["Q"] = torch.softmax(u, dim=1).to(torch.bfloat16)
    got = run_gpu(inp)
    ref = run_oracle(inp)
    assert abs(ref["loss"]) < 1e-3
    assert abs(float(got["loss"].cpu()) - ref["loss"]) < 2e-4


def test_bounded_wait_reports_timeout_and_context_survives():
    dev = torch.device("cuda:0")
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    assert pkg.flkl_wait_selftest(status.data_ptr(), 50,
                                  torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(status.cpu()) == 4  # FLKL_ERR_TIMEOUT
    # the context is still usable afterwards
    w = small_case(dtype="bf16", BT=64, H=64, V=256)
    inp = make_inputs(w)
    assert_close("bf16", run_gpu(inp), run_oracle(inp))


def test_autograd_module_matches_direct_call():
    w = small_case(dtype="bf16", BT=96, H=128, V=1000, bias=True, reduction="sum")
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    X = inp["X"].to(dev).requires_grad_(True)
    W = inp["W"].to(dev).requires_grad_(True)
    b = inp["b"].to(dev).requires_grad_(True)
    Q = inp["Q"].to(dev)
    mod = pkg.FusedLinearKLDivLoss(reduction="sum", accum_dtype=torch.float32)
    loss = mod(W, X, Q, bias=b)
    (2.0 * loss).backward()
    direct = run_gpu(inp, compute_dW=True, compute_db=True)
    assert torch.equal(loss.detach(), direct["loss"])
    assert torch.allclose(X.grad.float(), 2.0 * direct["dX"].float(), rtol=1e-2, atol=1e-6)
    assert torch.allclose(W.grad.float(), (2.0 * direct["dW"]).to(torch.bfloat16).float(),
                          rtol=1e-2, atol=1e-6)
    # frozen head through autograd: no weight gradient requested or produced
    W2 = inp["W"].to(dev)
    X2 = inp["X"].to(dev).requires_grad_(True)
    loss2 = mod(W2, X2, Q, bias=None)
    loss2.backward()
    assert W2.grad is None and X2.grad is not None


# ------------------------------------------------------------------ full-size workloads

def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    rows = set(int(x) for x in rng.choice(n, size=min(k, n), replace=False))
    rows |= {0, n - 1}
    return sorted(rows)


def _tile_edges(n, tile=256):
    """First and last index of every `tile`-wide block of [0, n): every
    vocabulary chunk of the CUDA path starts and ends on such a block, so
    these rows include each chunk's first and last row (the ragged last
    chunk among them), whatever the chunk width."""
    rows = set()
    for t0 in range(0, n, tile):
        rows |= {t0, min(n, t0 + tile) - 1}
    return rows


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_workload(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    got = run_gpu(inp)
    dx_rows = _sample(w.BT, 24, 1)
    dw_rows = sorted(set(_sample(w.V, 24, 2)) | _tile_edges(w.V)) if w.compute_dW else None
    ref = run_oracle(inp, dX_rows=dx_rows, dW_rows=dw_rows)
    assert_close(w.dtype, got, ref, dX_rows=dx_rows, dW_rows=dw_rows)
    # dX rows of dropped rows are exactly zero
    if inp["shift_labels"] is not None:
        drop = (inp["shift_labels"] == inp["ignore_index"]).nonzero().flatten()
        assert not torch.any(got["dX"][drop.to(got["dX"].device)] != 0)


def test_no_bt_by_v_allocation_at_full_size():
    """Peak device memory of one call of the headline workload stays below
    inputs + outputs + workspace, and the workspace holds no BT x V array:
    it is below one bf16 BT x V array, the first chunk's logits that pass 1
    keeps for pass 2 (fp32) included."""
    w = WORKLOADS["bf16_bt1024_h4096_v128256"]
    dev = torch.device("cuda:0")
    inp = make_inputs(w, device=dev)
    r = run_gpu(inp)  # warm: allocates outputs + workspace once
    out = {"loss": r["loss"], "dX": r["dX"], "dW": r["dW"]}
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    pkg.forward_backward(inp["X"], inp["W"], None, inp["Q"], compute_dW=True, out=out,
                         workspace=r["workspace"])
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated(dev) - base == 0
    assert r["workspace"].numel() < w.BT * w.V * 2


def test_profiled_entry_records_every_launch_and_matches():
    """flkl_forward_backward_profiled gives the same results as the plain
    entry and tags every launch with its kind, in launch order."""
    w = small_case(dtype="bf16", BT=130, H=128, V=2056, bias=True)
    inp = make_inputs(w)
    dev = torch.device("cuda:0")
    ref = run_gpu(inp)
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out = {k: torch.empty_like(ref[k]) for k in ("loss", "dX", "dW", "db")}
    ws = torch.empty_like(ref["workspace"])
    stream = torch.cuda.current_stream()
    cap = 64
    events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * cap)]
    for e in events:
        e.record(stream)
    p = lambda t: None if t is None else t.data_ptr()
    st, kinds, flops, n = pkg.flkl_forward_backward_profiled(
        p(g["X"]), p(g["W"]), p(g["b"]), p(g["Q"]), None, -100, w.BT, w.H, w.V, 1, 1.0, 1e-10, 0,
        1, 1, 1, p(out["loss"]), p(out["dX"]), p(out["dW"]), p(out["db"]), p(ws), ws.numel(),
        stream.cuda_stream, events, cap)
    torch.cuda.synchronize()
    assert st == 0 and n == len(kinds)
    names = [pkg.LAUNCH_KINDS[k] for k in kinds]
    nchunks = names.count("chunk")
    assert nchunks >= 2
    # the loss sum runs inside the combine launch
    assert names == (["prepare", "stats", "combine", "grad"] + ["chunk"] * nchunks + ["db"])
    # every GEMM FLOP of the call is attributed once: stats, pass 2, dX and
    # dW; pass 2 of the first chunk reads the logits pass 1 kept (no GEMM)
    gemm = 2.0 * w.BT * w.H * w.V
    chunk0 = pkg.flkl_vocab_chunks(w.BT, w.H, w.V, 1, True, True)[1]
    assert abs(sum(flops) - (4 * gemm - 2.0 * w.BT * w.H * chunk0)) <= 1e-6 * gemm
    assert flops[0] == 0.0 and flops[-1] == 0.0 and flops[names.index("grad")] == 0.0
    for i in range(n):
        assert events[2 * i].elapsed_time(events[2 * i + 1]) >= 0.0
    for k in ("loss", "dX", "dW", "db"):
        assert torch.equal(out[k], ref[k]), k


def test_batch_pipeline_matches_direct_calls():
    """The double-buffered host-batch pipeline gives, step by step, the loss
    of direct calls on the same batches, for the KL and the CE losses."""
    from lm_head_projection_b200.pipeline import BatchPipeline

    dev = torch.device("cuda:0")
    for ce in (False, True):
        ws = [small_case(dtype="bf16", BT=96, H=128, V=1000, bias=True, ce=ce, ignore_frac=0.1,
                         seed=s) for s in (1, 2, 3)]
        inps = [make_inputs(w) for w in ws]
        W = inps[0]["W"].to(dev)
        b = inps[0]["b"].to(dev)
        opts = dict(ignore_index=-100, temperature=1.0, reduction="batchmean",
                    compute_dW=True, compute_db=True, accum_fp32=True)
        if not ce:
            opts["eps"] = 1e-10
        pipe = BatchPipeline(W, b, kind="ce" if ce else "kl", options=opts)
        direct = []
        for inp in inps:
            host = ([inp["X"].pin_memory(), inp["target"].pin_memory()] if ce else
                    [inp["X"].pin_memory(), inp["Q"].pin_memory(),
                     inp["shift_labels"].pin_memory()])
            pipe.submit(host)
            d = dict(inp, W=inps[0]["W"], b=inps[0]["b"])
            direct.append(float(run_gpu(d)["loss"].cpu()))
        pipe.finish()
        torch.cuda.synchronize()
        got = pipe.losses().tolist()
        assert got == direct, (ce, got, direct)
        last = run_gpu(dict(inps[-1], W=inps[0]["W"], b=inps[0]["b"]))
        assert torch.equal(pipe.out["dX"], last["dX"])
        assert torch.equal(pipe.out["dW"], last["dW"])
