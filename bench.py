#!/usr/bin/env python
"""Throughput of the fused linear-head + KL-divergence loss (forward + backward).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one flkl_forward_backward call over one batch of BT rows: loss, dX
and (when the workload trains the head) dW/db, with every input resident in
device memory.  Prints one JSON line on rank 0.

* value      rows (tokens) per second over all ranks, timed with CUDA events
             on the launch stream around exactly K steps (max over ranks);
* e2e        the same metric through the public Python API with the batch
             (X, Q or targets, labels) copied from pinned host memory every
             step (BatchPipeline: the copy of step i+1 overlaps the loss of
             step i) and every loss read back; the head W stays resident;
* roofline   the dominant kernel (largest share of the step's device time)
             from a second, profiled run of K steps: its GEMM FLOPs per launch
             over its average launch time, against the measured bf16 peak;
* cpu_baseline  the fp64 oracle on the host cores on a bounded row sample.

Multi-GPU (launched with torch.distributed.run): every rank runs its own
batch (weak scaling, data parallel); the only collectives are the timing
barrier and the max-over-ranks reduction of the elapsed time.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from lm_head_projection_b200.workloads import (CE_WORKLOADS, HEADLINE, WORKLOADS,  # noqa: E402
                                               make_inputs)

ALL_WORKLOADS = {**WORKLOADS, **CE_WORKLOADS}

METRIC = "fwd+bwd tokens/s at H=4096,V=128256 bf16; % of roofline (tensor/HBM)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


GEMM_SOURCES = ("flkl_api.cu", "ptx.cuh", "row_kernels.cuh", "tc_gemm.cuh")


def kernel_source_hash() -> str:
    """Hash of the CUDA sources the fused-loss kernels are built from."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lm_head_projection_b200", "csrc")
    for fn in GEMM_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def dram_traffic(workload: str, launch_kind: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
    `launch_kind` for `workload`, from the committed ncu summary, or None when
    there is none or the kernel sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_hash") != kernel_source_hash():
        return None
    v = vals.get(f"dram_bytes_per_launch_{launch_kind}")
    return float(v) if v else None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=list(ALL_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-rows", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="loss",
                    choices=["loss", "rms_norm", "layer_norm", "logprob", "jsd"],
                    help="loss: the fused linear KL / CE loss (default); rms_norm / "
                         "layer_norm: the norm backward with frozen-parameter flags; logprob: "
                         "selective log-probability forward + backward on a CE workload; "
                         "jsd: fused linear JSD with a teacher head of the same shape")
    ap.add_argument("--norm-shape", default="8192x8192", help="ROWSxH for --op *_norm")
    ap.add_argument("--norm-dtype", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--frozen", action="store_true", help="norm weight (and bias) frozen")
    ap.add_argument("--calls", type=int, default=0,
                    help="profiling helper: run this many plain calls of --workload through "
                         "the public API, print their CUDA-event times and exit (no bench "
                         "line); a small case for ncu is --workload NAME with --rows R")
    ap.add_argument("--rows", type=int, default=0,
                    help="with --calls: take the workload with BT=R rows instead of its own")
    ap.add_argument("--dp", action="store_true",
                    help="data-parallel training step: whole-batch kept-row count and "
                         "all-reduce of loss, dW, db (NCCL) inside each timed step")
    return ap.parse_args()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="flkl_clocks_", suffix=".csv")
        self.proc = None
        self.t_start = time.time()
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[3], parts[4:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # samples under load: the upper half of the observed clocks
        clocks = sorted(r[0] for r in rows)
        active = [r for r in rows if r[0] >= clocks[len(clocks) // 4]]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3][1:5])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in active), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ helpers

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} needs {n_gpus} ranks (WORLD_SIZE={world}); launch "
                         "with python -m torch.distributed.run --nproc-per-node N")
    return world, rank, local


def max_over_ranks(value: float, device) -> float:
    """The maximum of `value` over all ranks (a no-op without a process
    group): a multi-GPU time is the slowest rank's time."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample(w, rows, seed=123):
    """Inputs of a `rows`-row sample of workload `w` (fresh draw), as fp64
    numpy arrays, plus the oracle's keyword arguments."""
    import numpy as np

    inp = make_inputs(w.with_(BT=rows, seed=seed), device="cpu")
    f = lambda t: None if t is None else t.float().numpy().astype(np.float64)
    if w.ce:
        args = (f(inp["X"]), f(inp["W"]), f(inp["b"]), inp["target"].numpy())
        kw = dict(ignore_index=inp["ignore_index"], temperature=inp["temperature"],
                  reduction=inp["reduction"], compute_dW=inp["compute_dW"],
                  compute_db=inp["compute_db"], ce=True)
        return args, kw
    args = (f(inp["X"]), f(inp["W"]), f(inp["b"]), f(inp["Q"]))
    kw = dict(shift_labels=None if inp["shift_labels"] is None else inp["shift_labels"].numpy(),
              ignore_index=inp["ignore_index"], temperature=inp["temperature"], eps=inp["eps"],
              reduction=inp["reduction"], compute_dW=inp["compute_dW"],
              compute_db=inp["compute_db"])
    return args, kw


def host_threads():
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        nt = max((i.get("num_threads", 0) for i in threadpool_info()), default=0)
        cores = nt or cores
    except Exception:
        pass
    return cores


def time_oracle(args, kw):
    from oracle import ce_forward_backward, forward_backward

    kw = dict(kw)
    fn = ce_forward_backward if kw.pop("ce", False) else forward_backward
    t0 = time.perf_counter()
    fn(*args, **kw)
    return time.perf_counter() - t0


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch.distributed as dist

    import lm_head_projection_b200 as pkg

    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    w = ALL_WORKLOADS[args.workload].with_(seed=ALL_WORKLOADS[args.workload].seed + rank)
    inp = make_inputs(w, device=dev)
    X, W, b, Q, lab = inp["X"], inp["W"], inp["b"], inp["Q"], inp["shift_labels"]
    tgt = inp.get("target")
    dt_code = pkg.DTYPES[X.dtype]
    compute_db = inp["compute_db"]

    def api_call(out=None, workspace=None, check_status=False):
        """The public Python API call a user makes for this workload."""
        if w.ce:
            return pkg.cross_entropy_forward_backward(
                X, W, b, tgt, inp["ignore_index"], inp["temperature"], inp["reduction"],
                compute_dW=inp["compute_dW"], compute_db=compute_db,
                accum_fp32=inp["accum_fp32"], out=out, workspace=workspace,
                check_status=check_status)
        return pkg.forward_backward(X, W, b, Q, lab, inp["ignore_index"], inp["temperature"],
                                    inp["eps"], inp["reduction"], compute_dW=inp["compute_dW"],
                                    compute_db=compute_db, accum_fp32=inp["accum_fp32"],
                                    out=out, workspace=workspace, check_status=check_status)

    r0 = api_call(check_status=True)
    ws = r0["workspace"]
    out = {k: r0[k] for k in ("loss", "dX", "dW", "db")}
    stream = torch.cuda.current_stream(dev)
    p = lambda t: None if t is None else t.data_ptr()
    call_args = (p(X), p(W), p(b), p(Q), p(lab), inp["ignore_index"], w.BT, w.H, w.V, dt_code,
                 inp["temperature"], inp["eps"], pkg.REDUCTIONS[inp["reduction"]],
                 inp["compute_dW"], compute_db, inp["accum_fp32"], p(out["loss"]), p(out["dX"]),
                 p(out["dW"]), p(out["db"]), p(ws), ws.numel(), stream.cuda_stream)
    ce_args = (p(X), p(W), p(b), p(tgt), inp["ignore_index"], w.BT, w.H, w.V, dt_code,
               inp["temperature"], pkg.REDUCTIONS[inp["reduction"]], inp["compute_dW"],
               compute_db, inp["accum_fp32"], p(out["loss"]), p(out["dX"]), p(out["dW"]),
               p(out["db"]), p(ws), ws.numel(), stream.cuda_stream)

    n_total = torch.zeros((), dtype=torch.int64, device=dev)
    mask = tgt if w.ce else lab
    exchanged = [t for t in (out["loss"], out["dW"], out["db"]) if t is not None]

    def step():
        if not args.dp:
            s = (pkg.flkl_ce_forward_backward(*ce_args) if w.ce
                 else pkg.flkl_forward_backward(*call_args))
        else:
            # the data-parallel step of lm_head_projection_b200.dp, raw entry points
            s = pkg.flkl_count_valid(p(mask), w.BT, inp["ignore_index"], p(n_total),
                                     stream.cuda_stream)
            if s == 0:
                if world > 1:
                    dist.all_reduce(n_total)
                s = (pkg.flkl_ce_forward_backward_dp(*ce_args, p(n_total)) if w.ce
                     else pkg.flkl_forward_backward_dp(*call_args, p(n_total)))
            if s == 0 and world > 1:
                for t in exchanged:
                    dist.all_reduce(t)
        if s != 0:
            raise pkg.FlklError(s, "flkl_forward_backward")

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").replace(",", "").isdigit() else local
    clocks = ClockSampler(gpu_index)
    time.sleep(0.3)

    # ---------------- timed region: exactly K steps
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    status = pkg.flkl_device_status(ws.data_ptr(), stream.cuda_stream)
    if status != 0:
        raise pkg.FlklError(status, "device status after the timed region")

    # ---------------- per-launch breakdown: K profiled steps
    cap = 256
    events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * cap)]
    for e in events:  # torch creates the CUDA event on its first record
        e.record(stream)
    torch.cuda.synchronize()
    per_kind = {}  # kind -> [ms, launches, gemm flops]
    launches_per_step = 0
    for _ in range(args.steps):
        st, kinds, flops, n = pkg.flkl_forward_backward_profiled(*call_args, events, cap,
                                                                 ce_target=p(tgt))
        if st != 0:
            raise pkg.FlklError(st, "flkl_forward_backward_profiled")
        launches_per_step = n
        torch.cuda.synchronize()
        for i, k in enumerate(kinds):
            d = per_kind.setdefault(pkg.LAUNCH_KINDS[k], [0.0, 0, 0.0])
            d[0] += events[2 * i].elapsed_time(events[2 * i + 1])
            d[1] += 1
            d[2] += flops[i]
    clocks.stop()
    clk = clocks.summary()

    total_prof_ms = sum(v[0] for v in per_kind.values())
    dominant = max(per_kind, key=lambda k: per_kind[k][0])
    peaks, peaks_src = load_peaks()
    peak_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    dom_ms, dom_n, dom_flops = per_kind[dominant]
    if dom_flops > 0:
        achieved = dom_flops / (dom_ms * 1e-3) / 1e12  # = flops per launch / avg launch time
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak_sust,
                    "unit": "TFLOP/s", "frac": round(achieved / peak_sust, 4),
                    "traffic": dram_traffic(w.name, dominant),
                    "kernel": f"tc_group_kernel ({dominant} launches)",
                    "flops_per_launch": dom_flops / dom_n,
                    "avg_launch_ms": round(dom_ms / dom_n, 4),
                    "peak_note": f"bf16_tflops_sustained of {peaks_src}",
                    "share": round(dom_ms / total_prof_ms, 3)}
    else:
        roofline = {"bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": None, "traffic": None, "kernel": dominant}
    breakdown = {k: {"ms_per_step": round(v[0] / args.steps, 4), "launches_per_step":
                     round(v[1] / args.steps, 2), "share": round(v[0] / total_prof_ms, 3),
                     "tflops": round(v[2] / (v[0] * 1e-3) / 1e12, 1) if v[2] else None}
                 for k, v in sorted(per_kind.items())}

    ms_per_step = ms / args.steps
    tokens = w.BT * world
    value = tokens / (ms_per_step * 1e-3)
    counted = w.flops_counted()
    step_tflops = counted / (ms_per_step * 1e-3) / 1e12
    roof_time = max(counted / (peaks["bf16_tflops"] * 1e12),
                    (algorithmic_bytes(w) / (peaks["hbm_gbs"] * 1e9)))
    step_roofline = {"counted_flops": counted, "tflops": round(step_tflops, 1),
                     "frac_of_burst": round(roof_time / (ms_per_step * 1e-3), 4),
                     "frac_of_sustained": round(
                         max(counted / (peak_sust * 1e12),
                             algorithmic_bytes(w) / (peaks["hbm_gbs"] * 1e9))
                         / (ms_per_step * 1e-3), 4),
                     "peaks": peaks_src}

    # ---------------- end to end: batch from pinned host memory, loss back
    # End to end through the public API: every step's batch (X and the
    # teacher Q, or the targets, and the shift labels) comes from pinned host
    # memory; BatchPipeline overlaps the copy of step i+1 with the loss of
    # step i (two device buffers, a copy stream) and reads every loss back.
    from lm_head_projection_b200.pipeline import BatchPipeline

    batch = [t for t in ((X, tgt) if w.ce else (X, Q, lab)) if t is not None]
    hosts = [t.cpu().pin_memory() for t in batch]
    h2d = sum(h.numel() * h.element_size() for h in hosts)
    opts = dict(ignore_index=inp["ignore_index"], temperature=inp["temperature"],
                reduction=inp["reduction"], compute_dW=inp["compute_dW"],
                compute_db=compute_db, accum_fp32=inp["accum_fp32"])
    if not w.ce:
        opts["eps"] = inp["eps"]
    pipe = BatchPipeline(W, b, kind="ce" if w.ce else "kl", options=opts,
                         compute_stream=stream, max_steps=args.steps + args.warmup + 4)
    for _ in range(max(1, args.warmup)):
        pipe.submit(hosts)
    pipe.finish()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    pipe.copy.wait_event(e0)
    for _ in range(args.steps):
        pipe.submit(hosts)
    pipe.finish()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e = {"value": round(tokens / (e2e_ms / args.steps * 1e-3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = min(args.cpu_sample_rows, w.BT)
        oa, okw = oracle_sample(w, rows)
        dt = time_oracle(oa, okw)
        cores = host_threads()
        cpu = {"value": round(rows / dt, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{rows} rows of {w.name} (full H, V, same flags), fp64 numpy, "
                         f"inputs pre-converted to fp64, {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.name, "global_batch": w.BT * world, "BT_per_gpu": w.BT,
                       "H": w.H, "V": w.V, "compute_dW": w.compute_dW,
                       "compute_db": bool(compute_db), "reduction": w.reduction,
                       "temperature": w.temperature,
                       "parallelism": f"dp{world}" + ("-allreduce" if args.dp else "-replicas"),
                       "l2": "inputs larger than L2 (W, Q), no flush"},
            "e2e": e2e, "roofline": roofline, "step_roofline": step_roofline,
            "kernels": breakdown,
            "gpu_launches": int((launches_per_step + (1 if args.dp else 0)) * args.steps),
            "clocks": clk, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def algorithmic_bytes(w) -> float:
    """X, W, Q and labels read once, dX and dW/db written once."""
    e = 4 if w.dtype == "fp32" else 2
    pe = 4 if (w.accum_fp32 or w.dtype == "fp32") else 2
    b = w.BT * w.H * e * 2 + w.V * w.H * e + (w.BT * 8 if w.ce else w.BT * w.V * e)
    if w.compute_dW:
        b += w.V * w.H * pe
    if w.bias:
        b += w.V * e + (w.V * pe if w.compute_db else 0)
    if w.ignore_frac > 0:
        b += w.BT * 8
    return float(b)


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    w = ALL_WORKLOADS[args.workload]
    rows = max(1, min(args.ref_rows, w.BT))
    oa, okw = oracle_sample(w, rows)
    for _ in range(args.warmup):
        time_oracle(oa, okw)
    times = [time_oracle(oa, okw) for _ in range(args.steps)]
    cores = host_threads()
    total = sum(times)
    value = rows * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "global_batch": rows, "H": w.H, "V": w.V,
                   "parallelism": "host"},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"{rows} rows of {w.name} per step (full H, V, same "
                                   "flags), fp64 numpy oracle, inputs pre-converted to fp64"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_norm(args):
    """Norm backward on one GPU: device time of each launch (CUDA events on the
    launching stream), with L2 flushed between launches outside the events."""
    import numpy as np

    from lm_head_projection_b200 import norm
    from lm_head_projection_b200.workloads import make_norm_inputs

    rows, H = (int(v) for v in args.norm_shape.lower().split("x"))
    layer = args.op == "layer_norm"
    train = not args.frozen
    dev = torch.device("cuda", 0)
    inp = {k: v.to(dev) for k, v in make_norm_inputs(rows, H, args.norm_dtype, 0).items()}
    e = 4 if args.norm_dtype == "fp32" else 2

    import lm_head_projection_b200 as pkg

    # outputs through the public call once, then the C entry point itself
    # (preallocated buffers) inside the timed launches
    if layer:
        r0 = norm.layer_norm_backward(inp["dY"], inp["X"], inp["W"], compute_dW=train,
                                      compute_db=train)
    else:
        r0 = norm.rms_norm_backward(inp["dY"], inp["X"], inp["W"], compute_dW=train)
    need = pkg.flkl_norm_workspace_size(rows, H, train, layer and train)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    p = lambda t: None if t is None else t.data_ptr()
    stream0 = torch.cuda.current_stream(dev)
    dt_code = 0 if args.norm_dtype == "fp32" else 1
    if layer:
        c_args = (p(inp["dY"]), p(inp["X"]), p(inp["W"]), rows, H, dt_code, 1e-5, train, train,
                  True, p(r0["dX"]), p(r0["dW"]), p(r0["db"]), p(ws), ws.numel(),
                  stream0.cuda_stream)
        entry = pkg.flkl_layer_norm_backward
    else:
        c_args = (p(inp["dY"]), p(inp["X"]), p(inp["W"]), rows, H, dt_code, 1e-6, train, True,
                  p(r0["dX"]), p(r0["dW"]), p(ws), ws.numel(), stream0.cuda_stream)
        entry = pkg.flkl_rms_norm_backward

    def step():
        st = entry(*c_args)
        if st != 0:
            raise pkg.FlklError(st, entry.__name__)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    time.sleep(0.3)
    stream = torch.cuda.current_stream(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    if pkg.flkl_norm_device_status(stream0.cuda_stream) != 0:
        raise pkg.FlklError(4, "norm kernel wait")
    ms = sorted(a.elapsed_time(b) for a, b in evs)
    med = ms[len(ms) // 2]
    n_grads = (2 if layer else 1) if train else 0
    algo = 3 * rows * H * e + H * e + n_grads * H * 4
    peaks, peak_src = load_peaks()
    peak = peaks.get("hbm_gbs")
    achieved = algo / (med * 1e-3) / 1e9
    # the oracle on the host cores, the same shape
    from oracle.norm_oracle import layer_norm_backward as o_ln
    from oracle.norm_oracle import rms_norm_backward as o_rms
    host = {k: v.float().cpu().numpy().astype(np.float64) for k, v in inp.items()}
    t0 = time.perf_counter()
    if layer:
        o_ln(host["dY"], host["X"], host["W"], 1e-5, train, train)
    else:
        o_rms(host["dY"], host["X"], host["W"], 1e-6, train)
    t_cpu = time.perf_counter() - t0
    name = f"{args.op}_{args.norm_dtype}_{rows}x{H}{'_frozen' if args.frozen else ''}"
    line = {
        "metric": "norm_backward_rows_per_s", "value": round(rows / (med * 1e-3), 1),
        "unit": "rows/s", "n_gpus": 1, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(med, 5), "ms_min": round(ms[0], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if args.norm_dtype == "fp32" else "bf16", "data": "synthetic",
        "config": {"workload": name, "rows": rows, "H": H, "l2": "flushed between launches"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4) if peak else None,
                     "traffic": None, "algorithmic_bytes": algo, "peak_source": peak_src},
        "cpu_baseline": {"value": round(rows / t_cpu, 1), "unit": "rows/s",
                         "cores": host_threads(), "kind": "oracle",
                         "sample": f"the whole {rows}x{H} problem once, fp64 numpy"},
        "clocks": clocks.summary(),
        "gpu_launches": args.steps * (1 + n_grads),
    }
    print(json.dumps(line), flush=True)


def run_logprob(args):
    """Selective log-probability on one GPU: one step = the forward call
    (per-row target log-probabilities) and the backward call for upstream
    gradients (dX, dW), on the cross-entropy workload's inputs; CUDA events
    around exactly K steps."""
    import numpy as np

    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.workloads import CE_WORKLOADS

    name = args.workload if args.workload in CE_WORKLOADS else "ce_bf16_bt1024_h4096_v128256"
    w = CE_WORKLOADS[name]
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, device=dev)
    X, W, b, tgt = inp["X"], inp["W"], inp["b"], inp["target"]
    dt = pkg.DTYPES[X.dtype]
    cw, cb = bool(w.compute_dW), bool(inp["compute_db"])
    ws = torch.empty(pkg.flkl_workspace_size(w.BT, w.H, w.V, dt, cw, cb), dtype=torch.uint8,
                     device=dev)
    logp = torch.empty(w.BT, dtype=torch.float32, device=dev)
    dlogp = torch.randn(w.BT, generator=torch.Generator(device=dev).manual_seed(1),
                        device=dev, dtype=torch.float32)
    dX = torch.empty_like(X)
    dW = torch.empty((w.V, w.H), dtype=torch.float32, device=dev) if cw else None
    db = torch.empty((w.V,), dtype=torch.float32, device=dev) if cb else None
    p = lambda t: None if t is None else t.data_ptr()
    stream = torch.cuda.current_stream(dev)
    fa = (p(X), p(W), p(b), p(tgt), inp["ignore_index"], w.BT, w.H, w.V, dt, w.temperature,
          cw, cb, p(logp), p(ws), ws.numel(), stream.cuda_stream)
    ba = (p(X), p(W), p(b), p(tgt), inp["ignore_index"], w.BT, w.H, w.V, dt, w.temperature,
          p(dlogp), cw, cb, True, p(dX), p(dW), p(db), p(ws), ws.numel(), stream.cuda_stream)

    def step():
        s = pkg.flkl_selective_logprob_forward(*fa)
        if s == 0:
            s = pkg.flkl_selective_logprob_backward(*ba)
        if s != 0:
            raise pkg.FlklError(s, "flkl_selective_logprob")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    if pkg.flkl_device_status(p(ws), stream.cuda_stream) != 0:
        raise pkg.FlklError(4, "device status after the timed region")
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_src = load_peaks()
    flops = 2.0 * w.BT * w.H * w.V * (2 + (1 if cw else 0))
    achieved = flops / (ms * 1e-3) / 1e12
    # the oracle on the host cores: a bounded sample of rows, forward + backward
    from oracle import selective_logprob, selective_logprob_backward
    rows = min(args.cpu_sample_rows, w.BT)
    host = make_inputs(w.with_(BT=rows, seed=123), device="cpu")
    f = lambda t: None if t is None else t.float().numpy().astype(np.float64)
    Xh, Wh, bh, th = f(host["X"]), f(host["W"]), f(host["b"]), host["target"].numpy()
    t0 = time.perf_counter()
    selective_logprob(Xh, Wh, bh, th, inp["ignore_index"], w.temperature)
    selective_logprob_backward(Xh, Wh, bh, th, np.ones(rows), inp["ignore_index"],
                               w.temperature, compute_dW=cw, compute_db=cb)
    t_cpu = time.perf_counter() - t0
    line = {
        "metric": "selective log-prob fwd+bwd tokens/s", "value": round(w.BT / (ms * 1e-3), 1),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": name, "BT": w.BT, "H": w.H, "V": w.V, "compute_dW": cw,
                   "compute_db": cb, "l2": "inputs larger than L2 (W), no flush"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "traffic": None, "scope": "whole step (counted FLOPs)",
                     "peak_source": peak_src},
        "cpu_baseline": {"value": round(rows / t_cpu, 2), "unit": "tokens/s",
                         "cores": host_threads(), "kind": "oracle",
                         "sample": f"{rows} rows of {name}, fp64 numpy, {t_cpu:.1f} s"},
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def run_jsd(args):
    """Fused linear JSD on one GPU: the headline student head (bf16 BT=1024,
    H=4096, V=128256, dW) against a teacher head of the same shape (its own
    hidden states and weights); CUDA events around exactly K calls."""
    import numpy as np

    import lm_head_projection_b200 as pkg
    from lm_head_projection_b200.workloads import WORKLOADS

    w = WORKLOADS["bf16_bt1024_h4096_v128256"]
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, device=dev)
    tw = w.with_(seed=w.seed + 1000)
    tin = make_inputs(tw, device=dev)
    X, W, Xt, Wt = inp["X"], inp["W"], tin["X"], tin["W"]
    beta = 0.5
    r0 = pkg.jsd_forward_backward(X, W, None, Xt, Wt, None, beta=beta, compute_dW=True,
                                  check_status=True)
    ws = r0["workspace"]
    p = lambda t: None if t is None else t.data_ptr()
    stream = torch.cuda.current_stream(dev)
    a = (p(X), p(W), None, p(Xt), p(Wt), None, None, -100, w.BT, w.H, w.H, w.V, 1, 1.0, beta,
         0, True, False, True, p(r0["loss"]), p(r0["dX"]), p(r0["dW"]), None, p(ws),
         ws.numel(), stream.cuda_stream)

    def step():
        s = pkg.flkl_jsd_forward_backward(*a)
        if s != 0:
            raise pkg.FlklError(s, "flkl_jsd_forward_backward")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    time.sleep(0.3)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.stop()
    if pkg.flkl_device_status(p(ws), stream.cuda_stream) != 0:
        raise pkg.FlklError(4, "device status after the timed region")
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_src = load_peaks()
    # counted: teacher and student logits, dX and dW; executed: 8 such GEMMs
    counted = 2.0 * w.BT * w.V * w.H * 4
    achieved = counted / (ms * 1e-3) / 1e12
    from oracle import jsd_forward_backward as oracle_jsd
    rows = min(args.cpu_sample_rows, 256)
    f = lambda t: t[:rows].float().cpu().numpy().astype(np.float64)
    Wh, Wth = W.float().cpu().numpy().astype(np.float64), Wt.float().cpu().numpy().astype(
        np.float64)
    t0 = time.perf_counter()
    oracle_jsd(f(X), Wh, None, f(Xt), Wth, None, beta=beta, compute_dW=True)
    t_cpu = time.perf_counter() - t0
    line = {
        "metric": "fused linear JSD fwd+bwd tokens/s", "value": round(w.BT / (ms * 1e-3), 1),
        "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "jsd_bf16_bt1024_h4096_ht4096_v128256", "BT": w.BT, "H": w.H,
                   "Ht": w.H, "V": w.V, "beta": beta, "compute_dW": True,
                   "l2": "inputs larger than L2 (W, Wt), no flush"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "traffic": None,
                     "scope": "whole call; counted = teacher + student logits, dX, dW "
                              "(8 GEMMs of that size run)", "peak_source": peak_src},
        "cpu_baseline": {"value": round(rows / t_cpu, 2), "unit": "tokens/s",
                         "cores": host_threads(), "kind": "oracle",
                         "sample": f"{rows} rows, fp64 numpy, {t_cpu:.1f} s"},
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def run_calls(args):
    """A few plain calls of one workload (for profilers such as ncu): inputs
    drawn on the device, each call timed with CUDA events, device status
    checked at the end."""
    import lm_head_projection_b200 as pkg

    w = ALL_WORKLOADS[args.workload]
    if args.rows:
        w = w.with_(BT=args.rows)
    dev = torch.device("cuda", 0)
    inp = make_inputs(w, device=dev)
    r, times = None, []
    for _ in range(args.calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if w.ce:
            r = pkg.cross_entropy_forward_backward(
                inp["X"], inp["W"], inp["b"], inp["target"], inp["ignore_index"],
                inp["temperature"], inp["reduction"], compute_dW=inp["compute_dW"],
                compute_db=inp["compute_db"], accum_fp32=inp["accum_fp32"], out=r,
                workspace=None if r is None else r["workspace"])
        else:
            r = pkg.forward_backward(inp["X"], inp["W"], inp["b"], inp["Q"], inp["shift_labels"],
                                     inp["ignore_index"], inp["temperature"], inp["eps"],
                                     inp["reduction"], compute_dW=inp["compute_dW"],
                                     compute_db=inp["compute_db"], accum_fp32=inp["accum_fp32"],
                                     out=r, workspace=None if r is None else r["workspace"])
        e1.record()
        torch.cuda.synchronize()
        times.append(round(e0.elapsed_time(e1), 4))
    status = pkg.flkl_device_status(r["workspace"].data_ptr(),
                                    torch.cuda.current_stream().cuda_stream) if r else 0
    print(json.dumps({"workload": w.name, "BT": w.BT, "H": w.H, "V": w.V, "ms": times,
                      "status": status}), flush=True)
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    a = parse()
    if a.calls > 0:
        run_calls(a)
    elif a.op == "jsd":
        run_jsd(a)
    elif a.op == "logprob":
        run_logprob(a)
    elif a.op != "loss":
        run_norm(a)
    elif a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
