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


def code_only(src: str) -> str:
    """C / CUDA source without its comments and blank space (string and
    character literals kept as they are), so that editing a comment does not
    count as a change of the code."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if src.startswith("//", i):
            i = src.find("\n", i)
            i = n if i < 0 else i
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the code (comments and blank space left out) of the CUDA
    sources the fused-loss kernels are built from."""
    import hashlib

    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lm_head_projection_b200", "csrc")
    for fn in GEMM_SOURCES:
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode() + b"\0" + code_only(f.read()).encode())
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
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip timing the other bf16 workloads after the headline")
    ap.add_argument("--op", default="loss",
                    choices=["loss", "rms_norm", "layer_norm", "logprob", "jsd", "memory"],
                    help="loss: the fused linear KL / CE loss (default); rms_norm / "
                         "layer_norm: the norm backward with frozen-parameter flags; logprob: "
                         "selective log-probability forward + backward on a CE workload; "
                         "jsd: fused linear JSD with a teacher head of the same shape; "
                         "memory: peak device memory of one call at the pages' head shape")
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
    """nvidia-smi clocks and throttle reasons every 20 ms in the background;
    summary() keeps the samples taken between mark_start() and mark_end()
    (the timed region), by nvidia-smi's own timestamps."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="flkl_clocks_", suffix=".csv")
        self.proc = None
        self.t0 = self.t1 = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(gpu_index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        import datetime

        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[4], parts[5:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        inside = [r for r in rows if self.t0 is not None and self.t1 is not None
                  and self.t0 <= r[0] <= self.t1]
        window = "timed region"
        if not inside:  # a region shorter than the sampling period: the nearest sample after it
            after = [r for r in rows if self.t1 is not None and r[0] >= self.t1]
            inside, window = (after[:1] or rows[-1:]), "first sample after the timed region"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[4][1:5])
                          if v.lower() == "active"})
        power = [float(r[3]) for r in inside if r[3].replace(".", "", 1).isdigit()]
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": rows[0][2],
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_median": statistics.median(power) if power else None}


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

class Case:
    """One workload's inputs, outputs and the raw C-ABI arguments of its call
    (the public API is called once to allocate outputs and the workspace)."""

    def __init__(self, pkg, w, dev, stream):
        self.pkg, self.w, self.stream = pkg, w, stream
        inp = make_inputs(w, device=dev)
        self.inp = inp
        X, W, b, Q, lab = inp["X"], inp["W"], inp["b"], inp["Q"], inp["shift_labels"]
        tgt = inp.get("target")
        self.compute_db = inp["compute_db"]
        r0 = self.api_call(check_status=True)
        self.ws = r0["workspace"]
        self.out = {k: r0[k] for k in ("loss", "dX", "dW", "db")}
        p = lambda t: None if t is None else t.data_ptr()
        dt_code = pkg.DTYPES[X.dtype]
        out, ws = self.out, self.ws
        self.kl_args = (p(X), p(W), p(b), p(Q), p(lab), inp["ignore_index"], w.BT, w.H, w.V,
                        dt_code, inp["temperature"], inp["eps"],
                        pkg.REDUCTIONS[inp["reduction"]], inp["compute_dW"], self.compute_db,
                        inp["accum_fp32"], p(out["loss"]), p(out["dX"]), p(out["dW"]),
                        p(out["db"]), p(ws), ws.numel(), stream.cuda_stream)
        self.ce_args = (p(X), p(W), p(b), p(tgt), inp["ignore_index"], w.BT, w.H, w.V, dt_code,
                        inp["temperature"], pkg.REDUCTIONS[inp["reduction"]],
                        inp["compute_dW"], self.compute_db, inp["accum_fp32"], p(out["loss"]),
                        p(out["dX"]), p(out["dW"]), p(out["db"]), p(ws), ws.numel(),
                        stream.cuda_stream)
        self.tgt_ptr = p(tgt)

    def api_call(self, out=None, workspace=None, check_status=False):
        """The public Python API call a user makes for this workload."""
        pkg, w, inp = self.pkg, self.w, self.inp
        if w.ce:
            return pkg.cross_entropy_forward_backward(
                inp["X"], inp["W"], inp["b"], inp["target"], inp["ignore_index"],
                inp["temperature"], inp["reduction"], compute_dW=inp["compute_dW"],
                compute_db=self.compute_db, accum_fp32=inp["accum_fp32"], out=out,
                workspace=workspace, check_status=check_status)
        return pkg.forward_backward(inp["X"], inp["W"], inp["b"], inp["Q"], inp["shift_labels"],
                                    inp["ignore_index"], inp["temperature"], inp["eps"],
                                    inp["reduction"], compute_dW=inp["compute_dW"],
                                    compute_db=self.compute_db, accum_fp32=inp["accum_fp32"],
                                    out=out, workspace=workspace, check_status=check_status)

    def call(self) -> int:
        pkg = self.pkg
        return (pkg.flkl_ce_forward_backward(*self.ce_args) if self.w.ce
                else pkg.flkl_forward_backward(*self.kl_args))

    def profiled_steps(self, steps: int, cap: int = 32, before=None):
        """`steps` calls through the profiled entry, events around every
        launch, no synchronisation between calls (the same back-to-back launch
        stream as the timed steps); `before()` runs right before the first
        call (after the events are ready).  Returns per-kind [ms, launches,
        GEMM FLOPs], the launches per call, and the elapsed ms per call from
        the first event to the last."""
        pkg, st = self.pkg, self.stream
        events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * cap * steps)]
        for e in events:  # torch creates the CUDA event on its first record
            e.record(st)
        torch.cuda.synchronize()
        if before is not None:
            before()
        recs = []
        for i in range(steps):
            r = pkg.flkl_forward_backward_profiled(*self.kl_args,
                                                   events[2 * cap * i: 2 * cap * (i + 1)], cap,
                                                   ce_target=self.tgt_ptr)
            if r[0] != 0:
                raise pkg.FlklError(r[0], "flkl_forward_backward_profiled")
            if r[3] > cap:
                raise RuntimeError(f"{r[3]} launches per call exceed the {cap} recorded")
            recs.append(r)
        torch.cuda.synchronize()
        per_kind = {}
        for i, (_, kinds, flops, n) in enumerate(recs):
            base = 2 * cap * i
            for j, k in enumerate(kinds):
                d = per_kind.setdefault(pkg.LAUNCH_KINDS[k], [0.0, 0, 0.0])
                d[0] += events[base + 2 * j].elapsed_time(events[base + 2 * j + 1])
                d[1] += 1
                d[2] += flops[j]
        n = recs[0][3]
        elapsed = events[0].elapsed_time(events[2 * cap * (steps - 1) + 2 * n - 1])
        return per_kind, n, elapsed / steps


def sm_clock_summary(buf: torch.Tensor, window_ms: float):
    """Median, 10th and 90th percentile SM clock (MHz) of a flkl_clock_trace
    record over its first `window_ms`."""
    a = buf.cpu().tolist()
    t, c = a[0::2], a[1::2]
    mhz = []
    for i in range(1, len(t)):
        if t[i] - t[0] > window_ms * 1e6:
            break
        if t[i] > t[i - 1]:
            mhz.append((c[i] - c[i - 1]) / (t[i] - t[i - 1]) * 1e3)
    if not mhz:
        return None
    mhz.sort()
    return {"median": round(statistics.median(mhz)), "p10": round(mhz[len(mhz) // 10]),
            "p90": round(mhz[(9 * len(mhz)) // 10]), "samples": len(mhz)}


def timed_steps(case, steps, barrier=lambda: None, before=None):
    """Exactly `steps` calls between two events on the launch stream, with a
    barrier and a synchronisation on both sides; `before()` runs after the
    first synchronisation, right before the first event; returns elapsed
    ms."""
    st = case.stream
    barrier()
    torch.cuda.synchronize()
    if before is not None:
        before()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        s = case.call()
        if s != 0:
            raise case.pkg.FlklError(s, "flkl_forward_backward")
    e1.record(st)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1)


def kernel_roofline(w, per_kind, steps, peaks, peaks_src, ms_per_step):
    """Roofline of the dominant kernel, tc_group_kernel (every GEMM launch of
    a step: pass 1, pass 2 of the first chunk and one grouped launch per
    vocabulary chunk), over a step: the method's counted FLOPs (one logits
    GEMM, dX and dW when trained: 2*BT*H*V each) per step over the kernel's
    device time per step, against the measured burst bf16 peak (the timed
    region is a few hundred ms at most); the executed FLOPs (adding the
    recompute of the logits in pass 2) are reported beside it."""
    gemm_kinds = [k for k, v in per_kind.items() if v[2] > 0]
    gemm_ms = sum(per_kind[k][0] for k in gemm_kinds) / steps
    launches = sum(per_kind[k][1] for k in gemm_kinds) / steps
    executed = sum(per_kind[k][2] for k in gemm_kinds) / steps
    counted = w.flops_counted()
    burst = peaks["bf16_tflops"]
    sust = peaks.get("bf16_tflops_sustained", burst)
    achieved = counted / (gemm_ms * 1e-3) / 1e12
    traffic = None
    parts = {k: dram_traffic(w.name, k) for k in gemm_kinds}
    if all(v is not None for v in parts.values()) and parts:
        traffic = sum(parts[k] * per_kind[k][1] / steps for k in gemm_kinds)
    algo = algorithmic_bytes(w)
    kind_name = "tc_group_kernel" if w.dtype == "bf16" else "k_simt_* (fp32 FMA)"
    return {
        "bound": "tensor" if w.dtype == "bf16" else "alu", "kernel": kind_name,
        "unit_of_work": "one step's launches of the kernel "
                        f"({launches:g} per step: {', '.join(sorted(gemm_kinds))})",
        "achieved": round(achieved, 1), "peak": burst, "unit": "TFLOP/s",
        "frac": round(achieved / burst, 4),
        "peak_note": f"bf16_tflops (burst) of {peaks_src} MEASURED_PEAKS.json",
        "counted_flops_per_step": counted, "executed_flops_per_step": executed,
        "executed_tflops": round(executed / (gemm_ms * 1e-3) / 1e12, 1),
        "frac_executed_of_burst": round(executed / (gemm_ms * 1e-3) / 1e12 / burst, 4),
        "frac_of_sustained": round(achieved / sust, 4),
        "kernel_ms_per_step": round(gemm_ms, 4),
        "share_of_step": round(gemm_ms / ms_per_step, 4),
        "traffic": traffic, "algorithmic_bytes": algo,
        "traffic_ratio": None if traffic is None else round(traffic / algo, 3),
        "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch kind "
                          f"(profiles/traffic_{w.name}.md) x launches per step"
                          if traffic is not None else
                          "none on file for the current kernel sources",
    }


def step_roofline(w, ms_per_step, peaks, peaks_src, executed=None):
    """Counted FLOPs of the step against the burst and sustained peaks.  The
    cap is the fraction the pass-2 recompute leaves: counted over executed
    GEMM FLOPs per step (from the library's profiled entry when `executed` is
    given; else with every chunk recomputed)."""
    counted = w.flops_counted()
    sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    t_burst = max(counted / (peaks["bf16_tflops"] * 1e12), algorithmic_bytes(w) / (peaks["hbm_gbs"] * 1e9))
    t_sust = max(counted / (sust * 1e12), algorithmic_bytes(w) / (peaks["hbm_gbs"] * 1e9))
    return {"counted_flops": counted,
            "tflops": round(counted / (ms_per_step * 1e-3) / 1e12, 1),
            "frac_of_burst": round(t_burst / (ms_per_step * 1e-3), 4),
            "frac_of_sustained": round(t_sust / (ms_per_step * 1e-3), 4),
            "cap_with_recompute": round(counted / executed, 4) if executed else
            round((2 + int(w.compute_dW)) / (3 + int(w.compute_dW)), 4),
            "peaks": peaks_src}


def breakdown(per_kind, steps, ms_per_step):
    total = sum(v[0] for v in per_kind.values())
    out = {k: {"ms_per_step": round(v[0] / steps, 4),
               "launches_per_step": round(v[1] / steps, 2),
               "share_of_kernel_time": round(v[0] / total, 4),
               "executed_tflops": round(v[2] / (v[0] * 1e-3) / 1e12, 1) if v[2] else None}
           for k, v in sorted(per_kind.items())}
    return out, total / steps


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
    stream = torch.cuda.current_stream(dev)
    case = Case(pkg, w, dev, stream)
    inp, out, ws = case.inp, case.out, case.ws
    X, W, b, Q, lab = inp["X"], inp["W"], inp["b"], inp["Q"], inp["shift_labels"]
    tgt = inp.get("target")
    compute_db = case.compute_db
    p = lambda t: None if t is None else t.data_ptr()

    n_total = torch.zeros((), dtype=torch.int64, device=dev)
    mask = tgt if w.ce else lab
    exchanged = [t for t in (out["loss"], out["dW"], out["db"]) if t is not None]

    def step():
        if not args.dp:
            s = case.call()
        else:
            # the data-parallel step of lm_head_projection_b200.dp, raw entry points
            s = pkg.flkl_count_valid(p(mask), w.BT, inp["ignore_index"], p(n_total),
                                     stream.cuda_stream)
            if s == 0:
                if world > 1:
                    dist.all_reduce(n_total)
                s = (pkg.flkl_ce_forward_backward_dp(*case.ce_args, p(n_total)) if w.ce
                     else pkg.flkl_forward_backward_dp(*case.kl_args, p(n_total)))
            if s == 0 and world > 1:
                for t in exchanged:
                    dist.all_reduce(t)
        if s != 0:
            raise pkg.FlklError(s, "flkl_forward_backward")

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
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
    clocks.mark_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    barrier()
    clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    status = pkg.flkl_device_status(ws.data_ptr(), stream.cuda_stream)
    if status != 0:
        raise pkg.FlklError(status, "device status after the timed region")
    clk = clocks.summary()
    ms_per_step = ms / args.steps

    # ---------------- per-launch breakdown: K more steps through the profiled
    # entry, back to back as in the timed region (no synchronisation between
    # steps), with the in-kernel SM clock sampled next to them
    trace_n = 4096
    trace_iv = max(1000, int(ms_per_step * args.steps * 1e6 * 1.5 / trace_n))
    trace = torch.zeros(2 * trace_n, dtype=torch.int64, device=dev)
    side = torch.cuda.Stream(dev)
    torch.cuda.synchronize()
    per_kind, launches_per_step, prof_ms = case.profiled_steps(
        args.steps, before=lambda: pkg.flkl_clock_trace(trace.data_ptr(), trace_n, trace_iv,
                                                        side.cuda_stream))
    torch.cuda.synchronize()
    sm_clock = sm_clock_summary(trace, prof_ms * args.steps)
    if pkg.flkl_device_status(ws.data_ptr(), stream.cuda_stream) != 0:
        raise pkg.FlklError(4, "device status after the profiled steps")
    kinds, kernel_sum = breakdown(per_kind, args.steps, ms_per_step)
    peaks, peaks_src = load_peaks()
    roofline = kernel_roofline(w, per_kind, args.steps, peaks, peaks_src, ms_per_step)
    sroof = step_roofline(w, ms_per_step, peaks, peaks_src,
                          executed=sum(v[2] for v in per_kind.values()) / args.steps)
    breakdown_check = {
        "profiled_ms_per_step": round(prof_ms, 4),
        "kernel_sum_ms_per_step": round(kernel_sum, 4),
        "kernel_sum_over_timed_step": round(kernel_sum / ms_per_step, 4),
        "note": "the profiled steps run back to back like the timed ones; the kernel sum "
                "leaves out the gaps between launches"}

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
    tokens = w.BT * world
    e2e = {"value": round(tokens / (e2e_ms / args.steps * 1e-3), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4}
    del pipe

    # ---------------- the other bf16 workloads, same process (rank 0, N = 1)
    others = None
    if (rank == 0 and world == 1 and not args.dp and not args.no_other_workloads
            and args.workload == HEADLINE):
        others = {}
        for name in OTHER_WORKLOADS:
            try:
                others[name] = measure_other(pkg, ALL_WORKLOADS[name], dev, stream, args,
                                             peaks, peaks_src, gpu_index)
            except Exception as exc:  # keep the headline line whatever happens here
                others[name] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            torch.cuda.empty_cache()

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
        value = tokens / (ms_per_step * 1e-3)
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": w.name, "global_batch": w.BT * world, "BT_per_gpu": w.BT,
                       "H": w.H, "V": w.V, "compute_dW": w.compute_dW,
                       "compute_db": bool(compute_db), "reduction": w.reduction,
                       "temperature": w.temperature,
                       "parallelism": f"dp{world}" + ("-allreduce" if args.dp else "-replicas"),
                       "l2": "inputs larger than L2 (W, Q), no flush"},
            "e2e": e2e, "roofline": roofline, "step_roofline": sroof,
            "kernels": kinds, "breakdown_check": breakdown_check,
            "gpu_launches": int((launches_per_step + (1 if args.dp else 0)) * args.steps),
            "clocks": clk, "sm_clock_in_kernel_mhz": sm_clock,
            "gemm_ctas": pkg.flkl_gemm_ctas(),
            "other_workloads": others, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


OTHER_WORKLOADS = ("bf16_bt2048_h4096_v128256_frozen_ignore_t2_sum",
                   "bf16_bt4096_h4096_v128256_bias_mean_peaked",
                   "bf16_bt8192_h4096_v151936_frozen")


def measure_other(pkg, w, dev, stream, args, peaks, peaks_src, gpu_index):
    """One more bf16 workload in the same process: 3 warm-up calls, then
    min(K, 10) timed calls (CUDA events, inputs larger than L2), the in-kernel
    SM clock next to them and nvidia-smi clocks during them."""
    case = Case(pkg, w, dev, stream)
    steps = max(1, min(args.steps, 10))
    for _ in range(3):
        if case.call() != 0:
            raise pkg.FlklError(1, w.name)
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_index)
    time.sleep(0.3)
    trace_n = 2048
    est = 2.0 * w.flops_counted() / 1e15 * 1e3  # ms per step at 0.5 PFLOP/s, generous
    trace_iv = max(1000, int(est * steps * 1e6 * 1.5 / trace_n))
    trace = torch.zeros(2 * trace_n, dtype=torch.int64, device=dev)
    side = torch.cuda.Stream(dev)
    torch.cuda.synchronize()
    clocks.mark_start()
    ms = timed_steps(case, steps, before=lambda: pkg.flkl_clock_trace(
        trace.data_ptr(), trace_n, trace_iv, side.cuda_stream))
    torch.cuda.synchronize()
    clocks.mark_end()
    clocks.stop()
    if pkg.flkl_device_status(case.ws.data_ptr(), stream.cuda_stream) != 0:
        raise pkg.FlklError(4, w.name)
    msps = ms / steps
    per_kind, _, _ = case.profiled_steps(1)  # the GEMM FLOPs one call executes
    res = {"steps": steps, "warmup": 3, "ms_per_step": round(msps, 4),
           "tokens_per_s": round(w.BT / (msps * 1e-3), 1),
           "step_roofline": step_roofline(w, msps, peaks, peaks_src,
                                          executed=sum(v[2] for v in per_kind.values())),
           "clocks": clocks.summary(), "sm_clock_in_kernel_mhz": sm_clock_summary(trace, ms)}
    del case
    return res


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
    clocks.mark_start()
    for a, b in evs:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
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
    clocks.mark_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
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
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "traffic": None, "scope": "whole step (counted FLOPs), burst peak",
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
    clocks.mark_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    clocks.stop()
    if pkg.flkl_device_status(p(ws), stream.cuda_stream) != 0:
        raise pkg.FlklError(4, "device status after the timed region")
    ms = e0.elapsed_time(e1) / args.steps
    peaks, peak_src = load_peaks()
    # counted: teacher and student logits, dX and dW; executed: 8 such GEMMs
    # less the first vocabulary chunk's four (formed from the kept logits)
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
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                     "traffic": None,
                     "scope": "whole call; counted = teacher + student logits, dX, dW "
                              "(8 GEMMs of that size run, less the first vocabulary "
                              "chunk's four chunk-sized ones); burst peak",
                     "peak_source": peak_src},
        "cpu_baseline": {"value": round(rows / t_cpu, 2), "unit": "tokens/s",
                         "cores": host_threads(), "kind": "oracle",
                         "sample": f"{rows} rows, fp64 numpy, {t_cpu:.1f} s"},
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def run_memory(args):
    """Peak device memory of one fused forward + backward at the pages' head
    shape (bf16, H=4096, V=128256, trained head) for BT = 1024, 2048, 4096:
    through the C-ABI call (inputs, outputs and workspace) and through the
    autograd module (loss.backward() filling X.grad and W.grad), with the head
    gradient kept in bf16 and in fp32 (accum_dtype)."""
    import lm_head_projection_b200 as pkg

    dev = torch.device("cuda", 0)
    mb = lambda n: round(n / 2**20, 1)
    rows = []
    for BT in (1024, 2048, 4096):
        for accum in (False, True):
            w = WORKLOADS[HEADLINE].with_(BT=BT, accum_fp32=accum)
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            base = torch.cuda.memory_allocated(dev)
            inp = make_inputs(w, device=dev)
            torch.cuda.synchronize()
            in_bytes = torch.cuda.memory_allocated(dev) - base
            torch.cuda.reset_peak_memory_stats(dev)
            r = pkg.forward_backward(inp["X"], inp["W"], None, inp["Q"], compute_dW=True,
                                     accum_fp32=accum, check_status=True)
            torch.cuda.synchronize()
            call_peak = torch.cuda.max_memory_allocated(dev) - base
            ws = r["workspace"].numel()
            out_bytes = sum(t.numel() * t.element_size() for k, t in r.items()
                            if k != "workspace" and t is not None)
            del r
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            torch.cuda.reset_peak_memory_stats(dev)
            X = inp["X"].clone().requires_grad_()
            Wp = inp["W"].clone().requires_grad_()
            del inp["X"], inp["W"]
            mod = pkg.FusedLinearKLDivLoss(accum_dtype=torch.float32 if accum else None)
            loss = mod(Wp, X, inp["Q"])
            loss.backward()
            torch.cuda.synchronize()
            module_peak = torch.cuda.max_memory_allocated(dev) - base
            rows.append({"BT": BT, "head_grad": "fp32" if accum else "bf16",
                         "inputs_mb": mb(in_bytes), "outputs_mb": mb(out_bytes),
                         "workspace_mb": mb(ws), "call_peak_mb": mb(call_peak),
                         "module_fwd_bwd_peak_mb": mb(module_peak)})
            del X, Wp, loss, inp, mod
    line = {"metric": "peak device memory of one fused fwd+bwd (MiB)", "unit": "MiB",
            "higher_is_better": False, "n_gpus": 1, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "bf16_h4096_v128256_trained", "BT": [1024, 2048, 4096]},
            "rows": rows,
            "context": "the pages' fused kernel on an RTX 4060 Laptop: 4244 (BT 1024, "
                       "benchmark harness), 4310 (BT 2048), 6594 (BT 4096) MB, another machine "
                       "and implementation"}
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
    elif a.op == "memory":
        run_memory(a)
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
