"""Run the fused linear + KL call on one synthetic shape and print its timing.

    python -m lm_head_projection_b200.run_case --BT 1024 --H 4096 --V 16384 \
        [--dtype bf16] [--frozen] [--bias] [--calls 3] [--workload NAME]

Used for profiling one shape in isolation (e.g. under ncu on a small case):
the inputs follow the workload recipe of ``workloads.small_case`` (or a named
workload), are drawn on the device, and each call is timed with CUDA events.
"""

from __future__ import annotations

import argparse
import json

import torch

import lm_head_projection_b200 as pkg
from lm_head_projection_b200.workloads import WORKLOADS, make_inputs, small_case


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--BT", type=int, default=1024)
    ap.add_argument("--H", type=int, default=4096)
    ap.add_argument("--V", type=int, default=16384)
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--frozen", action="store_true")
    ap.add_argument("--bias", action="store_true")
    ap.add_argument("--calls", type=int, default=3)
    ap.add_argument("--workload", default=None, choices=[None] + list(WORKLOADS))
    a = ap.parse_args()
    if a.workload:
        w = WORKLOADS[a.workload]
    else:
        w = small_case(dtype=a.dtype, BT=a.BT, H=a.H, V=a.V, bias=a.bias,
                       compute_dW=not a.frozen, w_std=0.02)
    dev = torch.device("cuda:0")
    inp = make_inputs(w, device=dev)
    r = None
    times = []
    for _ in range(a.calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        r = pkg.forward_backward(inp["X"], inp["W"], inp["b"], inp["Q"], inp["shift_labels"],
                                 inp["ignore_index"], inp["temperature"], inp["eps"],
                                 inp["reduction"], compute_dW=inp["compute_dW"],
                                 compute_db=inp["compute_db"], accum_fp32=inp["accum_fp32"],
                                 out=None if r is None else r,
                                 workspace=None if r is None else r["workspace"])
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    status = pkg.flkl_device_status(r["workspace"].data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    print(json.dumps({"case": w.name, "BT": w.BT, "H": w.H, "V": w.V, "ms": times,
                      "loss": float(r["loss"].cpu()), "status": status}))
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
