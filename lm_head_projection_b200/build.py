"""Builds the CUDA library in-tree: lm_head_projection_b200/_flkl.so (sm_100a).

    python -m lm_head_projection_b200.build [--verbose-ptxas]
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "_flkl.so")
SOURCES = ["flkl_api.cu", "norm_api.cu"]
HEADERS = ["ptx.cuh", "tc_gemm.cuh", "row_kernels.cuh", "simt_f32.cuh", "norm_bwd.cuh",
           "jsd_kernels.cuh"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_rebuild() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "flkl.h"))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not needs_rebuild():
        return LIB
    cmd = [
        nvcc_path(), "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"),
        "-o", LIB + ".tmp",
    ] + [os.path.join(CSRC, s) for s in SOURCES]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
