"""The C ABI from plain C: include/flkl.h compiles as C11 with gcc, a program
links against the built library and calls host-side entry points (sizes,
status strings, argument rejections that return before any launch)."""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "flkl.h"

int main(void) {
  if (flkl_abi_version() != FLKL_ABI_VERSION) return 1;
  if (strcmp(flkl_status_string(FLKL_OK), "ok") != 0) return 2;
  size_t ws = flkl_workspace_size(1024, 4096, 128256, FLKL_DTYPE_BF16, 1, 0);
  if (ws == 0 || ws >= (size_t)1024 * 128256 * 2) return 3;
  if (flkl_workspace_size(-1, 4096, 128256, FLKL_DTYPE_BF16, 1, 0) != 0) return 4;
  if (flkl_jsd_workspace_size(1024, 4096, 4096, 128256, FLKL_DTYPE_BF16, 1, 0) == 0) return 5;
  /* rejected on the host: reduction none, then a bad dtype */
  if (flkl_forward_backward(0, 0, 0, 0, 0, -100, 4, 64, 64, FLKL_DTYPE_BF16, 1.f, 1e-10f,
                            FLKL_REDUCTION_NONE, 0, 0, 1, 0, 0, 0, 0, 0, 0, 0)
      != FLKL_ERR_UNSUPPORTED) return 6;
  if (flkl_forward_backward(0, 0, 0, 0, 0, -100, 4, 64, 64, 7, 1.f, 1e-10f,
                            FLKL_REDUCTION_SUM, 0, 0, 1, 0, 0, 0, 0, 0, 0, 0)
      != FLKL_ERR_INVALID_ARG) return 7;
  if (flkl_rms_norm_backward(0, 0, 0, 4, 4095, FLKL_DTYPE_BF16, 1e-6f, 0, 1, 0, 0, 0, 0, 0)
      == FLKL_OK) return 8;
  printf("c abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_compiles_as_c_and_links(tmp_path):
    import lm_head_projection_b200 as pkg

    lib = pkg.library_path()
    assert os.path.exists(lib)
    src = tmp_path / "abi.c"
    src.write_text(C_SRC)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), "-o", str(exe), lib, f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c abi ok" in r.stdout, (r.returncode, r.stdout, r.stderr)
