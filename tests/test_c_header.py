"""The boundary from plain C: a C11 program that includes include/rmm.h,
links librmm.so and calls the host-side entry points (keep count, workspace
size, argument validation, error strings) compiles without warnings and runs
without a GPU. Shows that the header is C, not C++, and that a caller needs
neither Python nor torch."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

from input_adaptive_reduced_02_b200 import rmm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "rmm.h"

static int fails = 0;
#define CHECK(c) do { if (!(c)) { printf("FAIL line %d: %s\n", __LINE__, #c); ++fails; } } while (0)

int main(void) {
  /* k = ceil(rho * K); rho outside (0, 1] is -1 */
  CHECK(rmm_keep_count(0.5, 4096) == 2048);
  CHECK(rmm_keep_count(0.3, 4096) == 1229);
  CHECK(rmm_keep_count(1.0, 7) == 7);
  CHECK(rmm_keep_count(0.0, 10) == -1);
  CHECK(rmm_keep_count(1.5, 10) == -1);
  /* the workspace of the linear workload: status, scores, indices, A_S, B_S */
  CHECK(rmm_workspace_size(1, 4096, 4096, 4096, 2048, RMM_BF16) ==
        (size_t)1024 + 4096 * 4 + 2048 * 4 + (size_t)4096 * 2048 * 2 * 2);
  /* argument errors come back before any device work */
  void* p = (void*)(uintptr_t)1024;
  rmm_status st = rmm_matmul_reduced(p, 8, p, 8, 4, 8, 8, 1.5, RMM_BF16, RMM_SCORE_PRODUCT, p, 8, RMM_F32,
                                     NULL, p, (size_t)1 << 20, (cudaStream_t)0);
  CHECK(st == RMM_ERR_INVALID);
  CHECK(strstr(rmm_last_error_string(), "rho") != NULL);
  CHECK(rmm_select((const float*)p, 1, 10, 11, (int32_t*)p, NULL, (cudaStream_t)0) == RMM_ERR_INVALID);
  CHECK(rmm_select(NULL, 0, 10, 3, NULL, NULL, (cudaStream_t)0) == RMM_OK);  /* empty batch */
  CHECK(rmm_gemv_gather(p, 8, 0, p, 8, 0, 1, 17, 8, 8, (const int32_t*)p, 3, RMM_BF16, p, 8, 0, RMM_F32,
                        (cudaStream_t)0) == RMM_ERR_INVALID);  /* M above 16 */
  printf("%s\n", fails ? "FAILED" : "C ABI OK");
  return fails != 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INC), reason="needs gcc and CUDA headers")
def test_header_compiles_as_c_and_host_calls_work(tmp_path):
    rmm.lib()  # fails loudly if the library has not been built
    lib = rmm.library_path()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    cc = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                         "-I", CUDA_INC, str(src), "-o", str(exe), "-L", libdir, "-l:librmm.so",
                         f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and "C ABI OK" in run.stdout, run.stdout + run.stderr
