"""The boundary is a C ABI: both headers compile as strict C99, a C program links against the
library and gets the host-side results of the entry points (version, status strings, workspace
sizes, argument checks that return before any CUDA call).  CPU only; needs gcc."""
import os
import shutil
import subprocess

import pytest

from async_rl_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "bi_isloss.h"
#include "bi_model.h"

int main(void) {
  if (bi_version() <= 0) return 1;
  if (strcmp(bi_status_string(BI_ERR_BAD_OFFSETS), "BI_ERR_BAD_OFFSETS") != 0) return 2;
  size_t full = bi_workspace_bytes_pstore(2000, 1536, 151936, 64);
  size_t small = bi_workspace_bytes(2000, 1536, 151936, 64);
  if (!(full > small && small > 0 && small == bi_workspace_bytes_min(2000, 1536, 151936, 64))) return 3;
  if (bi_workspace_bytes(-1, 128, 512, 0) != 0) return 4;
  /* argument checks return before any CUDA call */
  const uint16_t* fake = (const uint16_t*)(uintptr_t)(1u << 20);
  int32_t* st = (int32_t*)(uintptr_t)(1u << 21);
  if (bi_gemm_bf16(fake, fake, (uint16_t*)fake, 16, 250, 64, st, NULL) != BI_ERR_UNSUPPORTED_SHAPE) return 5;
  if (bi_rmsnorm(fake, fake, -1.0f, (uint16_t*)(uintptr_t)(1u << 22), 4, 64, st, NULL) != BI_ERR_INVALID_ARG) return 6;
  if (bi_logprob_fwd(NULL, fake, (const int32_t*)fake, 10, 128, 512, (float*)fake, NULL, st, (void*)fake, 1u << 20,
                     NULL) != BI_ERR_INVALID_ARG) return 7;
  bi_loss_cfg cfg = {BI_LOSS_PPO_CLIP, 0.2f, 0.2f, 0.0f, BI_LOSS_STORE_P};
  (void)cfg;
  printf("ok %zu %zu\n", full, small);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_links_and_calls_the_abi(tmp_path):
    build()
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(LIB)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
           "-o", str(exe), "-L", libdir, "-l:" + os.path.basename(LIB), "-Wl,-rpath," + libdir]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    assert proc.returncode == 0, proc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.startswith("ok ")
