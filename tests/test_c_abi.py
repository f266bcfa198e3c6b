"""The boundary as a C program sees it: include/sage.h compiles as C99 with warnings
as errors, and a program linked against libsage.so calls the host-side entry points
(no GPU needed: sizes, the host-pipeline workspace, argument validation)."""

import os
import shutil
import subprocess

import pytest

from quantized_attention_06_b200 import _lib as L
from quantized_attention_06_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "sage.h"

int main(void) {
  sage_problem_t p;
  memset(&p, 0, sizeof(p));
  p.batch = 2; p.heads_q = 4; p.heads_kv = 2; p.seqlen = 300; p.head_dim = 128;
  p.dtype = SAGE_FP16; p.cu_seqlens_host = NULL; p.granularity = SAGE_GRAN_BLOCK;
  sage_sizes_t s;
  if (sage_buffer_sizes(&p, &s) != SAGE_OK) return 1;
  if (s.t_pad != 768 || s.q8 != 4u * 768u * 128u || s.k_scale != 2u * (768u / 64u) * 4u) return 2;
  p.granularity = SAGE_GRAN_THREAD;
  if (sage_buffer_sizes(&p, &s) != SAGE_OK || s.q_scale != 4u * 768u * 4u) return 3;
  if (sage_host_workspace_bytes(&p, 1, SAGE_FP16) == 0) return 4;
  p.head_dim = 96;
  if (sage_buffer_sizes(&p, &s) != SAGE_ERR_UNSUPPORTED) return 5;
  p.head_dim = 128;
  int32_t cu[3] = {0, 100, 300};
  p.cu_seqlens_host = cu;
  if (sage_attn_host(&p, 0, &cu, &cu, &cu, &cu, SAGE_FP16, 0.0f, 0, 0, &cu, 1, NULL) !=
      SAGE_ERR_INVALID_ARGUMENT) return 6;
  if (sage_debug_watchdog_selftest(0, NULL) != SAGE_ERR_INVALID_ARGUMENT) return 7;
  if (strcmp(sage_status_string(SAGE_ERR_TOO_LARGE), "SAGE_ERR_TOO_LARGE") != 0) return 8;
  printf("c-abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_compiles_links_and_calls_the_host_entry_points(tmp_path):
    lib = build.build()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), lib, f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.strip() == "c-abi ok"
    assert os.path.basename(L.LIB_PATH) == os.path.basename(lib)
