"""include/sla.h is a C header: a C99 program that includes it compiles with
warnings as errors, links against libsla.so and calls the entry points that
need no GPU (argument checks, sizes, status strings).  No kernel is launched."""
import os
import shutil
import subprocess

import pytest

from sparse_linear_attention_b200 import sla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SRC = r"""
#include <stdio.h>
#include <string.h>
#include "sla.h"

int main(void) {
  sla_shape s;
  s.B = 1; s.H = 12; s.N = 32760; s.d = 128; s.bq = 128; s.bkv = 64; s.in_dtype = SLA_BF16;
  if (sla_keep_count(0.03, 512) != 15) return 1;
  if (sla_keep_count(0.03, 1182) != 35) return 2;
  if (sla_workspace_size(&s, SLA_MODE_SLA2_TOPK) == 0) return 3;
  if (sla2_attn_bwd_workspace_size(&s) == 0 || sla_attn_bwd_workspace_size(&s) == 0) return 4;
  if (strcmp(sla_status_string(SLA_OK), "SLA_OK") != 0) return 5;
  /* a null shape is refused before anything is launched, with a detail */
  if (sla_route(NULL, NULL, NULL, NULL, NULL, SLA_MODE_SLA2_TOPK, 15, 0, NULL, NULL, NULL, NULL, 0, NULL)
      != SLA_ERR_INVALID_ARG) return 6;
  if (sla_last_error_detail()[0] == '\0') return 7;
  /* an unsupported key block size */
  s.bkv = 32;
  if (sla_workspace_size(&s, SLA_MODE_SLA2_TOPK) != 0) return 8;
  printf("c-abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c_and_links(tmp_path):
    sla.lib()  # libsla.so must exist (built by __graft_entry__.build())
    src = tmp_path / "use_sla.c"
    src.write_text(C_SRC)
    exe = tmp_path / "use_sla"
    libdir = os.path.dirname(sla.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), os.path.join(libdir, "libsla.so"), f"-Wl,-rpath,{libdir}"]
    out = subprocess.run(cmd, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, (run.returncode, run.stderr)
    assert run.stdout.strip() == "c-abi ok"
