"""The boundary is plain C: include/ring_attn.h compiles as strict C99, and a
C program links against libring_attn.so and gets the documented statuses
back from calls that are rejected (or are empty) before any device work, so
this runs without a GPU."""

from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "ring_attention_ordered_b200")
LIB = os.path.join(PKG, "libring_attn.so")

C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "ring_attn.h"

int main(void) {
  ra_status s;
  size_t n = 0;
  if (ring_attn_version() < 104) return 1;
  /* n_ring = 0: rejected before any pointer is looked at */
  s = ring_attn_fwd(NULL, NULL, NULL, NULL, NULL, 1, 2, 2, 512, 128, 0, 1, 0.1f, NULL);
  if (s != RA_ERR_INVALID_ARG) return 2;
  if (ring_attn_last_error()[0] == '\0') return 3;
  if (strcmp(ring_attn_status_string(s), "RA_ERR_INVALID_ARG") != 0) return 4;
  if (ring_attn_bwd_workspace_size(1, 2, 512, &n) != RA_OK || n != 4096) return 5;
  /* the FP8 forward takes head dim 128 only */
  s = ring_attn_fwd_fp8(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 2, 2, 512, 64, 4, 1,
                        0.1f, NULL);
  if (s != RA_ERR_UNSUPPORTED) return 6;
  /* empty problems launch nothing and succeed */
  if (ring_attn_quantize_fp8(NULL, NULL, NULL, 0, 512, 2, 128, NULL) != RA_OK) return 7;
  if (ring_attn_merge(NULL, NULL, NULL, NULL, NULL, NULL, 0, 64, NULL) != RA_OK) return 8;
  if (ring_attn_set_schedule(RA_SCHEDULE_HEAD_MAJOR) != RA_OK) return 9;
  if (ring_attn_set_schedule(RA_SCHEDULE_AUTO) != RA_OK) return 10;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_a_c_program_links(tmp_path):
    if not os.path.exists(LIB):
        pytest.skip("library not built")
    src = tmp_path / "abi.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), str(src), "-L", PKG, "-lring_attn",
           f"-Wl,-rpath,{PKG}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.strip() == "ok"
