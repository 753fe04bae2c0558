"""The header is plain C: a C99 program that includes only include/svdq.h
compiles with -Wall -Werror, links against libsvdq.so and calls the
host-only entry points (no GPU needed): version, scale-buffer size, status
strings, and argument validation that fails before anything is enqueued."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "svdquant_w4a4_gemm_b200", "lib")

PROGRAM = r"""
#include <stdio.h>
#include "svdq.h"

int main(void) {
  printf("version %d\n", svdq_version());
  printf("scale_bytes %zu\n", svdq_nvfp4_scale_bytes(4096, 3072));
  printf("ok_string %s\n", svdq_status_string(SVDQ_OK));
  /* K not a multiple of 64: rejected on the host, nothing is enqueued */
  svdq_status st = svdq_quantize_act((const void*)16, 4, 96, 96, NULL, NULL, 0, (const float*)16,
                                     NULL, (uint8_t*)16, (uint8_t*)16, NULL, NULL);
  printf("status %d %s\n", (int)st, st == SVDQ_ERR_INVALID_ARG ? "invalid_arg" : "other");
  printf("detail %s\n", svdq_last_error_detail());
  void* ys[3] = {(void*)16, (void*)16, (void*)16};
  st = svdq_w4a4_linear_split(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL, 4, 384, 64, 3,
                              ys, 128, SVDQ_ACT_GELU_TANH, NULL);
  printf("split %s\n", st == SVDQ_ERR_INVALID_ARG ? "invalid_arg" : "other");
  printf("workspace %d\n", SVDQ_QUANTIZE_WORKSPACE_BYTES);
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(tmp_path):
    if not os.path.exists(os.path.join(LIBDIR, "libsvdq.so")):
        import svdquant_w4a4_gemm_b200.build as b
        b.build()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", LIBDIR, "-lsvdq", f"-Wl,-rpath,{LIBDIR}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    assert "scale_bytes 786432" in out
    assert "status 1 invalid_arg" in out and "K=96" in out
    assert "split invalid_arg" in out
    assert "workspace 16" in out
    assert int(out.split("version ")[1].split()[0]) >= 100
