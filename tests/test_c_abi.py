"""The boundary is a real C ABI: a C99 program includes taco_attn.h, links libtaco_attn.so and calls it
(only calls that need no GPU: version, host-side argument rejection and the error message). CPU only."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_kv_cache_tree_b200")
LIB = os.path.join(PKG, "libtaco_attn.so")

C_SOURCE = r"""
#include <stdio.h>
#include <string.h>
#include "taco_attn.h"

int main(void) {
  int ok = 1;
  printf("version %d\n", (int)taco_attn_version());
  /* a NULL q is rejected on the host before any CUDA call */
  taco_status st = paged_tree_attention(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0.125f, NULL, TACO_DTYPE_BF16,
                                        2, 4, 8, 2, 128, 16, 40, 8, NULL);
  ok &= (st == TACO_ERR_INVALID_ARG) && strlen(taco_attn_last_error()) > 0;
  /* an unsupported head_dim */
  st = paged_kv_append((void*)16, (void*)16, (const int32_t*)16, (const int32_t*)16, (void*)16, (void*)16,
                       TACO_DTYPE_F16, 2, 4, 2, 96, 16, 40, 8, NULL);
  ok &= (st == TACO_ERR_UNSUPPORTED);
  /* an empty batch is a no-op */
  st = lookahead_propose((const int32_t*)16, (const int32_t*)16, NULL, 0, (const int32_t*)16, 4, 0, 16,
                         (int32_t*)16, (int32_t*)16, (int32_t*)16, NULL);
  ok &= (st == TACO_OK);
  printf("%s\n", ok ? "c-abi ok" : "c-abi FAILED");
  return ok ? 0 : 1;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_links_and_calls_the_library(tmp_path):
    if not os.path.exists(LIB):
        from paged_kv_cache_tree_b200 import build_lib

        build_lib.build()
    src = tmp_path / "use_taco.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "use_taco"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-L", PKG, "-ltaco_attn", "-Wl,-rpath," + PKG, "-o", str(exe)], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "c-abi ok" in run.stdout
