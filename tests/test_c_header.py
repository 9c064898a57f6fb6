"""include/attn.h is a C header: a plain C99 program compiles against it with
warnings as errors, links against libattn.so, and gets the documented status
codes from the host-side validation (no CUDA call is reached)."""

import os
import shutil
import subprocess

import pytest

from exact_attention_150_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "attn.h"

#define EXPECT(cond) do { if (!(cond)) { printf("FAILED line %d: %s\n", __LINE__, #cond); return 1; } } while (0)

int main(void) {
  static char buf[64];
  void* p = (void*)(((unsigned long)buf + 15u) & ~15ul);  /* 16-byte aligned, never dereferenced */
  const int* cu = (const int*)p;
  EXPECT(strcmp(attn_status_string(ATTN_OK), "ok") == 0);
  EXPECT(attn_fwd(NULL, p, p, p, (float*)p, 1, 1, 128, 128, 64, 0.125f, ATTN_CAUSAL_NONE, ATTN_BF16, NULL)
         == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_fwd(p, p, p, p, (float*)p, 1, 1, 128, 128, 96, 0.125f, ATTN_CAUSAL_NONE, ATTN_BF16, NULL)
         == ATTN_ERR_UNSUPPORTED);
  EXPECT(attn_fwd(p, p, p, p, (float*)p, 1, 1, 128, 128, 64, 0.125f, 7, ATTN_BF16, NULL) == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_fwd(NULL, NULL, NULL, NULL, NULL, 0, 1, 128, 128, 64, 0.125f, ATTN_CAUSAL_TOP_LEFT, ATTN_FP16, NULL)
         == ATTN_OK);
  EXPECT(attn_bwd(p, p, p, p, (const float*)p, p, p, p, p, NULL, 1, 1, 128, 128, 256, 0.1f,
                  ATTN_CAUSAL_BOTTOM_RIGHT, ATTN_BF16, NULL) == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_bwd(p, p, p, p, (const float*)p, p, p, p, p, p, 1, 1, 128, 128, 96, 0.1f,
                  ATTN_CAUSAL_BOTTOM_RIGHT, ATTN_BF16, NULL) == ATTN_ERR_UNSUPPORTED);
  EXPECT(attn_bwd_deterministic(p, p, p, p, (const float*)p, p, NULL, p, p, p, 1, 1, 128, 128, 64, 0.1f,
                                ATTN_CAUSAL_NONE, ATTN_FP16, NULL) == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_bwd_phase(p, p, p, p, (const float*)p, p, p, p, p, p, 1, 1, 128, 128, 64, 0.1f,
                        ATTN_CAUSAL_NONE, ATTN_FP16, 9, NULL) == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_bwd_workspace_bytes(1, 1, 128, 128, 64) > 0);
  EXPECT(attn_bwd_workspace_bytes(0, 1, 128, 128, 64) == 0);
  EXPECT(attn_fwd_varlen(p, p, p, p, (float*)p, NULL, cu, 2, 1, 300, 300, 200, 200, 64, 0.1f,
                         ATTN_CAUSAL_TOP_LEFT, ATTN_BF16, NULL) == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_bwd_varlen(p, p, p, p, (const float*)p, p, p, p, p, p, NULL, cu, 2, 1, 300, 300, 200, 200, 256, 0.1f,
                         ATTN_CAUSAL_NONE, ATTN_BF16, 0, NULL) == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_bwd_varlen_workspace_bytes(2, 1, 300, 200, 64) > 0);
  EXPECT(attn_fwd_fp8(p, p, p, p, (float*)p, 1, 1, 128, 128, 64, 0.1f, 1.f, 1.f, 1.f, ATTN_CAUSAL_NONE, NULL)
         == ATTN_ERR_UNSUPPORTED);
  EXPECT(attn_fwd_fp8(NULL, p, p, p, (float*)p, 1, 1, 128, 128, 128, 0.1f, 1.f, 1.f, 1.f, ATTN_CAUSAL_TOP_LEFT, NULL)
         == ATTN_ERR_INVALID_ARG);
  EXPECT(attn_bwd_noalloc_max_scratch_bytes() > 0);
  EXPECT(attn_selftest_wait_timeout(0, (int*)p, NULL) == ATTN_ERR_INVALID_ARG);
  printf("ok\n");
  return 0;
}
"""


def test_header_compiles_as_c99_and_links(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib = build.build()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-lattn", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", out.stdout + out.stderr
