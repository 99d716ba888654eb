"""The boundary is a C ABI: include/sbattn.h compiles as plain C99 (gcc, no
CUDA or torch headers) and a C program links the shared library and calls
its host-only entry points and argument checks.  No GPU is touched: every
call below returns before launching anything."""

import os
import shutil
import subprocess

import pytest

from block_sparse_attention_qk_b200 import build as sb_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include "sbattn.h"

int main(void) {
  int K = 0;
  int rc = sbattn_keep_count(1953, 0.75, &K);
  if (rc != SBATTN_OK || K != 489) { printf("keep_count rc=%d K=%d\n", rc, K); return 1; }
  if (sbattn_keep_count(1953, 1.5, &K) != SBATTN_ERR_INVALID_ARG) return 2;
  if (sbattn_version() <= 0) return 3;
  if (sbattn_strerror(SBATTN_ERR_MISALIGNED) == NULL) return 4;
  /* null inputs are rejected on the host, before any CUDA call */
  if (sbattn_forward(NULL, NULL, NULL, NULL, NULL, 1, NULL, 1, 64, 1, 128, 0.f, NULL, NULL) != SBATTN_ERR_INVALID_ARG)
    return 5;
  if (sbattn_adaln_modulate(NULL, NULL, NULL, NULL, 1, 1, 8, 1e-6f, NULL) != SBATTN_ERR_INVALID_ARG) return 6;
  if (sbattn_swiglu(NULL, NULL, NULL, 1, 8, 8, NULL) != SBATTN_ERR_INVALID_ARG) return 7;
  if (sbattn_select_workspace_bytes(1, 124992, 40, 128) != (size_t)2 * 40 * 1953 * 128 * 4) return 8;
  /* the status path: a misaligned status word is rejected before any CUDA
     call; with no status word the call only checks the stream, which on a
     machine without a GPU reports a CUDA error instead of crashing */
  if (sbattn_check_status((const int32_t*)(uintptr_t)0x1002, NULL) != SBATTN_ERR_MISALIGNED) return 9;
  rc = sbattn_check_status(NULL, NULL);
  if (rc != SBATTN_OK && rc != SBATTN_ERR_CUDA) { printf("check_status rc=%d\n", rc); return 10; }
  printf("c abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_is_c99_and_library_links(tmp_path):
    so = sb_build.build()
    src = tmp_path / "abi.c"
    src.write_text(C_SOURCE)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(str(so))
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe), "-L", libdir, "-lsbattn", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "c abi ok" in r.stdout
