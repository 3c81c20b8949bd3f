"""The public header as plain C: a C99 program includes it, links the library
and calls the host-side entry points (no GPU needed).

The header must compile as C with warnings as errors, and the library's
answers through the C linkage must equal those seen through the Python
binding: the workspace sizes, the status strings, and the argument checks
that return before any device work.
"""
import os
import shutil
import subprocess

import pytest

from block_sparse_attention_flash_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

C_SOURCE = r"""
#include <stdio.h>
#include <math.h>
#include "sparse_attn.h"

int main(void) {
  printf("version %d\n", sa_version());
  printf("ok %s\n", sa_status_string(SA_OK));
  printf("invalid %s\n", sa_status_string(SA_ERR_INVALID_ARG));
  printf("mask_ws %zu\n", sa_build_mask_workspace(1, 12, 32760, 128, 64));
  printf("bwd_ws %zu\n", sa_sparse_attn_bwd_workspace(1, 12, 32760));
  printf("host_ws %zu\n", sa_sparse_attn_fwd_host_workspace(75600, 128, 2));
  /* argument checks that return before any device work */
  printf("radial_neg %d\n", (int)sa_radial_mask(-1, 4, 4, 64, NULL, NULL));
  printf("radial_empty %d\n", (int)sa_radial_mask(0, 4, 4, 64, NULL, NULL));
  printf("fwd_neg %d\n", (int)sa_sparse_attn_fwd(NULL, NULL, NULL, -1, 1, 256, 128, 128, NULL, 0, 0, 0, NULL, NULL,
                                                 INFINITY, 0.0f, SA_ORDER_ASCENDING, 0, NULL, NULL, NULL));
  printf("fwd_d96 %d\n", (int)sa_sparse_attn_fwd(NULL, NULL, NULL, 1, 1, 256, 96, 128, NULL, 0, 0, 0, NULL, NULL,
                                                 INFINITY, 0.0f, SA_ORDER_ASCENDING, 0, NULL, NULL, NULL));
  return 0;
}
"""


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c99_and_links(lib, tmp_path):
    src = tmp_path / "consumer.c"
    exe = tmp_path / "consumer"
    src.write_text(C_SOURCE)
    libdir = os.path.dirname(ops.LIB_PATH)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), "-L", libdir, "-lsparse_attn", f"-Wl,-rpath,{libdir}", "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    assert int(got["version"]) == lib.sa_version()
    assert got["ok"] == "SA_OK" and got["invalid"] == ops.status_string(ops.SA_ERR_INVALID_ARG)
    assert int(got["mask_ws"]) == ops.sa_build_mask_workspace(1, 12, 32760, 128, 64)
    assert int(got["bwd_ws"]) == ops.sa_sparse_attn_bwd_workspace(1, 12, 32760)
    assert int(got["host_ws"]) == ops.sa_sparse_attn_fwd_host_workspace(75600, 128, 2)
    assert int(got["radial_neg"]) == ops.SA_ERR_INVALID_ARG
    assert int(got["radial_empty"]) == ops.SA_OK
    assert int(got["fwd_neg"]) == ops.SA_ERR_INVALID_ARG
    assert int(got["fwd_d96"]) in (ops.SA_ERR_INVALID_ARG, ops.SA_ERR_UNSUPPORTED)
