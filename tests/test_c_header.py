"""The boundary is a plain C ABI: include/dbst.h compiles as C99 with no C++ or
CUDA headers, and a C program links libdbst.so and calls it (argument
validation only; no device needed)."""
import os
import shutil
import subprocess

import pytest

from dynamic_block_sparse_tile_b200 import build as dbst_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "dbst.h"

int main(void) {
  dbst_geom g = {1, 2, 128, 4, 8, 16, 2, 4, 8};
  dbst_geom bad = g;
  bad.D = 96;
  if (strcmp(dbst_status_string(DBST_OK), "ok") != 0) return 1;
  if (dbst_mask_workspace_bytes(&g) == 0 || dbst_mask_workspace_bytes(&bad) != 0) return 2;
  if (dbst_attn_backward_workspace_bytes(&g) != (size_t)(2 * 512 * 8)) return 3;
  if (dbst_tile_reorder(NULL, NULL, &g, NULL) != DBST_EINVAL) return 4;
  if (dbst_block_sparse_attn(NULL, NULL, NULL, &g, NULL, NULL, 0.0f, NULL, NULL, NULL) != DBST_EINVAL) return 5;
  if (dbst_squad_workspace_bytes(1, 2, 16384, 128, 128) != (size_t)4 * 2 * 16384 * 128 * 2) return 6;
  printf("c abi ok\n");
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_is_c99_and_library_links(tmp_path):
    lib = dbst_build.build()
    src = tmp_path / "abi.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "abi"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-ldbst", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.strip() == "c abi ok"
