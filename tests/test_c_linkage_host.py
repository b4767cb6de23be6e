"""The library is usable from plain C: a C99 program that includes
include/csa2.h links against libcsa2.so and calls entry points that need no
GPU (the version, a workspace size, a status string, an argument error)."""
import os
import shutil
import subprocess

import pytest

import kv_cache_decode_csa2_b200 as K
from kv_cache_decode_csa2_b200 import csa2 as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "csa2.h"
int main(void) {
  csa2_rows keys = {0};
  int32_t bad = csa2_index_full(NULL, NULL, &keys, NULL, NULL, 1, 64, 128, 16, NULL, 0, 0, NULL, NULL,
                                0, NULL, NULL, NULL, 0, NULL, NULL);
  printf("%d %zu %d %s\n", csa2_version(), csa2_topk_pool_workspace(1, 16384, 512), bad,
         csa2_status_string(CSA2_ERR_TIMEOUT));
  return 0;
}
"""


def test_c_program_links_and_calls_the_library(tmp_path):
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    K.lib()                                   # built
    lib_dir = os.path.dirname(B.LIB_PATH)
    src = tmp_path / "use_csa2.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "use_csa2"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-L", lib_dir, "-lcsa2", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split(maxsplit=3)
    assert out[0] == "200" and out[1] == "256" and out[2] == "1"
    assert out[3].strip() == "bounded wait timed out"
