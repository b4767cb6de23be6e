"""The Python binding's ctypes structs have the C header's layout: gcc compiles
a probe that prints sizeof and offsetof of every field of csa2_rows,
csa2_layer and csa2_plan_shape from include/csa2.h, and each must equal the
binding's.  A mismatch would hand the library garbage pointers."""
import ctypes
import os
import shutil
import subprocess

import pytest

from kv_cache_decode_csa2_b200 import csa2 as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STRUCTS = {"csa2_rows": B.csa2_rows, "csa2_layer": B.csa2_layer, "csa2_plan_shape": B.csa2_plan_shape}


def _probe(tmp_path) -> dict:
    gcc = shutil.which("gcc") or shutil.which("cc")
    if gcc is None:
        pytest.skip("no C compiler")
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "csa2.h"', "int main(void) {"]
    for name, cls in STRUCTS.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "probe"
    subprocess.run([gcc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    res = {}
    for ln in out.splitlines():
        struct, field, val = ln.split()
        res[(struct, field)] = int(val)
    return res


def test_ctypes_structs_match_the_header(tmp_path):
    c = _probe(tmp_path)
    for name, cls in STRUCTS.items():
        assert ctypes.sizeof(cls) == c[(name, "size")], name
        for field, _ in cls._fields_:
            assert getattr(cls, field).offset == c[(name, field)], f"{name}.{field}"
