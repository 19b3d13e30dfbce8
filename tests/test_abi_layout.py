"""The C structs of include/hga.h and their ctypes mirrors in the binding have
the same layout: a small C program built against the header (plain gcc, no
GPU) prints every field's offset and every struct's size, and the test
compares them with the mirrors'.  A field added on one side only fails here."""
import ctypes
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hga():
    from long_context_hga_b200 import build
    build.build()
    from long_context_hga_b200 import hga as mod
    return mod


# struct name in the header -> mirror class name in hga.py
STRUCTS = {
    "hga_params": "CParams",
    "hga_group_cache": "CGroupCache",
    "hga_store_stats": "CStoreStats",
}


def _c_layout(tmp_path, mirrors):
    lines = ['#include "hga.h"', "#include <stdio.h>", "#include <stddef.h>", "int main(void) {"]
    for cname, pyname in STRUCTS.items():
        cls = mirrors[pyname]
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    layout = {}
    for line in out.splitlines():
        struct, key, value = line.split()
        layout[(struct, key)] = int(value)
    return layout


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_struct_mirrors_match_the_header(hga, tmp_path):
    mirrors = {pyname: getattr(hga, pyname) for pyname in STRUCTS.values()}
    layout = _c_layout(tmp_path, mirrors)
    for cname, pyname in STRUCTS.items():
        cls = mirrors[pyname]
        assert layout[(cname, "size")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert layout[(cname, field)] == getattr(cls, field).offset, (cname, field)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_params_mirror_has_every_header_field(hga, tmp_path):
    """Every int32 member of hga_params in the header appears in the mirror
    (the header is parsed for member declarations between the braces)."""
    text = open(os.path.join(ROOT, "include", "hga.h")).read()
    body = text[text.index("typedef struct hga_params {"):text.index("} hga_params;")]
    names = []
    for line in body.splitlines():
        code = line.split("/*")[0].strip()
        if code.startswith("int32_t ") and code.endswith(";"):
            names.append(code[len("int32_t "):-1].strip())
    assert names == [f for f, _ in hga.CParams._fields_]
