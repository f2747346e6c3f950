"""The ctypes mirrors of the two C shape structs have the C layout: every
field's offset and the struct size, as gcc lays them out from the C sources
(the library's public header, and the oracle's own definition)."""
import ctypes
import os
import subprocess

import oracle
from sparse_long_context_mse_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _c_layout(tmp_path, prelude, struct, fields):
    """offsetof of each field and sizeof, from a C program gcc builds."""
    lines = [prelude, "#include <stddef.h>", "#include <stdio.h>", "int main(void) {"]
    for f in fields:
        lines.append(f'  printf("%zu\\n", offsetof({struct}, {f}));')
    lines.append(f'  printf("%zu\\n", sizeof({struct}));')
    lines.append("  return 0;\n}")
    src = tmp_path / "layout.c"
    exe = tmp_path / "layout"
    src.write_text("\n".join(lines) + "\n")
    subprocess.check_call(["gcc", "-std=c99", "-w", "-o", str(exe), str(src), "-lm"])
    out = subprocess.check_output([str(exe)]).decode().split()
    return [int(x) for x in out[:-1]], int(out[-1])


def _ctypes_layout(cls):
    return [getattr(cls, name).offset for name, _ in cls._fields_], ctypes.sizeof(cls)


def test_losa_shape_matches_header(tmp_path):
    names = [n for n, _ in api.Shape._fields_]
    inc = os.path.join(ROOT, "include", "losa.h")
    got = _c_layout(tmp_path, f'#include "{inc}"', "losa_shape", names)
    assert _ctypes_layout(api.Shape) == got


def test_oracle_shape_matches_oracle_source(tmp_path):
    names = [n for n, _ in oracle.Shape._fields_]
    src = os.path.join(ROOT, "oracle", "losa_oracle.c")
    got = _c_layout(tmp_path, f'#include "{src}"', "oracle_shape", names)
    assert _ctypes_layout(oracle.Shape) == got


def test_header_compiles_as_c_and_cpp(tmp_path):
    inc = os.path.join(ROOT, "include", "losa.h")
    for compiler, std in (("gcc", "-std=c99"), ("g++", "-std=c++17")):
        src = tmp_path / ("h.c" if compiler == "gcc" else "h.cpp")
        src.write_text(f'#include "{inc}"\nint main(void) {{ losa_shape s = {{0}}; return s.num_seqs; }}\n')
        subprocess.check_call([compiler, std, "-Wall", "-Werror", "-o", str(tmp_path / "h"),
                               str(src)])
