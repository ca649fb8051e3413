"""The ctypes mirrors of include/moe.h's structs have the C layout.

A small C program built with the system compiler against the header prints
each struct's size and field offsets; the binding's ctypes structures must
agree field by field (a mismatch would silently shift every argument after
it).  CPU only.
"""

import ctypes
import os
import shutil
import subprocess

import pytest

from mixture_experts_routed_03_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STRUCTS = {
    "moe_problem_t": (api.Problem, ["num_tokens", "hidden", "intermediate_hidden", "num_experts", "num_topk",
                                     "activation_clamp", "format", "fast_math", "tile_regime",
                                     "shared_expert", "activation", "activation_alpha"]),
    "moe_act_t": (api.Act, ["x", "x_scale", "x_rowwise_scale"]),
    "moe_weights_t": (api.Weights, [f[0] for f in api.Weights._fields_]),
    "moe_layout_t": (api.Layout, [f[0] for f in api.Layout._fields_]),
}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    d = tmp_path_factory.mktemp("abi")
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe.h"', "int main(void) {"]
    for name, (_, fields) in STRUCTS.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for f in fields:
            lines.append(f'  printf("{name} {f} %zu\\n", offsetof({name}, {f}));')
    lines += ["  return 0;", "}"]
    src = d / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = d / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    table = {}
    for line in out.splitlines():
        s, f, v = line.split()
        table[(s, f)] = int(v)
    return table


@pytest.mark.parametrize("name", list(STRUCTS))
def test_ctypes_struct_matches_c(c_layout, name):
    cls, fields = STRUCTS[name]
    assert ctypes.sizeof(cls) == c_layout[(name, "size")]
    assert [f[0] for f in cls._fields_] == fields
    for f in fields:
        assert getattr(cls, f).offset == c_layout[(name, f)], (name, f)
