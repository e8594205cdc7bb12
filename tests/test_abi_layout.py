"""The ctypes mirrors of the C ABI structs have the header's layout.

A small C program is compiled against include/nanoflow.h (gcc, no CUDA) and prints sizeof of every
struct and offsetof of every field; the binding's ctypes.Structure classes must agree exactly, or
arguments would be handed to the library misplaced without any error.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

import intra_device_overlapped_b200 as nf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STRUCTS = ["nf_model_config", "nf_layer_weights", "nf_global_weights", "nf_batch_desc", "nf_plan_opts", "nf_plan",
           "nf_iter_io", "nf_cost_model", "nf_trace_entry", "nf_op_time", "nf_sched_config", "nf_sched_iter",
           "nf_sched_stats"]


def c_layout(tmp_path):
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "nanoflow.h"', "int main(void) {"]
    for name in STRUCTS:
        lines.append(f'  printf("{name} %zu\\n", sizeof({name}));')
        for field, _ in getattr(nf, name)._fields_:
            lines.append(f'  printf("{name}.{field} %zu\\n", offsetof({name}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return dict((k, int(v)) for k, v in (ln.split() for ln in out.splitlines()))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_ctypes_structs_match_the_header(tmp_path):
    c = c_layout(tmp_path)
    for name in STRUCTS:
        cls = getattr(nf, name)
        assert ctypes.sizeof(cls) == c[name], name
        for field, _ in cls._fields_:
            assert getattr(cls, field).offset == c[f"{name}.{field}"], (name, field)
