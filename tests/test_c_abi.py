"""The C ABI from a C program (not through ctypes): tests/c_abi_check.c is compiled as C99
against include/mimoattn.h, linked with libmimoattn.so and run.  Host-only calls: no GPU."""
import os
import shutil
import subprocess

import pytest

import global_attention_attn_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_c_program_links_and_validates(tmp_path):
    lib = M.LIB_PATH
    assert os.path.exists(lib), "build the library first (python -m global_attention_attn_b200.build)"
    exe = tmp_path / "c_abi_check"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), lib, "-Wl,-rpath," + os.path.dirname(lib),
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_ctypes_structs_match_the_c_layout(tmp_path):
    """Every field of the binding's ctypes structs sits at the offset the C compiler gives
    the same-named field of include/mimoattn.h, and the sizes agree (no missing field)."""
    import ctypes as C
    structs = {"mimo_layer": M.MimoLayer, "mimo_prefill_args": M.MimoPrefillArgs,
               "mimo_decode_args": M.MimoDecodeArgs, "mimo_append_args": M.MimoAppendArgs}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "mimoattn.h"', "int main(void) {"]
    want = {}
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} sizeof %zu\\n", sizeof({cname}));')
        want[f"{cname} sizeof"] = C.sizeof(py)
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
            want[f"{cname} {fname}"] = getattr(py, fname).offset
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    got = {line.rsplit(" ", 1)[0]: int(line.rsplit(" ", 1)[1]) for line in out}
    assert got == want
