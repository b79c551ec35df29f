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
