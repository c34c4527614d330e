"""The C ABI used from a plain C program (gcc, C11, -Wall -Werror), linked against the in-tree
library: no C++, CUDA headers or torch on the caller's side.  Host-side validation only, so it
runs without a GPU."""
import os
import shutil
import subprocess

import pytest

from w2a4_gemm_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_links_and_validates(tmp_path):
    lib = build.build()
    exe = tmp_path / "abi_from_c"
    src = os.path.join(ROOT, "tests", "c_abi", "abi_from_c.c")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                    lib, f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
