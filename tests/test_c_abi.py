"""The C ABI from a plain C11 program (host only, no GPU needed): the header
compiles as C with warnings as errors, the program links against
libdualflow.so and gets every documented answer back."""

import os
import shutil
import subprocess

import pytest

from dual_flow_transformer_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_plain_c_program_against_the_library(tmp_path):
    L.load()  # builds the library if needed
    lib_dir = os.path.dirname(L.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi", "abi_check.c"),
                    "-L", lib_dir, "-ldualflow", "-Wl,-rpath," + lib_dir, "-o", exe],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
