"""The C ABI used from plain C: compile tests/c_abi_check.c with gcc against include/moe.h,
link the built library, run it (host-side paths only, no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from sparse_moe_layer_03_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_links_and_runs(tmp_path):
    lib_dir = os.path.dirname(B.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    cmd = ["gcc", "-std=c11", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe, "-L", lib_dir, "-l:libmoe.so",
           "-Wl,-rpath," + lib_dir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
