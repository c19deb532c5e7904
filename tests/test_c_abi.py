"""The C ABI from plain C: compile tests/c/abi_check.c with gcc against include/crisp.h, link the
in-tree libcrisp.so, run it (no GPU needed; it only makes calls that are refused before launch)."""
import os
import shutil
import subprocess

import pytest

from dynamic_block_sparse_proxy_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_links_and_calls_the_library(tmp_path):
    B.build()
    libdir = os.path.join(ROOT, "dynamic_block_sparse_proxy_b200")
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", libdir, "-lcrisp",
           f"-Wl,-rpath,{libdir}", "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout and r.stdout.count("ok ") >= 10
