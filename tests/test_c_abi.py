"""The C ABI used from C: tests/c/abi_host_check.c is compiled with gcc against
include/svdq.h, linked to the package's libsvdq_b200.so, and run (host-only
calls; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import w4a4_rank_corrected_act_b200 as svdq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_against_the_header_and_library(tmp_path):
    lib = svdq.LIB_PATH
    if not os.path.exists(lib):
        pytest.skip("the shared library is not built")
    exe = tmp_path / "abi_host_check"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-o", str(exe),
           lib, f"-Wl,-rpath,{libdir}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
