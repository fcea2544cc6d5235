"""The boundary is a plain C ABI: a C program that includes only
include/fa.h and links libfa_b200.so builds and gets the documented status
codes from the host-side argument checks (no GPU involved)."""
import os
import shutil
import subprocess

import pytest

import io_aware_exact_21_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_caller(tmp_path):
    lib = fa.library_path()
    fa.load_library()
    cuda_inc = "/usr/local/cuda/include"
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-o", str(exe), lib,
           "-Wl,-rpath," + os.path.dirname(lib)]
    subprocess.check_call(cmd)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
