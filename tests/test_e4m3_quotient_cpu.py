"""The FP8 quantiser's quotient step (csrc/e4m3_quotient.cuh), built for the
host with g++ (tests/host/e4m3_quotient_check.cc): the e4m3 code it leads to
is the real quotient x / s rounded once to e4m3, on random values and on
constructed cases where the float32 quotient lands on an e4m3 midpoint."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_quotient_codes_are_the_exactly_rounded_quotient(tmp_path):
    exe = tmp_path / "e4m3_quotient_check"
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                           "-I", os.path.join(ROOT, "io_aware_exact_21_b200", "csrc"),
                           os.path.join(ROOT, "tests", "host", "e4m3_quotient_check.cc"),
                           "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
