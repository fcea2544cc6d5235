"""The kernels' tile schedule and mask classification, built for the host
with g++ (tests/host/schedule_check.cc): every row block of every (sequence,
head) is visited by exactly one CTA for the pair and pair + snake-tail walks,
fixed and packed, at several grid sizes; a block's key-tile range holds every
key its rows may see; a tile classified as unmasked has no disallowed pair."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_schedule_and_mask_invariants(tmp_path):
    exe = tmp_path / "schedule_check"
    subprocess.check_call(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                           "-I", os.path.join(ROOT, "io_aware_exact_21_b200", "csrc"),
                           os.path.join(ROOT, "tests", "host", "schedule_check.cc"), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
