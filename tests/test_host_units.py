"""Host-only C++ units of the library, built with g++ and run on the CPU (no
GPU, no CUDA runtime): the per-device record of one-time set-up steps."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_device_flags_are_per_device(tmp_path):
    exe = tmp_path / "device_flags_test"
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-pthread",
                    "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "l2_row_b200", "csrc"),
                    os.path.join(ROOT, "tests", "host", "device_flags_test.cpp"), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
