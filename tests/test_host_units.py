"""Host-only C++ units of the library, built with g++ and run on the CPU (no
GPU, no CUDA runtime): the per-device record of one-time set-up steps, and
the C ABI's struct layout against the ctypes binding's."""
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


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_abi_struct_layout_matches_binding(tmp_path):
    """Every field of ds_wseg and ds_aseg sits where the binding puts it
    (the C compiler's layout of include/ds.h)."""
    from l2_row_b200 import ds

    exe = tmp_path / "abi_layout"
    subprocess.run(["gcc", "-std=c11", "-O1", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "host", "abi_layout.c"), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    c = {}
    for line in out:
        if line.strip():
            t, f, v = line.split()
            c[(t, f)] = int(v)
    for name, cls in (("ds_wseg", ds.ds_wseg), ("ds_aseg", ds.ds_aseg)):
        assert c[(name, "size")] == ct_sizeof(cls), name
        for f, _ in cls._fields_:
            assert c[(name, f)] == getattr(cls, f).offset, (name, f)


def ct_sizeof(cls) -> int:
    import ctypes

    return ctypes.sizeof(cls)
