"""The algebra of the tensor-core decode, checked on the host (no GPU).

decode_tc_kernel replaces decode's 128-point transform by an f16 matrix
product with fp32 accumulation.  tests/tc_algebra_check.cpp builds the kernel's
A and B operands by the same rules (the code slots of nq_tc_slots.cuh, the
coset and constant slots, the column order) and checks, for random vectors of
both code widths, that every code lands in exactly one slot and that the
product equals the integer transform H t exactly, with every partial sum below
2^18 in magnitude (so that no fp32 summation order can round it).  The GPU
tests then compare the kernel itself with the oracle bit for bit.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tensor_core_decode_algebra_is_exact(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = tmp_path / "tc_algebra_check"
    build = subprocess.run([cxx, "-O2", "-std=c++17", os.path.join(HERE, "tc_algebra_check.cpp"),
                            "-o", str(exe)], capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "bits 2: 0 failures" in run.stdout and "bits 3: 0 failures" in run.stdout


def test_planted_coset_sign_is_caught(tmp_path):
    """The same check with the coset weights' sign flipped must fail."""
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    exe = tmp_path / "tc_algebra_planted"
    build = subprocess.run([cxx, "-O2", "-std=c++17", "-DPLANT_COSET_SIGN",
                            os.path.join(HERE, "tc_algebra_check.cpp"), "-o", str(exe)],
                           capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert run.returncode != 0

