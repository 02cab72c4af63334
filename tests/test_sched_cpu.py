"""The CTA-pair GEMM's work lists (data-parallel and stream-K), checked on the
host: the schedule header is plain C++, compiled here with the system C++
compiler and exercised by ``tests/sched_check.cpp`` over many tile counts,
pair counts and reduction lengths (exact cover, HEAD/TAIL pairing and order)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_nf4_quantized_06_b200", "csrc")


def test_pair_work_lists(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    exe = tmp_path / "sched_check"
    subprocess.run([cxx, "-std=c++17", "-O2", "-I", CSRC, os.path.join(ROOT, "tests", "sched_check.cpp"),
                    "-o", str(exe)], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")
