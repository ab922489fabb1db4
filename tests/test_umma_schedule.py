"""Host-side check of the tensor-core GEMV's stream-K schedule (csrc/umma_sched.h), compiled
with the host C++ compiler: full coverage, bounded jobs per CTA, unique partial slots and an
ordered fixup walk over many (SM count, tile count, units per tile)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stream_k_schedule(tmp_path):
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        pytest.skip("no host C++ compiler")
    exe = tmp_path / "sched_check"
    src = os.path.join(ROOT, "tests", "native", "sched_check.cpp")
    inc = os.path.join(ROOT, "decode_lm_head_b200", "csrc")
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", inc, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")
