"""Host-side checks of the kernels' work splits, compiled with the host C++ compiler from the
same headers the kernels include: the tensor-core GEMV's stream-K schedule (csrc/umma_sched.h:
full coverage, bounded jobs per CTA, unique partial slots and an ordered fixup walk over many
(SM count, tile count, units per tile)) and the Q6_K K-slice split (csrc/q6k_slices.h)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_native(tmp_path, name):
    cxx = shutil.which("g++") or shutil.which("c++")
    if not cxx:
        pytest.skip("no host C++ compiler")
    exe = tmp_path / name
    src = os.path.join(ROOT, "tests", "native", name + ".cpp")
    inc = os.path.join(ROOT, "decode_lm_head_b200", "csrc")
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", inc, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")


def test_stream_k_schedule(tmp_path):
    _run_native(tmp_path, "sched_check")


def test_q6k_k_slices(tmp_path):
    # slices tile K in order, differ by at most one super-block (longer first), the slice-end
    # test marks each slice's last super-block, and the SM sub-partitions' loads differ by at
    # most one (seven each at K = 7168)
    _run_native(tmp_path, "q6k_slices_check")
