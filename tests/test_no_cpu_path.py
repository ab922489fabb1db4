"""The product path has no CPU fallback: host tensors are refused before anything runs, and a
missing library is an error at the first call, not a silent switch to another path."""

import os
import subprocess
import sys

import pytest
import torch

import decode_lm_head_b200 as dl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_host_tensors_are_refused_by_every_entry():
    w = torch.zeros(16, 128, dtype=torch.uint8)
    s = torch.ones(16, dtype=torch.float32)
    x = torch.zeros(2, 128, dtype=torch.bfloat16)
    calls = [
        lambda: dl.lm_head_fp8_w8a16(w, s, x),
        lambda: dl.w8a8_quantize_rows(x),
        lambda: dl.w8a8_proj(w, s, x),
        lambda: dl.w8a8_silu_proj(w, s, x, x),
        lambda: dl.w4a16_gemv(torch.zeros(16, 64, dtype=torch.uint8), torch.zeros(16, 8, dtype=torch.uint8),
                              1.0, x),
        lambda: dl.nvfp4_quantize_rows(x),
        lambda: dl.q8_1_quantize_rows(x),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="no CPU path"):
            call()


def test_missing_library_raises_at_first_call():
    code = ("import decode_lm_head_b200 as dl\n"
            "try:\n"
            "    dl.lib()\n"
            "except RuntimeError as e:\n"
            "    print('raised:', e)\n"
            "else:\n"
            "    print('loaded')\n")
    env = dict(os.environ, DLMH_LIBRARY=os.path.join(ROOT, "_no_such_dir", "libdlmh.so"), CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert "raised:" in r.stdout and "is missing" in r.stdout
