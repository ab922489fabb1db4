"""The allocation-free W8A8 entry point, w8a8_proj_noalloc, against w8a8_proj.

w8a8_proj_noalloc serves callers that cannot call cudaMalloc: engines whose device memory
belongs to a pre-reserved pool or another framework's allocator, and decode loops that
cannot afford cudaMalloc's implicit synchronization.  Its activation scratch is a fixed
device array inside the library.  This test calls it through the C ABI, twice in a row on
different rows (so the second call cannot pass on the first call's leftovers), and checks
each result against w8a8_proj on a caller scratch, within the parity tolerance (the
kernels are the same, so the bits match too).  The file name sorts last, so a failing run
that stops at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import synth
from parity_util import assert_bf16_close

pytestmark = pytest.mark.gpu


def _call_noalloc(w, s, x, out):
    n, k = w.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return dl.lib().w8a8_proj_noalloc(ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(s.data_ptr()), n, k,
                                      ctypes.c_void_p(x.data_ptr()), x.stride(0), x.shape[0],
                                      ctypes.c_void_p(out.data_ptr()), out.stride(0), stream)


@pytest.mark.parametrize("n", [3000, 38188])
def test_w8a8_proj_noalloc_matches_w8a8_proj_twice(n):
    # n = 38188 (299 tiles: two whole tiles per SM plus a remainder): w8a8_proj hands the whole
    # tiles out from its per-stream queue, w8a8_proj_noalloc takes them in the static order;
    # a whole tile's bits do not depend on which CTA ran it, so the outputs must be identical
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    k = 5120
    w = synth.fp8_weight(n, k, 31, "cuda")
    s = synth.row_scales(n, 31, "cuda")
    for call, rows in enumerate((130, 37)):
        x = synth.bf16_rows(rows, k, 40 + call, "cuda", std=0.5)
        out = torch.empty(rows, n, dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(w, s, x, out) == 0
        ref = dl.w8a8_proj(w, s, x)
        torch.cuda.synchronize()
        got_b, ref_b = synth.to_numpy_bits(out), synth.to_numpy_bits(ref)
        assert_bf16_close(got_b, ref_b, f"w8a8_proj_noalloc call {call + 1}")
        assert np.array_equal(got_b, ref_b)


def test_w8a8_proj_noalloc_rejects_k_above_its_limit():
    assert dl.lib().w8a8_proj_noalloc(None, None, 16, 16384 + 16, None, 16400, 1, None, 16, None) == -7
