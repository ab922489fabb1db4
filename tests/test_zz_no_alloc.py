"""The allocation-free W8A8 entry point, w8a8_proj_noalloc, against w8a8_proj and the oracle.

w8a8_proj_noalloc serves callers that cannot call cudaMalloc: engines whose device memory
belongs to a pre-reserved pool or another framework's allocator, and decode loops that
cannot afford cudaMalloc's implicit synchronization.  Its activation scratch is a fixed
device array inside the library.  This test calls it through the C ABI, twice in a row on
different rows (so the second call cannot pass on the first call's leftovers), and checks
each result against w8a8_proj on a caller scratch (the kernels are the same, so the bits
match) and against the CPU oracle within the parity tolerance.  It covers the tensor-core
pass (k = 5120, with and without stream-K partial sums) and the register-fragment pass
(k = 1040, no partial sums), and checks that warm calls take nothing from the library pool
and no device memory from the driver.  The file name sorts last, so a failing run that stops
at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import synth
from oracle import gemv as og
from parity_util import assert_bf16_close

pytestmark = pytest.mark.gpu


def _call_noalloc(w, s, x, out):
    n, k = w.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return dl.lib().w8a8_proj_noalloc(ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(s.data_ptr()), n, k,
                                      ctypes.c_void_p(x.data_ptr()), x.stride(0), x.shape[0],
                                      ctypes.c_void_p(out.data_ptr()), out.stride(0), stream)


@pytest.mark.parametrize("n,k", [(3000, 5120), (38188, 5120), (1000, 1040)])
def test_w8a8_proj_noalloc_matches_w8a8_proj_and_oracle_twice(n, k):
    # 38188 x 5120 (299 tiles: two whole tiles per SM plus a remainder) uses the fixed
    # partial-sum area; 1000 x 1040 (k % 128 != 0) runs the register-fragment kernels
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = synth.fp8_weight(n, k, 31, "cuda")
    s = synth.row_scales(n, 31, "cuda")
    sub = np.arange(0, n, max(1, n // 400))
    for call, rows in enumerate((130, 37)):
        x = synth.bf16_rows(rows, k, 40 + call, "cuda", std=0.5)
        out = torch.empty(rows, n, dtype=torch.bfloat16, device="cuda")
        assert _call_noalloc(w, s, x, out) == 0
        ref = dl.w8a8_proj(w, s, x)
        torch.cuda.synchronize()
        got_b, ref_b = synth.to_numpy_bits(out), synth.to_numpy_bits(ref)
        assert np.array_equal(got_b, ref_b), f"w8a8_proj_noalloc call {call + 1} differs from w8a8_proj"
        oracle = og.w8a8_proj(synth.to_numpy_bits(w)[sub], synth.to_numpy_bits(s)[sub], synth.to_numpy_bits(x))
        assert_bf16_close(got_b[:, sub], oracle, f"w8a8_proj_noalloc call {call + 1} vs oracle")
    assert dl.device_fault(reset=True) == 0


def test_w8a8_proj_noalloc_warm_calls_allocate_nothing():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    n, k = 38188, 5120
    w = synth.fp8_weight(n, k, 32, "cuda")
    s = synth.row_scales(n, 32, "cuda")
    x = synth.bf16_rows(64, k, 32, "cuda", std=0.5)
    out = torch.empty(64, n, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(w, s, x, out) == 0          # warm: the first call looks the array up
    torch.cuda.synchronize()
    before, _ = dl.pool_stats(reset_high=True)
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert _call_noalloc(w, s, x, out) == 0
    torch.cuda.synchronize()
    cur, high = dl.pool_stats()
    assert cur <= before and high <= before, "w8a8_proj_noalloc took scratch from the library pool"
    assert torch.cuda.mem_get_info()[0] == free0, "device memory was allocated during the calls"


def test_w8a8_proj_noalloc_rejects_k_above_its_limit():
    assert dl.lib().w8a8_proj_noalloc(None, None, 16, 16384 + 16, None, 16400, 1, None, 16, None) == -7
