"""Failure detection on the GPU without a GPU fault: the bounded mbarrier wait that every
TMA / tensor-core kernel here uses gives up on a barrier that nothing completes, records its
fault bit for the host and returns; the context stays usable and the library's kernels keep
working afterwards."""

import time

import numpy as np
import pytest
import torch

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import synth
from oracle import gemv as og
from parity_util import assert_bf16_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dl.device_fault(reset=True)
    t0 = time.perf_counter()
    dl.check_bounded_wait()               # raises DlmhError if the wait did not give up
    elapsed = time.perf_counter() - t0
    assert elapsed < 30.0
    assert dl.device_fault() == 0         # the check clears its own bit
    # the context is still healthy: a GEMV right after is correct
    n, k = 512, 1024
    w = synth.fp8_weight(n, k, 3, "cuda")
    s = synth.row_scales(n, 3, "cuda")
    x = synth.bf16_rows(3, k, 3, "cuda")
    out = synth.to_numpy_bits(dl.lm_head_fp8_w8a16(w, s, x))
    ref = og.w8a16_gemv(synth.to_numpy_bits(w), synth.to_numpy_bits(s), synth.to_numpy_bits(x))
    assert_bf16_close(out, ref, "GEMV after the bounded-wait check")
    assert dl.device_fault() == 0
