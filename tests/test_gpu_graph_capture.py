"""Tensor-core calls captured into a CUDA graph on a stream that already ran them eagerly.

Without a caller workspace the captured call's scratch comes from the library pool (a graph
memory node) and its whole tiles go in the static order; every replay must give the eager
call's bits.  At 100 rows (MMA N = 208) the GEMV runs as clusters of CTA pairs.  (With a workspace the eager calls take the queue order: see
test_gpu_workspace.py.)
"""

import numpy as np
import pytest
import torch

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("rows", [5, 40, 100])
def test_lm_head_graph_replays_match_eager(rows):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    n, k = 38188, 1024  # 299 row tiles of 128: two whole tiles per SM plus a remainder
    w = synth.fp8_weight(n, k, 33, "cuda")
    s = synth.row_scales(n, 33, "cuda")
    x = synth.bf16_rows(rows, k, 34, "cuda", std=0.5)
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        eager = dl.lm_head_fp8_w8a16(w, s, x)  # the stream's first eager call
        out = torch.zeros_like(eager)
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        dl.lm_head_fp8_w8a16(w, s, x, out=out)
    want = synth.to_numpy_bits(eager)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(synth.to_numpy_bits(out), want)
    del g
