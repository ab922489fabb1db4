"""The caller-owned workspace of the tensor-core passes (dlmh_workspace_bytes /
dlmh_set_workspace), on the GPU.

A stream with a bound workspace takes every internal scratch area from it and never touches
the library pool (the pool's peak use does not move), hands its whole weight tiles out from
the workspace's queue, and gives exactly the bits of the pool path (static tile order).  A
workspace smaller than a call needs is refused before anything is launched.
"""

import numpy as np
import pytest
import torch

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import synth
from oracle import gemv as og
from parity_util import assert_bf16_close

pytestmark = pytest.mark.gpu

DEV = "cuda"


def bits(t):
    return synth.to_numpy_bits(t)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dl.lib()


def _workspace(nbytes):
    # 256-byte aligned view of a torch buffer
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=DEV)
    off = (-buf.data_ptr()) % 256
    return buf, buf[off:off + nbytes]


@pytest.mark.parametrize("n,k", [(38188, 5120), (4096, 14336), (1000, 1024)])
def test_workspace_calls_match_pool_calls_and_allocate_nothing(n, k):
    # 38188 x 5120: 299 tiles, two whole waves on 148 SMs plus a stream-K remainder (queue and
    # partial sums used); 4096 x 14336: the down projection, every tile a remainder tile
    w = synth.fp8_weight(n, k, 41, DEV)
    s = synth.row_scales(n, 41, DEV)
    x = synth.bf16_rows(130, k, 41, DEV, std=0.5)
    w2 = synth.fp8_weight(n, k, 42, DEV, tensor_id=6)
    s2 = synth.row_scales(n, 42, DEV, tensor_id=7)
    xq = torch.empty(128 * k, dtype=torch.uint8, device=DEV)
    xs = torch.empty(128, dtype=torch.float32, device=DEV)
    st = torch.cuda.Stream()
    calls = {
        "w8a16": lambda m: dl.lm_head_fp8_w8a16(w, s, x[:m], stream=st),
        "w8a8": lambda m: dl.w8a8_proj(w, s, x[:m], xq_scratch=xq, xscale_scratch=xs, stream=st),
        "pair": lambda m: torch.cat(dl.w8a8_gate_up_proj(w, s, w2, s2, x[:m], xq_scratch=xq, xscale_scratch=xs,
                                                         stream=st), dim=1),
    }
    rows = (1, 17, 130)
    with torch.cuda.stream(st):
        pool = {(name, m): bits(f(m)) for name, f in calls.items() for m in rows}
    st.synchronize()
    need = max(dl.workspace_bytes(op, n, k, 130) for op in (dl.OP_W8A16, dl.OP_W8A8, dl.OP_W8A8_PAIR))
    _, ws = _workspace(need)
    dl.set_workspace(ws, stream=st)
    try:
        torch.cuda.synchronize()
        before, _ = dl.pool_stats(reset_high=True)
        with torch.cuda.stream(st):
            for rep in range(2):  # twice: the queue must be back at zero after every launch
                for (name, m), want in pool.items():
                    got = bits(calls[name](m))
                    assert np.array_equal(got, want), f"{name} rows={m} rep={rep}"
        st.synchronize()
        cur, high = dl.pool_stats()
        assert high <= before and cur <= before, "a call with a bound workspace used the library pool"
        assert int(ws[:8].view(torch.int32).abs().sum()) == 0, "tile queue not back at zero"
    finally:
        dl.set_workspace(None, stream=st)
    if k % 128 == 0:
        ref = og.w8a8_proj(bits(w)[:300], bits(s)[:300], bits(x))
        assert_bf16_close(pool[("w8a8", 130)][:, :300], ref, "w8a8 via workspace vs oracle")
    assert dl.device_fault(reset=True) == 0


def test_workspace_too_small_is_refused_before_any_launch():
    n, k = 38188, 5120
    w = synth.fp8_weight(n, k, 43, DEV)
    s = synth.row_scales(n, 43, DEV)
    x = synth.bf16_rows(16, k, 43, DEV, std=0.5)
    st = torch.cuda.Stream()
    need = dl.workspace_bytes(dl.OP_W8A16, n, k, 16)
    _, ws = _workspace(need - 256)
    dl.set_workspace(ws, stream=st)
    try:
        out = torch.full((16, n), 5.0, dtype=torch.bfloat16, device=DEV)
        xq = torch.zeros(128 * k, dtype=torch.uint8, device=DEV)
        xs = torch.zeros(128, dtype=torch.float32, device=DEV)
        with pytest.raises(dl.DlmhError) as e:
            dl.lm_head_fp8_w8a16(w, s, x, out=out, stream=st)
        assert e.value.code == -9
        # a 128-row W8A8 call needs more than this workspace too (MMA N = 128 columns of
        # partial sums); it is refused before its quantize runs
        x128 = synth.bf16_rows(128, k, 44, DEV, std=0.5)
        assert dl.workspace_bytes(dl.OP_W8A8, n, k, 128) > need - 256
        outb = torch.full((128, n), 5.0, dtype=torch.bfloat16, device=DEV)
        with pytest.raises(dl.DlmhError) as e:
            dl.w8a8_proj(w, s, x128, out=outb, xq_scratch=xq, xscale_scratch=xs, stream=st)
        assert e.value.code == -9
        st.synchronize()
        assert bool((out == 5.0).all()) and bool((outb == 5.0).all())
        assert int(xq.count_nonzero()) == 0 and int(xs.count_nonzero()) == 0
    finally:
        dl.set_workspace(None, stream=st)


def test_workspace_survives_graph_capture_with_the_static_order():
    # eager calls on a stream with a workspace take the queue order; a call captured on it
    # takes the static order, with its codes and partial sums in the workspace; replays give
    # the eager bits
    n, k, rows = 38188, 1024, 40
    w = synth.fp8_weight(n, k, 45, DEV)
    s = synth.row_scales(n, 45, DEV)
    x = synth.bf16_rows(rows, k, 45, DEV, std=0.5)
    st = torch.cuda.Stream()
    _, ws = _workspace(dl.workspace_bytes(dl.OP_W8A16, n, k, rows))
    dl.set_workspace(ws, stream=st)
    try:
        with torch.cuda.stream(st):
            eager = dl.lm_head_fp8_w8a16(w, s, x)
            out = torch.zeros_like(eager)
        st.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            dl.lm_head_fp8_w8a16(w, s, x, out=out)
        for _ in range(2):
            out.zero_()
            g.replay()
            torch.cuda.synchronize()
            assert np.array_equal(bits(out), bits(eager))
        del g
    finally:
        dl.set_workspace(None, stream=st)
