"""CPU checks of the C ABI: the library loads, exports what include/dlmh.h declares, plans
row chunks as the oracle's reading of the pages does, and rejects bad arguments before
launching anything (no GPU is needed for any of this)."""

import ctypes

import pytest

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import _lib
from oracle import plan as op

L = None


@pytest.fixture(scope="module", autouse=True)
def _load():
    global L
    L = dl.lib()


def test_library_exports_every_declared_function():
    names = _lib.header_functions()
    assert len(names) >= 13
    for name in names:
        assert hasattr(L, name), name


def test_error_strings_and_version():
    assert dl.version() >= 100
    for code in range(-9, 1):
        assert dl.error_string(code)
    assert dl.error_string(-99) == "unknown status"


@pytest.mark.parametrize("opid,k,width", [(dl.OP_W8A16, 5120, 128), (dl.OP_W8A16, 1040, 16), (dl.OP_W8A8, 5120, 128),
                                           (dl.OP_W8A8, 14336, 128), (dl.OP_W8A8, 1040, 32), (dl.OP_W4A16, 4096, 16),
                                           (dl.OP_Q6K, 7168, 64),
                                           (dl.OP_W4A4, 4096, 32), (dl.OP_W4A4, 14336, 8), (dl.OP_W4A4, 6144, 16)])
def test_plan_matches_oracle_rules(opid, k, width):
    for rows in range(0, 301):
        plan = dl.plan_chunks(opid, rows, k)
        ref = op.chunk_plan(rows, width)
        assert [(o, c) for o, c, _ in plan] == ref
        if opid == dl.OP_Q6K:
            widths = [8, 16, 32, 64]
        elif opid == dl.OP_W4A4:
            widths = [8, 16, 32]
        elif opid in (dl.OP_W8A8, dl.OP_W8A16) and k % 128 == 0:
            widths = list(range(16, 129, 16))  # tensor-core tier: MMA N in steps of 16
        else:
            widths = [8, 16, 32]
        for _, c, tier in plan:
            i = op.select_tier(c, widths, [True] * len(widths))
            assert tier == widths[i]


def test_plan_rejects():
    assert L.dlmh_plan_chunks(dl.OP_W4A16, 33, 4096, None, None, None, 0) == 3  # 16 + 16 + 1
    assert L.dlmh_plan_chunks(dl.OP_W8A16, -1, 5120, None, None, None, 0) == -4
    assert L.dlmh_plan_chunks(9, 1, 5120, None, None, None, 0) == -2
    # k % 128 != 0 keeps the register-fragment tiers, whose activation tile must fit on chip
    assert L.dlmh_plan_chunks(dl.OP_W8A16, 1, 65552, None, None, None, 0) == -7
    arr = (ctypes.c_int * 1)()
    assert L.dlmh_plan_chunks(dl.OP_W8A16, 140, 5120, arr, arr, arr, 1) == -8


# Fake device addresses: the argument checks must reject these calls before any CUDA call
# (on this GPU-less host a call that got past them would return DLMH_ERR_CUDA instead).
A = 1 << 20          # 16-byte aligned
U = A + 2            # 2-byte aligned only


def test_w8a16_argument_errors():
    f = L.lm_head_fp8_w8a16
    assert f(None, A, 16, 64, A, 64, 1, A, 16, None) == -1
    assert f(A, A, 16, 64, None, 64, 1, A, 16, None) == -1
    assert f(A, A, 0, 64, A, 64, 1, A, 16, None) == -2
    assert f(A, A, 16, 63, A, 64, 1, A, 16, None) == -2
    assert f(A, A, 16, 64, A, 32, 1, A, 16, None) == -5
    assert f(A, A, 16, 64, A, 64, 1, A, 8, None) == -5
    assert f(U, A, 16, 64, A, 64, 1, A, 16, None) == -3
    assert f(A, A, 16, 64, U, 64, 1, A, 16, None) == -3
    assert f(A, A, 16, 64, A, 68, 1, A, 16, None) == -3
    assert f(A, A, 16, 64, A, 64, -1, A, 16, None) == -4
    assert f(A, A, 16, 8208, A, 8208, 1, A, 16, None) == -7


def test_w8a8_argument_errors():
    assert L.w8a8_quantize_rows(A, 64, 129, 64, A, 64, A, None) == -4
    assert L.w8a8_quantize_rows(A, 64, 1, 64, U, 64, A, None) == -3
    assert L.w8a8_quantize_rows(A, 64, 1, 64, A, 48, A, None) == -5
    assert L.w8a8_silu_quantize_rows(A, None, 64, 1, 64, A, 64, A, None) == -1
    assert L.w8a8_gemv(A, A, 16, 64, A, 64, A, 129, A, 16, None) == -4
    assert L.w8a8_proj(A, A, 16, 64, A, 64, 1, A, 16, None, A, None) == -1
    assert L.w8a8_silu_proj(A, A, 16, 64, A, None, 64, 1, A, 16, A, A, None) == -1
    # gate+up pair: every pointer of both weights is checked before anything launches
    assert L.w8a8_gate_up_proj(A, A, None, A, 16, 64, A, 64, 1, A, A, 16, A, A, None) == -1
    assert L.w8a8_gate_up_proj(A, A, A, None, 16, 64, A, 64, 1, A, A, 16, A, A, None) == -1
    assert L.w8a8_gate_up_proj(A, A, U, A, 16, 64, A, 64, 1, A, A, 16, A, A, None) == -3
    assert L.w8a8_gate_up_proj(A, A, A, A, 16, 64, A, 64, 1, A, None, 16, A, A, None) == -1
    assert L.w8a8_gate_up_proj(A, A, A, A, 16, 64, A, 64, 1, A, A, 8, A, A, None) == -5
    assert L.w8a8_gate_up_proj(A, A, A, A, 16, 64, A, 64, -1, A, A, 16, A, A, None) == -4
    assert L.w8a8_gate_up_proj(A, A, A, A, 16, 64, A, 64, 0, A, A, 16, A, A, None) == 0


def test_w4a16_argument_errors():
    f = L.w4a16_gemv
    assert f(A, A, ctypes.c_float(1.0), 16, 128, A, 128, -1, A, 16, None) == -4
    assert f(A, A, ctypes.c_float(1.0), 16, 64, A, 128, 1, A, 16, None) == -2
    assert f(A, U, ctypes.c_float(1.0), 16, 128, A, 128, 1, A, 16, None) == -3
    assert f(A, None, ctypes.c_float(1.0), 16, 128, A, 128, 1, A, 16, None) == -1


def test_q6k_argument_errors():
    assert L.q8_1_quantize_rows(A, 64, 1, 48, A, None) == -2
    assert L.q8_1_quantize_rows(A, 16, 1, 64, A, None) == -5
    assert L.q6k_mmvq(A, 16, 255, A, 1, A, 16, None) == -2
    assert L.q6k_mmvq(A + 1, 16, 256, A, 1, A, 16, None) == -3
    assert L.q6k_lm_head(A, 16, 256, A, 256, 1, A, 16, None, None) == -1
    assert L.q6k_lm_head(A, 16, 256, A, 256, -3, A, 16, A, None) == -4


def test_zero_rows_launch_nothing():
    # valid arguments with rows == 0 return OK without touching CUDA
    assert L.w8a8_quantize_rows(A, 64, 0, 64, A, 64, A, None) == 0
    assert L.q8_1_quantize_rows(A, 64, 0, 64, A, None) == 0


def test_w4a4_argument_errors():
    # nvfp4_quantize_rows(x, ldx, rows, k, xq, xs, xg, stream)
    assert L.nvfp4_quantize_rows(A, 64, 1, 40, A, A, A, None) == -2          # k % 16
    assert L.nvfp4_quantize_rows(A, 64, -1, 64, A, A, A, None) == -4
    assert L.nvfp4_quantize_rows(A, 64, 1, 64, A, None, A, None) == -1
    assert L.nvfp4_quantize_rows(A, 64, 1, 64, U, A, A, None) == -3          # codes 16-byte aligned
    assert L.nvfp4_quantize_rows(A, 64, 0, 64, None, None, None, None) == 0
    # w4a4_gemv(wp, ws, g, n, k, xq, xs, xg, rows, out, ldc, stream)
    assert L.w4a4_gemv(A, A, 1.0, 16, 128, A, A, A, 1, A, 16, None) == -2    # k % 256
    assert L.w4a4_gemv(None, A, 1.0, 16, 256, A, A, A, 1, A, 16, None) == -1
    assert L.w4a4_gemv(A, U, 1.0, 16, 256, A, A, A, 1, A, 16, None) == -3
    assert L.w4a4_gemv(A, A, 1.0, 16, 256, A, A + 1, A, 1, A, 16, None) == -3
    assert L.w4a4_gemv(A, A, 1.0, 16, 256, A, A, A, 1, A, 8, None) == -5
    assert L.w4a4_gemv(A, A, 1.0, 16, 256, None, None, None, 0, None, 16, None) == 0
    assert L.w4a4_gemv(A, A, 1.0, 16, 1 << 18, A, A, A, 1, A, 16, None) == -7  # no pass fits this k
    # w4a4_proj(wp, ws, g, n, k, x, ldx, rows, out, ldc, xq, xs, xg, stream)
    assert L.w4a4_proj(A, A, 1.0, 16, 256, A, 256, 1, A, 16, None, A, A, None) == -1
    assert L.w4a4_proj(A, A, 1.0, 16, 256, A, 256, 1, A, 16, U, A, A, None) == -3
    assert L.w4a4_proj(A, A, 1.0, 16, 256, A, 128, 1, A, 16, A, A, A, None) == -5


def test_dequant_argument_errors():
    f = L.nvfp4_dequant_bf16
    assert f(None, A, 1.0, 0, 16, 64, A, 64, None) == -1
    assert f(A, A, 1.0, 0, 16, 40, A, 64, None) == -2      # k % 16
    assert f(A, A, 1.0, 0, 16, 64, A, 32, None) == -5      # ldo < k
    assert f(A, U, 1.0, 0, 16, 64, A, 64, None) == -3
    assert f(A, A, 1.0, 0, 16, 64, A, 68, None) == -3      # ldo % 8
    e = L.e8m0_fp4_dequant_bf16
    assert e(A, None, 4, 16, 64, A, 64, None) == -1
    assert e(A, A, 7, 16, 64, A, 64, None) == -2           # 1024 elements not a multiple of 7 groups
    assert e(A, A, 0, 16, 64, A, 64, None) == -2
    assert e(U, A, 4, 16, 64, A, 64, None) == -3


def test_workspace_bytes_sizes_and_errors():
    # Sizes of the caller workspace (dlmh.h): a 256-byte tile queue, the W8A16 two-term codes
    # of the widest pass (2 roundup8(min(rows,128)) k + 512 bytes, rounded to 256), then the
    # stream-K partial sums, two slots of N_mma x 128 float32 per CTA (2 P CTAs, P = 74
    # parties), when the tile pairs do not make whole waves over the parties.  Worked by hand
    # for 148 SMs:
    ws = dl.workspace_bytes
    # FP8 head 248320 x 5120: 1940 tiles = 970 pairs, 13 whole waves + 8 remainder pairs
    assert ws(dl.OP_W8A16, 248320, 5120, 128, 148) == 256 + (2 * 128 * 5120 + 512) + 2 * 148 * 256 * 128 * 4
    assert ws(dl.OP_W8A8, 248320, 5120, 128, 148) == 256 + 2 * 148 * 128 * 128 * 4
    assert ws(dl.OP_W8A8, 248320, 5120, 1000, 148) == ws(dl.OP_W8A8, 248320, 5120, 128, 148)  # 128-row passes
    assert ws(dl.OP_W8A16, 248320, 5120, 3, 148) == 256 + (2 * 8 * 5120 + 512) + 2 * 148 * 16 * 128 * 4
    # 148 x 128 rows: whole waves only, no partial sums
    assert ws(dl.OP_W8A8, 148 * 128, 5120, 64, 148) == 256
    # 147 tiles are 74 tile pairs: one whole wave over the 74 parties (CTA pairs), at any N
    assert ws(dl.OP_W8A8, 147 * 128, 5120, 64, 148) == 256
    assert ws(dl.OP_W8A8, 147 * 128, 5120, 128, 148) == 256
    # 150 tiles are 75 tile pairs: one whole wave and one remainder pair
    assert ws(dl.OP_W8A8, 150 * 128, 5120, 128, 148) == 256 + 2 * 148 * 128 * 128 * 4
    # down projection 4096 x 14336: 32 tiles < 148 SMs, all of them remainder tiles
    assert ws(dl.OP_W8A8, 4096, 14336, 1, 148) == 256 + 2 * 148 * 16 * 128 * 4
    # gate + up pair: the tiles of both weights
    assert ws(dl.OP_W8A8_PAIR, 14336, 4096, 16, 148) == 256 + 2 * 148 * 16 * 128 * 4
    # no tensor-core pass: nothing
    for op_, k in ((dl.OP_W8A16, 1040), (dl.OP_W8A8, 1040), (dl.OP_W4A16, 4096), (dl.OP_Q6K, 7168),
                   (dl.OP_W4A4, 4096)):
        assert ws(op_, 1000, k, 16, 148) == 0
    assert ws(dl.OP_W8A16, 1000, 5120, 0, 148) == 0
    # errors (no GPU is touched with an explicit SM count)
    f = L.dlmh_workspace_bytes
    assert f(6, 16, 128, 1, 148) == -2
    assert f(dl.OP_W8A8, 0, 128, 1, 148) == -2
    assert f(dl.OP_W8A8, 16, 128, 1, -1) == -2
    assert f(dl.OP_W8A8, 16, 128, -1, 148) == -4


def test_set_workspace_argument_errors():
    assert L.dlmh_set_workspace(A + 16, 1 << 20, None) == -3      # not 256-byte aligned
    assert L.dlmh_set_workspace(A, 255, None) == -9               # smaller than the tile queue
    assert dl.error_string(-9).startswith("the stream's workspace")


def test_plan_pair_op_runs_w8a8_passes():
    for rows in (1, 128, 129, 300):
        assert dl.plan_chunks(dl.OP_W8A8_PAIR, rows, 4096) == dl.plan_chunks(dl.OP_W8A8, rows, 4096)
