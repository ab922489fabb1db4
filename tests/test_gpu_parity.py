"""GPU parity: every entry point of libdlmh against the CPU oracle on the same seeded inputs.

Floating outputs must be within |err| <= 2^-7 |ref| + 1e-3 rms(ref); quantized bytes and
scales must be bit-exact; a row's output bits must not depend on how many rows share the
call (checked GPU against GPU).
"""

import numpy as np
import pytest
import torch

import decode_lm_head_b200 as dl
from decode_lm_head_b200 import synth
from oracle import gemv as og
from oracle import numerics as nx
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


# ---------------------------------------------------------------------------
# FP8 W8A16
# ---------------------------------------------------------------------------


def test_w8a16_tiny_config_all_rows():
    """N=8192, K=1024, M=1..4, seed 0 (the tiny FP8 config)."""
    n, k = 8192, 1024
    w = synth.fp8_weight(n, k, 0, DEV)
    s = synth.row_scales(n, 0, DEV)
    x = synth.bf16_rows(4, k, 0, DEV)
    ref = og.w8a16_gemv(bits(w), bits(s), bits(x))
    outs = {}
    for m in (1, 2, 3, 4):
        out = dl.lm_head_fp8_w8a16(w, s, x[:m])
        torch.cuda.synchronize()
        outs[m] = bits(out)
        assert_bf16_close(outs[m], ref[:m], f"w8a16 tiny M={m}")
    for m in (1, 2, 3):
        assert np.array_equal(outs[m], outs[4][:m]), f"row invariance M={m} vs 4"


@pytest.mark.parametrize("n,k", [(1000, 1040), (37, 5120), (4099, 2048), (1000, 6144)])
def test_w8a16_ragged_shapes_and_tiers(n, k):
    w = synth.fp8_weight(n, k, 5, DEV)
    s = synth.row_scales(n, 5, DEV)
    x = synth.bf16_rows(40, k, 5, DEV, std=0.5)
    ref = og.w8a16_gemv(bits(w), bits(s), bits(x))
    full = bits(dl.lm_head_fp8_w8a16(w, s, x))
    assert_bf16_close(full, ref, f"w8a16 n={n} k={k} M=40")
    for m in (1, 5, 8, 9, 16, 17, 33):
        part = bits(dl.lm_head_fp8_w8a16(w, s, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"
    # the same row placed at every position of a 16-row chunk gives the same bits
    xr = x[3:4].repeat(16, 1)
    rep = bits(dl.lm_head_fp8_w8a16(w, s, xr))
    assert (rep == full[3][None, :]).all()


@pytest.mark.parametrize("n,k", [(300, 1152), (9000, 384)])
def test_w8a16_tensor_core_tier_wide_rows(n, k):
    # k % 128 == 0: one tensor-core pass per 128 rows for every row count; 130 rows cross a
    # pass boundary, n leaves a ragged 128-row tile, an odd chunk count a half-empty stage
    w = synth.fp8_weight(n, k, 12, DEV)
    s = synth.row_scales(n, 12, DEV)
    x = synth.bf16_rows(130, k, 12, DEV, std=0.5)
    ref = og.w8a16_gemv(bits(w), bits(s), bits(x))
    full = bits(dl.lm_head_fp8_w8a16(w, s, x))
    assert_bf16_close(full, ref, f"w8a16 tensor-core tier n={n} k={k} M=130")
    for m in (1, 15, 16, 17, 64, 127, 128):
        part = bits(dl.lm_head_fp8_w8a16(w, s, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"
    assert np.array_equal(bits(dl.lm_head_fp8_w8a16(w, s, x[128:])), full[128:])
    assert dl.device_fault(reset=True) == 0


def test_w8a16_one_hot_weights_reproduce_activations():
    # W[n] = 1.0 at column n % k (scale 1): out[m, n] = x[m, n % k] exactly wherever
    # |x| >= 2^-13 max|x_m| (the two-term E4M3 split is exact there), within 2^-20 max|x_m|
    # elsewhere -- checks the K order, the hi/lo pairing and the row exponent end to end
    n, k = 2304, 1024
    cols = np.arange(n) % k
    codes = np.zeros((n, k), dtype=np.uint8)
    codes[np.arange(n), cols] = 0x38                     # E4M3 1.0
    w = torch.from_numpy(codes).to(DEV)
    s = torch.ones(n, dtype=torch.float32, device=DEV)
    x = synth.bf16_rows(37, k, 14, DEV)
    x[3] *= 1e-20
    x[4] *= 1e20
    out = nx.bf16_decode(bits(dl.lm_head_fp8_w8a16(w, s, x)))
    xv = nx.bf16_decode(bits(x))
    want = xv[:, cols]
    amax = np.abs(xv).max(axis=1, keepdims=True)
    big = np.abs(want) >= 2.0 ** -13 * amax
    assert np.array_equal(out[big], want[big])
    assert np.all(np.abs(out - want)[~big] <= 2.0 ** -20 * np.broadcast_to(amax, want.shape)[~big])


def test_w8a16_strided_io_and_zero_rows():
    n, k = 515, 1024
    w = synth.fp8_weight(n, k, 6, DEV)
    s = synth.row_scales(n, 6, DEV)
    xb = synth.bf16_rows(7, k + 64, 6, DEV)
    x = xb[:, :k]                           # ldx = k + 64
    outb = torch.full((7, n + 9), 7.0, dtype=torch.bfloat16, device=DEV)
    out = outb[:, :n]                       # ldc = n + 9
    dl.lm_head_fp8_w8a16(w, s, x, out=out)
    ref = og.w8a16_gemv(bits(w), bits(s), bits(x))
    assert_bf16_close(bits(out), ref, "w8a16 strided")
    assert (outb[:, n:] == 7.0).all(), "padding columns of out were written"
    empty = torch.empty(0, k, dtype=torch.bfloat16, device=DEV)
    canary = torch.full((1, n), 3.0, dtype=torch.bfloat16, device=DEV)
    dl.lm_head_fp8_w8a16(w, s, empty, out=canary[:0])
    assert (canary == 3.0).all()


def test_w8a16_extreme_codes_and_row_magnitudes():
    n, k = 64, 1024
    g = torch.Generator(device="cpu").manual_seed(7)
    codes = torch.randint(0, 256, (n, k), generator=g, dtype=torch.int32).to(torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x7E          # no NaN codes; keep +-448
    codes[:8] = codes[:8] & 0x87                   # rows of subnormal codes only
    w = codes.to(DEV)
    s = synth.row_scales(n, 7, DEV)
    x = synth.bf16_rows(6, k, 7, DEV)
    x[1] *= 1e-25                                  # tiny row
    x[2] *= 1e25                                   # huge row
    x[3, ::3] = 0                                  # zeros
    x[4] = 0                                       # all-zero row
    x[5, 5] = 3.0e38                               # one huge value beside ordinary ones
    out = bits(dl.lm_head_fp8_w8a16(w, s, x))
    ref = og.w8a16_gemv(bits(w), bits(s), bits(x))
    for m in range(5):
        assert_bf16_close(out[m:m + 1], ref[m:m + 1], f"w8a16 extreme row {m}")
    assert not nx.bf16_decode(out[4]).any()
    # Row 5: one 3e38 value among N(0,1) values.  k = 1024 takes the tensor-core path, whose
    # two-term E4M3 split of a row is exact for |x| >= 2^-13 max|x| (here x[5, 5] alone) and
    # may drop the rest (|x| <= 5 < 2^-13 * 3e38).  So, per output,
    #   |got - ref| <= 2^-7 |ref| + s[n] * sum over the other k of |e4m3(w[n, k]) x[5, k]|,
    # and where s[n] e4m3(w[n, 5]) 3e38 passes the BF16 range both sides round to the same
    # infinity.
    got5, ref5 = nx.bf16_decode(out[5]), nx.bf16_decode(ref[5])
    wv = nx.e4m3_decode(bits(w)).astype(np.float64)
    xv = nx.bf16_decode(bits(x)[5]).astype(np.float64)
    small = np.abs(xv) < 2.0 ** -13 * np.abs(xv).max()
    assert small.sum() == k - 1
    dropped = bits(s).view(np.float32).astype(np.float64) * (np.abs(wv[:, small]) @ np.abs(xv[small]))
    inf = np.isinf(ref5)
    assert inf.any() and np.array_equal(got5[inf], ref5[inf])
    fin = ~inf
    assert np.all(np.isfinite(got5[fin]))
    assert np.all(np.abs(got5[fin] - ref5[fin]) <= 2.0 ** -7 * np.abs(ref5[fin]) + dropped[fin])


# ---------------------------------------------------------------------------
# W8A8
# ---------------------------------------------------------------------------


def test_w8a8_quantize_rows_bit_exact():
    k = 5120
    x = synth.bf16_rows(128, k, 2, DEV, std=0.5)
    x[5] = 0
    x[6] = 0
    x[6, 17] = -2.5
    x[7] *= 1e-30
    x[8, :7] = torch.tensor([448.0, -448.0, 1e-4, -1e-4, 3.0, 0.0, -0.0], dtype=torch.bfloat16)
    xq, sx = dl.w8a8_quantize_rows(x)
    q_ref, sx_ref = og.w8a8_quantize_rows(bits(x))
    assert np.array_equal(bits(sx).view(np.uint32), sx_ref.view(np.uint32))
    assert np.array_equal(bits(xq), q_ref)
    for rows in (0, 1, 3):
        xq2, sx2 = dl.w8a8_quantize_rows(x[:rows])
        assert np.array_equal(bits(xq2), q_ref[:rows])


def test_w8a8_silu_quantize_bit_exact():
    # codes and scales bit-exact against the oracle's float32 SiLU steps, 128 rows of 14336
    k = 14336
    gate = synth.bf16_rows(128, k, 3, DEV, tensor_id=4)
    up = synth.bf16_rows(128, k, 3, DEV, tensor_id=5)
    xq, sx = dl.w8a8_silu_quantize_rows(gate, up)
    q_ref, sx_ref = og.silu_quantize_rows(bits(gate), bits(up))
    assert np.array_equal(bits(sx), sx_ref)
    assert np.array_equal(bits(xq), q_ref)


def test_w8a8_silu_quantize_every_bf16_gate():
    # every finite BF16 gate value once: row r holds the values whose exponent field is
    # 2r or 2r+1 (both signs, padded with zeros to 512), so each row's codes resolve them
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    rows = np.zeros((128, 512), np.uint16)
    for r in range(128):
        sel = allb[((allb >> 7) & 0xFF) // 2 == r]
        sel = sel[(sel & 0x7F80) != 0x7F80]
        rows[r, :sel.size] = sel
    # |up| <= 1 keeps silu(g)*up finite for the largest g
    up = bits(synth.bf16_rows(128, 512, 5, DEV, tensor_id=5, std=0.3).clamp(-1.0, 1.0))
    g_t = torch.from_numpy(rows.view(np.int16)).view(torch.bfloat16).to(DEV)
    u_t = torch.from_numpy(up.view(np.int16)).view(torch.bfloat16).to(DEV)
    xq, sx = dl.w8a8_silu_quantize_rows(g_t, u_t)
    q_ref, sx_ref = og.silu_quantize_rows(rows, up)
    assert np.array_equal(bits(sx), sx_ref)
    assert np.array_equal(bits(xq), q_ref)


@pytest.mark.parametrize("n,k", [(1000, 1024), (1000, 5120), (4096, 14336)])
def test_w8a8_gemv_and_proj(n, k):
    w = synth.fp8_weight(n, k, 8, DEV)
    s = synth.row_scales(n, 8, DEV)
    x = synth.bf16_rows(130, k, 8, DEV)
    full = bits(dl.w8a8_proj(w, s, x))
    q_ref, sx_ref = og.w8a8_quantize_rows(bits(x))
    sub = slice(None) if n <= 1000 else slice(0, n, 5)
    ref = og.w8a8_gemv(bits(w)[sub], bits(s)[sub], q_ref, sx_ref)
    assert_bf16_close(full[:, sub], ref, f"w8a8 proj n={n} k={k} M=130")
    for m in (1, 31, 32, 33, 128):
        part = bits(dl.w8a8_proj(w, s, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"
    xq, sx = dl.w8a8_quantize_rows(x[:128])
    direct = bits(dl.w8a8_gemv(w, s, xq, sx))
    assert np.array_equal(direct, full[:128])


@pytest.mark.parametrize("n,k", [(300, 1152), (130, 128), (9000, 384)])
def test_w8a8_tensor_core_tier_ragged(n, k):
    # k % 128 == 0 takes the tensor-core tier for every row count: ragged last 128-row tile,
    # an odd number of 128-byte chunks (a half-empty last stage), strided rows and outputs
    w = synth.fp8_weight(n, k, 11, DEV)
    s = synth.row_scales(n, 11, DEV)
    x = synth.bf16_rows(128, k, 11, DEV)
    xq_full = torch.zeros(128, k + 48, dtype=torch.uint8, device=DEV)
    xq, sx = dl.w8a8_quantize_rows(x)
    xq_full[:, :k] = xq
    out_full = torch.full((128, n + 24), 0x7FC0, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    dl.w8a8_gemv(w, s, xq_full[:, :k], sx, out=out_full[:, :n])
    got = bits(out_full[:, :n])
    q_ref, sx_ref = og.w8a8_quantize_rows(bits(x))
    ref = og.w8a8_gemv(bits(w), bits(s), q_ref, sx_ref)
    assert_bf16_close(got, ref, f"w8a8 tensor-core tier n={n} k={k}")
    assert np.all(bits(out_full[:, n:]) == 0x7FC0), "wrote past n"
    for m in (1, 15, 16, 17, 48, 100, 127):
        part = bits(dl.w8a8_gemv(w, s, xq[:m], sx[:m]))
        assert np.array_equal(part, got[:m]), f"row invariance M={m}"
    assert dl.device_fault(reset=True) == 0


def test_w8a8_silu_proj_down_projection():
    n, k = 4096, 14336
    w = synth.fp8_weight(n, k, 9, DEV)
    s = synth.row_scales(n, 9, DEV)
    gate = synth.bf16_rows(24, k, 9, DEV, tensor_id=4)
    up = synth.bf16_rows(24, k, 9, DEV, tensor_id=5)
    out = bits(dl.w8a8_silu_proj(w, s, gate, up))
    sub = slice(0, n, 7)
    ref = og.w8a8_silu_proj(bits(w)[sub], bits(s)[sub], bits(gate), bits(up))
    assert_bf16_close(out[:, sub], ref, "w8a8 silu proj")


@pytest.mark.parametrize("n,k", [(14336, 4096), (1000, 1152), (300, 1040)])
def test_w8a8_gate_up_pair_one_quantize(n, k):
    # gate and up read one quantized copy of x: k % 128 == 0 runs one tensor-core launch over
    # the tiles of both weights (ragged last tile at n = 1000, 300), k = 1040 two register GEMVs
    wg = synth.fp8_weight(n, k, 13, DEV, tensor_id=1)
    wu = synth.fp8_weight(n, k, 13, DEV, tensor_id=6)
    sg = synth.row_scales(n, 13, DEV, tensor_id=2)
    su = synth.row_scales(n, 13, DEV, tensor_id=7)
    x = synth.bf16_rows(130, k, 13, DEV)
    g_out = torch.full((130, n + 8), 0x7FC0, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    u_out = torch.full((130, n + 8), 0x7FC0, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    dl.w8a8_gate_up_proj(wg, sg, wu, su, x, gate_out=g_out[:, :n], up_out=u_out[:, :n])
    g, u = bits(g_out[:, :n]), bits(u_out[:, :n])
    assert np.all(bits(g_out[:, n:]) == 0x7FC0) and np.all(bits(u_out[:, n:]) == 0x7FC0), "wrote past n"
    sub = slice(None) if n <= 1000 else slice(0, n, 7)
    q_ref, sx_ref = og.w8a8_quantize_rows(bits(x))
    assert_bf16_close(g[:, sub], og.w8a8_gemv(bits(wg)[sub], bits(sg)[sub], q_ref, sx_ref), f"gate n={n} k={k}")
    assert_bf16_close(u[:, sub], og.w8a8_gemv(bits(wu)[sub], bits(su)[sub], q_ref, sx_ref), f"up n={n} k={k}")
    for m in (1, 16, 17, 128):
        pg, pu = dl.w8a8_gate_up_proj(wg, sg, wu, su, x[:m])
        assert np.array_equal(bits(pg), g[:m]) and np.array_equal(bits(pu), u[:m]), f"row invariance M={m}"
    assert dl.device_fault(reset=True) == 0


# ---------------------------------------------------------------------------
# NVFP4 W4A16
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("n,k", [(2000, 4096), (77, 1024), (300, 1152)])
def test_w4a16_tiers(n, k):
    wp, ws, gl = synth.nvfp4_weight(n, k, 10, DEV)
    x = synth.bf16_rows(32, k, 10, DEV)
    full = bits(dl.w4a16_gemv(wp, ws, gl, x))
    ref = og.w4a16_gemv(bits(wp), bits(ws), np.float32(gl), bits(x))
    assert_bf16_close(full, ref, f"w4a16 n={n} k={k} M=32")
    for m in (1, 4, 5, 6, 7, 8, 16, 17):
        part = bits(dl.w4a16_gemv(wp, ws, gl, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"


# ---------------------------------------------------------------------------
# load-time FP4 dequant (bit-exact)
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("n,k", [(14336, 4096), (37, 48), (300, 1152)])
def test_nvfp4_dequant_bit_exact_both_conventions(n, k):
    wp, ws, _ = synth.nvfp4_weight(n, k, 30, DEV)
    for stored, reciprocal in [(448.0, True), (1.0 / 448.0, False), (3.0, True), (0.0, True)]:
        out = bits(dl.nvfp4_dequant_bf16(wp, ws, stored, reciprocal))
        ref = og.nvfp4_dequant_bf16(bits(wp), bits(ws), stored, reciprocal)
        assert np.array_equal(out, ref), (stored, reciprocal)
    # strided output: the padding columns stay untouched
    outb = torch.full((n, k + 24), 7.0, dtype=torch.bfloat16, device=DEV)
    dl.nvfp4_dequant_bf16(wp, ws, 448.0, True, out=outb[:, :k])
    assert np.array_equal(bits(outb[:, :k]), og.nvfp4_dequant_bf16(bits(wp), bits(ws), 448.0, True))
    assert (outb[:, k:] == 7.0).all()


@pytest.mark.parametrize("n,k,groups", [(64, 4096, 64 * 4096 // 32), (3, 80, 5), (7, 32, 1), (256, 512, 1024)])
def test_e8m0_fp4_dequant_bit_exact(n, k, groups):
    g = torch.Generator(device="cpu").manual_seed(31)
    wp = torch.randint(0, 256, (n * k // 2,), generator=g, dtype=torch.int32).to(torch.uint8)
    sc = torch.randint(100, 160, (groups,), generator=g, dtype=torch.int32).to(torch.uint8)
    sc[0] = 0                                             # special codes decode to 0
    sc[-1] = 255
    if groups > 2:
        sc[1] = 254                                       # 6 * 2^127 overflows float32 -> inf
    wp, sc = wp.to(DEV), sc.to(DEV)
    out = bits(dl.e8m0_fp4_dequant_bf16(wp, sc, n, k))
    ref = og.e8m0_fp4_dequant_bf16(bits(wp), bits(sc), n, k)
    assert np.array_equal(out, ref)


# ---------------------------------------------------------------------------
# q8_1 and Q6_K
# ---------------------------------------------------------------------------


def test_q8_1_quantize_bit_exact():
    k = 7168
    x = synth.bf16_rows(9, k, 4, DEV)
    x[2, :64] = 0
    x[3, :32] = torch.arange(32, dtype=torch.float32).to(torch.bfloat16) - 16.5
    q8 = bits(dl.q8_1_quantize_rows(x))
    ref = og.q8_1_quantize_rows(bits(x))
    assert np.array_equal(q8, ref)


@pytest.mark.parametrize("n,k", [(1000, 7168), (33, 512)])
def test_q6k_mmvq_and_head(n, k):
    blocks = synth.q6k_blocks(n, k, 4, DEV)
    x = synth.bf16_rows(20, k, 4, DEV)
    full = bits(dl.q6k_lm_head(blocks, x))
    ref = og.q6k_mmvq(bits(blocks), og.q8_1_quantize_rows(bits(x)))
    assert_bf16_close(full, ref, f"q6k n={n} k={k} M=20")
    q8 = dl.q8_1_quantize_rows(x)
    direct = bits(dl.q6k_mmvq(blocks, q8))
    assert np.array_equal(direct, full)
    for m in (1, 7, 8, 9):
        part = bits(dl.q6k_lm_head(blocks, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"


@pytest.mark.parametrize("n,k", [(1000, 7168), (37, 512), (45, 1280), (1000, 8192), (300, 8448)])
def test_q6k_streamed_and_register_kernels_agree(n, k):
    # 16-byte-aligned blocks take the TMA-streamed kernel (8-row stages; 4-row ones at k = 8192),
    # 2-byte-aligned ones the register-load kernel; k = 8448 (33 super-blocks: slices of 3)
    # stages the activation codes in shared memory instead of registers.  All use the same
    # arithmetic in the same order
    blocks = synth.q6k_blocks(n, k, 6, DEV)
    flat = torch.zeros(blocks.numel() + 16, dtype=torch.uint8, device=DEV)
    flat[2:2 + blocks.numel()] = blocks.reshape(-1)
    shifted = flat[2:2 + blocks.numel()].view(blocks.shape)
    assert shifted.data_ptr() % 16 == 2
    x = synth.bf16_rows(8, k, 6, DEV)
    q8 = dl.q8_1_quantize_rows(x)
    a = bits(dl.q6k_mmvq(blocks, q8))
    b = bits(dl.q6k_mmvq(shifted, q8))
    assert np.array_equal(a, b)
    # one row: the streamed kernel's column-0 build against the register-load kernel
    assert np.array_equal(bits(dl.q6k_mmvq(blocks, q8[:1])), a[:1])
    assert np.array_equal(bits(dl.q6k_mmvq(shifted, q8[:1])), a[:1])
    assert_bf16_close(a, og.q6k_mmvq(bits(blocks), og.q8_1_quantize_rows(bits(x))), f"q6k streamed n={n} k={k}")
    assert dl.device_fault(reset=True) == 0


@pytest.mark.parametrize("n,k", [(1000, 7168), (45, 1280), (300, 512), (200, 8448)])
def test_q6k_wide_tiers_one_pass(n, k):
    # (45 x 1280: the weight buffer ends off a 16-byte boundary, so its last bytes are staged
    # with plain loads; at k <= 8192 the 16-row tier runs as two 8-row passes, at 8448 as one
    # pass of the wide kernel)
    # 9..64 rows take one pass of the wide kernel (tiers 16 / 32 / 64); every row count must
    # give the 8-row kernels' bits (same slices, same order), and the oracle's values
    blocks = synth.q6k_blocks(n, k, 7, DEV)
    x = synth.bf16_rows(64, k, 7, DEV)
    full = bits(dl.q6k_lm_head(blocks, x))
    ref = og.q6k_mmvq(bits(blocks), og.q8_1_quantize_rows(bits(x)))
    assert_bf16_close(full, ref, f"q6k wide n={n} k={k} M=64")
    for m in (1, 8, 9, 15, 16, 17, 32, 33, 63):
        part = bits(dl.q6k_lm_head(blocks, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"
    # q8_1 rows that are only 4-byte aligned: 8-row passes, the same bits
    q8 = dl.q8_1_quantize_rows(x[:40])
    flat = torch.zeros(q8.numel() + 16, dtype=torch.uint8, device=DEV)
    flat[4:4 + q8.numel()] = q8.reshape(-1)
    shifted = flat[4:4 + q8.numel()].view(q8.shape)
    assert shifted.data_ptr() % 16 == 4
    assert np.array_equal(bits(dl.q6k_mmvq(blocks, shifted)), full[:40])
    # super-blocks that start only 2-byte aligned as a whole: 8-row passes as well
    fb = torch.zeros(blocks.numel() + 16, dtype=torch.uint8, device=DEV)
    fb[2:2 + blocks.numel()] = blocks.reshape(-1)
    bshift = fb[2:2 + blocks.numel()].view(blocks.shape)
    assert np.array_equal(bits(dl.q6k_mmvq(bshift, q8)), full[:40])
    assert dl.device_fault(reset=True) == 0


def test_q6k_kernel_element_map_hand_probes():
    # The 15 hand-derived probe blocks of tests/golden/q6k_single_byte_probes.txt as the 15
    # weight rows of a K = 256 matrix, against 256 one-hot q8_1 rows (row m: d = 1, code 1 at
    # value m): out[m, n] is then value m of probe block n, exactly (every expected value is a
    # BF16 integer).  Run through the wide kernel (64-row passes), the streamed 8-row kernel
    # (q8 rows only 4-byte aligned) and the register kernel (blocks only 2-byte aligned).
    from q6k_probes import load

    probes = load()
    n = len(probes)
    blocks = torch.from_numpy(np.stack([b for _, b, _ in probes])[:, None, :].copy()).to(DEV)
    want = np.stack([e for _, _, e in probes]).T                 # [256 values, n]
    q8 = np.zeros((256, 8, 36), np.uint8)
    for m in range(256):
        q8[m, m // 32, 0:4] = (0x00, 0x3C, 0x00, 0x3C)         # d = 1.0, s = 1.0
        q8[m, m // 32, 4 + m % 32] = 1
    q8d = torch.from_numpy(q8).to(DEV)
    got = {"wide": bits(dl.q6k_mmvq(blocks, q8d))}
    flat = torch.zeros(q8d.numel() + 16, dtype=torch.uint8, device=DEV)
    flat[4:4 + q8d.numel()] = q8d.reshape(-1)
    got["streamed 8-row"] = bits(dl.q6k_mmvq(blocks, flat[4:4 + q8d.numel()].view(q8d.shape)))
    fb = torch.zeros(blocks.numel() + 16, dtype=torch.uint8, device=DEV)
    fb[2:2 + blocks.numel()] = blocks.reshape(-1)
    got["register 8-row"] = bits(dl.q6k_mmvq(fb[2:2 + blocks.numel()].view(blocks.shape), q8d))
    for kind, g in got.items():
        v = nx.bf16_decode(g)
        bad = np.argwhere(v != want)
        assert bad.size == 0, (f"{kind}: (value, probe) {bad[:6].tolist()} got {v[tuple(bad[:6].T)].tolist()} "
                               f"want {want[tuple(bad[:6].T)].tolist()} ({probes[bad[0][1]][0]})")
    assert dl.device_fault(reset=True) == 0


def test_q6k_two_passes_128_rows():
    # 128 rows: two 64-row weight passes; the oracle on every output, and row invariance
    # against one 64-row pass of each half
    n, k = 1000, 7168
    blocks = synth.q6k_blocks(n, k, 8, DEV)
    x = synth.bf16_rows(128, k, 8, DEV)
    full = bits(dl.q6k_lm_head(blocks, x))
    ref = og.q6k_mmvq(bits(blocks), og.q8_1_quantize_rows(bits(x)))
    assert_bf16_close(full, ref, "q6k M=128")
    assert np.array_equal(bits(dl.q6k_lm_head(blocks, x[:64])), full[:64])
    assert np.array_equal(bits(dl.q6k_lm_head(blocks, x[64:])), full[64:])
    for m in (65, 100):
        assert np.array_equal(bits(dl.q6k_lm_head(blocks, x[:m])), full[:m]), f"row invariance M={m}"
    assert dl.device_fault(reset=True) == 0


@pytest.mark.parametrize("n,k", [(14336, 4096), (300, 1024)])
def test_w4a16_above_32_rows(n, k):
    # every M in 1..128: passes of at most 32 rows (one w4a16_gemv_tiers kernel_within-sized
    # launch each); the oracle on every output at M = 128, row invariance at 33 and 64
    wp, ws, gl = synth.nvfp4_weight(n, k, 21, DEV)
    x = synth.bf16_rows(128, k, 21, DEV)
    full = bits(dl.w4a16_gemv(wp, ws, gl, x))
    ref = og.w4a16_gemv(bits(wp), bits(ws), np.float32(gl), bits(x))
    assert_bf16_close(full, ref, f"w4a16 {n}x{k} M=128")
    for m in (1, 32, 33, 64):
        assert np.array_equal(bits(dl.w4a16_gemv(wp, ws, gl, x[:m])), full[:m]), f"row invariance M={m}"
    assert dl.device_fault(reset=True) == 0


# ---------------------------------------------------------------------------
# NVFP4 W4A4 (FP4 activations)
# ---------------------------------------------------------------------------


def _w4a4_rows(m, k, seed):
    # N(0,1) rows at a spread of magnitudes, a zero row, -0 values and tiny values
    x = synth.bf16_rows(m, k, seed, DEV) * torch.logspace(-3, 2, m, device=DEV).to(torch.bfloat16)[:, None]
    if m > 2:
        x[1] = 0
        x[2, ::7] = -0.0
        x[2, 1::7] = 1e-30
    return x


@pytest.mark.parametrize("m,k", [(40, 4096), (5, 1040), (130, 256)])
def test_nvfp4_quantize_rows_bit_exact(m, k):
    x = _w4a4_rows(m, k, 14)
    q, s, g = dl.nvfp4_quantize_rows(x)
    q_ref, s_ref, g_ref = og.nvfp4_quantize_rows(bits(x))
    assert np.array_equal(bits(g), g_ref)
    assert np.array_equal(bits(s), s_ref)
    assert np.array_equal(bits(q), q_ref)


@pytest.mark.parametrize("n,k", [(14336, 4096), (300, 1024), (77, 512), (130, 14336)])
def test_w4a4_gemv_and_proj(n, k):
    wp, ws, gw = synth.nvfp4_weight(n, k, 15, DEV)
    x = _w4a4_rows(70, k, 15)
    full = bits(dl.w4a4_proj(wp, ws, gw, x))                     # passes of up to 32 rows
    sub = slice(None) if n <= 1000 else slice(0, n, 9)
    q_ref, s_ref, g_ref = og.nvfp4_quantize_rows(bits(x))
    ref = og.w4a4_gemv(bits(wp)[sub], bits(ws)[sub], float(gw), q_ref, s_ref, g_ref)
    assert_bf16_close(full[:, sub], ref, f"w4a4 n={n} k={k} M=70")
    for m in (1, 7, 8, 9, 16, 17, 32, 33):
        part = bits(dl.w4a4_proj(wp, ws, gw, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"
    q, sc, g = dl.nvfp4_quantize_rows(x)
    direct = bits(dl.w4a4_gemv(wp, ws, gw, q, sc, g))
    assert np.array_equal(direct, full)
    assert dl.device_fault(reset=True) == 0


# ---------------------------------------------------------------------------
# full-size heads, sampled outputs
# ---------------------------------------------------------------------------


def _sample_rows(n):
    idx = np.concatenate([np.arange(0, 1024), np.arange(1024, n - 1024, 97), np.arange(n - 1024, n)])
    return np.unique(idx)


def test_fp8_head_full_size_sampled():
    n, k = 248320, 5120
    w = synth.fp8_weight(n, k, 1, DEV)
    s = synth.row_scales(n, 1, DEV)
    x = synth.bf16_rows(128, k, 1, DEV, std=0.5)
    idx = _sample_rows(n)
    wi, si = bits(w[torch.from_numpy(idx).to(DEV)]), bits(s[torch.from_numpy(idx).to(DEV)])
    full = bits(dl.lm_head_fp8_w8a16(w, s, x))
    ref = og.w8a16_gemv(wi, si, bits(x))
    assert_bf16_close(full[:, idx], ref, "fp8 head W8A16 M=128 sampled")
    for m in (1, 2, 4, 8, 16, 17, 32):
        part = bits(dl.lm_head_fp8_w8a16(w, s, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"
    # W8A8 on the same head, one 128-row call
    out8 = bits(dl.w8a8_proj(w, s, x))
    ref8 = og.w8a8_proj(wi, si, bits(x))
    assert_bf16_close(out8[:, idx], ref8, "fp8 head W8A8 M=128 sampled")


def test_q6k_head_full_size_sampled():
    # the Q6_K head config: 8-row launches, swept to 64 rows
    n, k = 129280, 7168
    blocks = synth.q6k_blocks(n, k, 4, DEV)
    x = synth.bf16_rows(64, k, 4, DEV)
    idx = _sample_rows(n)
    out = bits(dl.q6k_lm_head(blocks, x))
    ref = og.q6k_mmvq(bits(blocks[torch.from_numpy(idx).to(DEV)]), og.q8_1_quantize_rows(bits(x)))
    assert_bf16_close(out[:, idx], ref, "q6k head M=64 sampled")
    for m in (1, 8, 9, 16):
        part = bits(dl.q6k_lm_head(blocks, x[:m]))
        assert np.array_equal(part, out[:m]), f"row invariance M={m}"


def test_nvfp4_full_size_all_tiers():
    # the NVFP4 config: 14336 x 4096, M in {1,4,5,6,7,8,16,32}; the oracle covers every output
    n, k = 14336, 4096
    wp, ws, gl = synth.nvfp4_weight(n, k, 20, DEV)
    x = synth.bf16_rows(32, k, 4, DEV)
    full = bits(dl.w4a16_gemv(wp, ws, gl, x))
    ref = og.w4a16_gemv(bits(wp), bits(ws), np.float32(gl), bits(x))
    assert_bf16_close(full, ref, "nvfp4 14336x4096 M=32")
    for m in (1, 4, 5, 6, 7, 8, 16):
        part = bits(dl.w4a16_gemv(wp, ws, gl, x[:m]))
        assert np.array_equal(part, full[:m]), f"row invariance M={m}"


def test_w8a8_silu_down_full_size_128_rows():
    # the W8A8 down-projection config: 4096 x 14336, one 128-row call from bf16(silu(g)*u)
    n, k = 4096, 14336
    w = synth.fp8_weight(n, k, 10, DEV)
    s = synth.row_scales(n, 10, DEV)
    gate = synth.bf16_rows(128, k, 3, DEV, tensor_id=4)
    up = synth.bf16_rows(128, k, 3, DEV, tensor_id=5)
    out = bits(dl.w8a8_silu_proj(w, s, gate, up))
    sub = slice(0, n, 3)
    ref = og.w8a8_silu_proj(bits(w)[sub], bits(s)[sub], bits(gate), bits(up))
    assert_bf16_close(out[:, sub], ref, "w8a8 silu down M=128")
    for m in (1, 16, 64):
        part = bits(dl.w8a8_silu_proj(w, s, gate[:m], up[:m]))
        assert np.array_equal(part, out[:m]), f"row invariance M={m}"
    assert dl.device_fault(reset=True) == 0
