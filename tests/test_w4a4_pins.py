"""Pins of the oracle's NVFP4 W4A4 path (the per-row FP4 activation quantize and the W4A4
GEMV) against things computed another way: the printed E2M1 table with a nearest-value
search, exact rational arithmetic, exactly representable rows, and the quantizer's error
bound."""

import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import gemv as og
from oracle import numerics as nx

TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # fp8_lut.rs, the printed e2m1_table (codes 0..7)


def _nearest_code(v):
    """Independent E2M1 rounding: nearest table magnitude, a tie to the even code (mantissa
    bit 0), beyond 6 the largest; the sign bit kept, also for a result of zero."""
    a = abs(Fraction(float(v)))
    best = min(range(8), key=lambda c: (abs(a - Fraction(TABLE[c])), c & 1))
    return best | (8 if np.signbit(v) else 0)


def _f32(v):
    return struct.unpack("<f", struct.pack("<f", v))[0]


def test_e2m1_rounding_against_nearest_search():
    vals = [i / 64.0 for i in range(-8 * 64, 8 * 64 + 1)]             # every 1/64 in [-8, 8]
    vals += [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0, 6.5, 1e30, -1e30, 1e-30, -1e-30, -0.0]
    vals += [np.nextafter(m, d) for m in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0) for d in (0.0, 10.0)]
    got = nx.e2m1_rn_sat(np.array(vals))
    for v, c in zip(vals, got):
        assert int(c) == _nearest_code(v), v


def test_pack_nibbles_inverts_unpack():
    rng = np.random.default_rng(41)
    p = rng.integers(0, 256, (3, 40), dtype=np.uint8)
    assert np.array_equal(nx.pack_nibbles(nx.unpack_nibbles(p)), p)


def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_quantize_reproduces_representable_rows():
    # row max 2688 -> g = 1; a block whose largest magnitude is 6 gets scale code 1.0, so
    # values from the E2M1 table come back exactly; a block at 2688 gets scale 448
    rng = np.random.default_rng(42)
    row = []
    for b in range(7):
        blk = [TABLE[i] * (-1) ** rng.integers(2) for i in rng.integers(0, 8, 16)]
        blk[int(rng.integers(16))] = 6.0
        row += blk
    row += [2688.0] + [448.0 * t for t in TABLE[1:]] + [0.0] * 8
    x = _bf16_bits([row])
    q, s, g = og.nvfp4_quantize_rows(x)
    assert g[0] == np.float32(1.0)
    assert list(nx.e4m3_decode(s[0])) == [1.0] * 7 + [448.0]
    back = og.nvfp4_dequant(q, s)[0] * float(g[0])
    assert np.array_equal(back, nx.bf16_decode(x)[0])


def test_quantize_steps_on_one_block():
    # follow the recipe by hand in exact arithmetic with float32 rounding at each step
    x = _bf16_bits([[0.3, -1.7, 2.2, 0.01, -0.02, 5.5, 3.3, -4.4, 0.9, 1.1, -0.6, 0.05, 2.9, -3.9, 0.0, 1.5]])
    q, s, g = og.nvfp4_quantize_rows(x)
    X = [float(v) for v in nx.bf16_decode(x)[0]]
    amax = max(abs(v) for v in X)
    gg = _f32(amax / 2688.0)
    assert g[0] == np.float32(gg)
    sf = _f32(amax / _f32(6.0 * gg))
    code = int(torch.tensor([sf]).to(torch.float8_e4m3fn).view(torch.uint8)[0])  # torch's RNE cast
    assert int(s[0, 0]) == code
    S = _f32(float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0]) * gg)
    codes = nx.unpack_nibbles(q)[0]
    for v, c in zip(X, codes):
        assert int(c) == _nearest_code(_f32(v / S)), v


def test_quantize_error_bound_and_zero_rows():
    rng = np.random.default_rng(43)
    x = _bf16_bits((rng.standard_normal((6, 256)) * rng.uniform(0.01, 50, (6, 1))).tolist())
    x[2] = 0                                                          # an all-zero row
    x[3, 16:32] = 0x8000                                              # a block of -0: scale 0
    x[4, 40] = 0x8000                                                 # one -0 in a live block
    q, s, g = og.nvfp4_quantize_rows(x)
    X = nx.bf16_decode(x)
    D = og.nvfp4_dequant(q, s) * g.astype(np.float64)[:, None]
    S = np.repeat(nx.e4m3_decode(s) * g.astype(np.float64)[:, None], 16, axis=1)
    # E2M1 spacing is at most 2 (between 4 and 6), and x / S stays below 6 * (1 + 1/16)
    # (the E4M3 scale rounds by at most 2^-4): every value is within one scale unit
    assert np.all(np.abs(D - X) <= S * (1.0 + 1e-6))
    assert g[2] == 0 and not s[2].any() and not q[2].any()
    assert not og.w4a4_proj(np.zeros((2, 128), np.uint8), np.zeros((2, 16), np.uint8), 1.0, x[2:3, :256]).any()
    assert s[3, 1] == 0 and not q[3, 8:16].any()                      # scale 0: codes 0
    assert nx.unpack_nibbles(q[4:5])[0, 40] == 8                      # -0 keeps its sign


def test_w4a4_gemv_brute_force_exact():
    rng = np.random.default_rng(44)
    N, K, M = 3, 48, 2
    wp = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    S = torch.from_numpy(rng.uniform(0.5, 4.0, (N, K // 16)).astype(np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()
    gw = np.float32(1.0) / np.float32(448.0)
    xq = rng.integers(0, 256, (M, K // 2)).astype(np.uint8)
    xs = torch.from_numpy(rng.uniform(0.01, 8.0, (M, K // 16)).astype(np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()
    xg = rng.uniform(1e-4, 1e-2, M).astype(np.float32)
    out = og.w4a4_gemv(wp, S, gw, xq, xs, xg)

    def dec(codes_byte, k):
        c = (codes_byte & 0xF) if k % 2 == 0 else (codes_byte >> 4)
        v = TABLE[c & 7]
        return -v if c & 8 else v

    def e4m3(c):
        return Fraction(float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0]))

    for m in range(M):
        for n in range(N):
            r = Fraction(0)
            for k in range(K):
                r += (Fraction(dec(int(wp[n, k // 2]), k)) * e4m3(int(S[n, k // 16])) *
                      Fraction(dec(int(xq[m, k // 2]), k)) * e4m3(int(xs[m, k // 16])))
            r *= Fraction(float(gw)) * Fraction(float(xg[m]))
            got = Fraction(float(nx.bf16_decode(out[m:m + 1, n:n + 1])[0, 0]))
            # correctly rounded: no BF16 value is closer to r than the result
            bits = int(out[m, n])
            for nb in (bits - 1, bits + 1):
                other = Fraction(float(nx.bf16_decode(np.array([[nb & 0xFFFF]], np.uint16))[0, 0]))
                assert abs(r - got) <= abs(r - other), (m, n)


def test_w4a4_proj_is_quantize_then_gemv():
    rng = np.random.default_rng(45)
    wp = rng.integers(0, 256, (5, 64)).astype(np.uint8)
    S = rng.integers(0x20, 0x50, (5, 8)).astype(np.uint8)
    x = _bf16_bits(rng.standard_normal((3, 128)).tolist())
    q, s, g = og.nvfp4_quantize_rows(x)
    assert np.array_equal(og.w4a4_proj(wp, S, 0.5, x), og.w4a4_gemv(wp, S, 0.5, q, s, g))
    with pytest.raises(ValueError):
        og.nvfp4_quantize_rows(x[:, :120])
