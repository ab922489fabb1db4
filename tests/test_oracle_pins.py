"""Pins for the CPU oracle: library routines, printed tables, closed forms, brute force.

None of these re-types an oracle formula: each compares the oracle with
something computed another way (torch / numpy conversion routines, exact
rational arithmetic in pure Python, values printed on the pages, or
properties that any correct implementation must have).
"""

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import gemv as og
from oracle import numerics as nx
from oracle import plan as op

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ---------------------------------------------------------------------------
# exact helpers (independent of the oracle's rounding code)
# ---------------------------------------------------------------------------


def _torch_e4m3(code):
    return float(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])


def _bf16_val(bits):
    return Fraction(float(torch.tensor([bits & 0xFFFF], dtype=torch.int32).to(torch.int16)
                          .view(torch.bfloat16).double()[0]))


def _assert_correctly_rounded_bf16(r, bits):
    """bits must be a nearest BF16 to the exact rational r, ties to even."""
    bits = int(bits) & 0xFFFF
    v = _bf16_val(bits)
    d = abs(r - v)
    for nb in (bits - 1, bits + 1):
        nb &= 0xFFFF
        if (nb & 0x7F80) == 0x7F80:      # inf / nan neighbour
            continue
        if (nb ^ bits) & 0x8000:         # crossed the sign: ignore (values are not near 0)
            continue
        dn = abs(r - _bf16_val(nb))
        assert d <= dn, (r, bits, nb)
        if d == dn:
            assert bits & 1 == 0, "tie must go to the even mantissa"


def _rand_e4m3_codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C        # no NaN codes
    return c


def _rand_bf16(rng, shape, scale=1.0):
    return torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# E4M3
# ---------------------------------------------------------------------------


def test_e4m3_table_matches_torch_all_codes():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    tab = nx.E4M3_TABLE
    assert np.array_equal(np.isnan(ref), np.isnan(tab))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], tab[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(tab[ok]))


def test_e4m3_table_landmarks():
    assert nx.e4m3_value(0x7E) == 448.0
    assert nx.e4m3_value(0x01) == 2.0 ** -9           # smallest subnormal
    assert nx.e4m3_value(0x07) == 7 * 2.0 ** -9       # largest subnormal
    assert nx.e4m3_value(0x08) == 2.0 ** -6           # smallest normal
    assert nx.e4m3_value(0x38) == 1.0
    assert nx.e4m3_value(0xB8) == -1.0
    assert math.copysign(1.0, nx.e4m3_value(0x80)) == -1.0 and nx.e4m3_value(0x80) == 0.0
    assert math.isnan(nx.e4m3_value(0x7F)) and math.isnan(nx.e4m3_value(0xFF))


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    mags = np.exp2(rng.uniform(-12, math.log2(448.0), 20000))
    vals = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    fin = nx.E4M3_TABLE[:0x7F]
    mids = ((fin[1:] + fin[:-1]) / 2).astype(np.float32)  # every midpoint is float32-exact
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(0))
    vals = np.concatenate([vals, mids, up, dn, -mids, -up, -dn, fin.astype(np.float32)])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = nx.e4m3_rn_sat(vals.astype(np.float64))
    assert np.array_equal(ref, got)


def test_e4m3_encode_saturation_and_ties():
    enc = lambda v: int(nx.e4m3_rn_sat(np.array([v]))[0])  # noqa: E731
    for v in (448.0, 449.0, 463.9, 464.0, 465.0, 480.0, 1e30):
        assert enc(v) == 0x7E, v
        assert enc(-v) == 0xFE, v
    assert enc(2.0 ** -10) == 0x00          # tie between 0 and 2^-9 -> even (0)
    assert enc(-(2.0 ** -10)) == 0x80
    assert enc(3 * 2.0 ** -10) == 0x02      # tie between 1 and 2 (x 2^-9) -> even
    assert enc(1.0 + 1.0 / 16) == 0x38      # tie between 1.0 and 1.125 -> 1.0
    assert enc(1.0 + 3.0 / 16) == 0x3A      # tie between 1.125 and 1.25 -> 1.25


# ---------------------------------------------------------------------------
# BF16 / F16
# ---------------------------------------------------------------------------


def _interesting_f32(rng, n):
    e = rng.integers(-149, 128, n)
    m = rng.uniform(1.0, 2.0, n)
    v = (np.ldexp(m, e) * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    bits = rng.integers(0, 2 ** 32, n, dtype=np.uint64).astype(np.uint32)
    raw = bits.view(np.float32)
    raw = raw[np.isfinite(raw)]
    ties = (rng.integers(0, 2 ** 16, n, dtype=np.uint64).astype(np.uint32) << 16 | 0x8000).view(np.float32)
    ties = ties[np.isfinite(ties)]
    return np.concatenate([v, raw, ties, np.array([0.0, -0.0, 3.3895314e38, 3.4e38], np.float32)])


def test_bf16_rn_matches_torch_on_float32_values():
    rng = np.random.default_rng(2)
    v = _interesting_f32(rng, 30000)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = nx.bf16_rn(v.astype(np.float64))
    assert np.array_equal(ref, got)


def test_bf16_rn_rounds_float64_once():
    # via float32 this would be a tie and go to 1.0 (0x3F80)
    assert int(nx.bf16_rn(np.array([1.0 + 2.0 ** -8 + 2.0 ** -30]))[0]) == 0x3F81
    assert int(nx.bf16_rn(np.array([1.0 + 2.0 ** -8]))[0]) == 0x3F80
    big = (2.0 - 2.0 ** -8) * 2.0 ** 127          # midpoint between max and 2^128 -> inf
    assert int(nx.bf16_rn(np.array([big]))[0]) == 0x7F80
    assert int(nx.bf16_rn(np.array([np.nextafter(big, 0)]))[0]) == 0x7F7F


def test_bf16_decode_matches_torch():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = nx.bf16_decode(bits)
    ok = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    assert np.array_equal(ref[ok], got[ok])


def test_f16_rn_matches_numpy_on_float32_values():
    rng = np.random.default_rng(3)
    v = _interesting_f32(rng, 30000)
    ref = v.astype(np.float16).view(np.uint16)
    got = nx.f16_rn(v.astype(np.float64))
    assert np.array_equal(ref, got)


def test_f16_rn_rounds_float64_once():
    assert int(nx.f16_rn(np.array([1.0 + 2.0 ** -11 + 2.0 ** -40]))[0]) == 0x3C01
    assert int(nx.f16_rn(np.array([65520.0]))[0]) == 0x7C00
    assert int(nx.f16_rn(np.array([65519.99]))[0]) == 0x7BFF


# ---------------------------------------------------------------------------
# E2M1, nibble order, E8M0, global fold
# ---------------------------------------------------------------------------


def test_e2m1_table_matches_printed_table():
    rows = _golden_rows("e2m1_table.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = nx.e2m1_decode(np.array([int(code)]))[0]
        assert got == float(val)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(val))


def test_nibble_order_even_index_is_low_nibble():
    codes = nx.unpack_nibbles(np.array([[0x21, 0xF0]], dtype=np.uint8))
    assert codes.tolist() == [[0x1, 0x2, 0x0, 0xF]]


def test_e8m0_matches_torch_and_page_specials():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for c in range(1, 255):
        assert nx.e8m0_value(c) == ref[c]
    for code, val in _golden_rows("e8m0_special.txt"):
        assert nx.e8m0_value(int(code)) == float(val)


def test_nvfp4_global_fold_cases():
    for conv, g, expect in _golden_rows("nvfp4_global_fold.txt"):
        got = nx.nvfp4_fold_global(float(g), conv == "reciprocal")
        assert float(got) == float.fromhex(expect), (conv, g)


# ---------------------------------------------------------------------------
# GEMV definitions against exact rational arithmetic
# ---------------------------------------------------------------------------


def test_w8a16_brute_force_exact():
    rng = np.random.default_rng(4)
    N, K, M = 5, 64, 3
    w = _rand_e4m3_codes(rng, (N, K))
    s = rng.uniform(1e-3, 4e-3, N).astype(np.float32)
    x = _rand_bf16(rng, (M, K))
    out = og.w8a16_gemv(w, s, x)
    for m in range(M):
        for n in range(N):
            r = sum(Fraction(_torch_e4m3(int(w[n, k]))) * _bf16_val(int(x[m, k])) for k in range(K))
            _assert_correctly_rounded_bf16(r * Fraction(float(s[n])), out[m, n])


def test_w8a16_single_weight_and_orientation():
    N, K = 3, 32
    w = np.zeros((N, K), np.uint8)
    w[1, 5] = 0x7E                                  # 448 at row 1, k = 5
    s = np.array([1.0, 0.5, 1.0], np.float32)
    x = np.zeros((2, K), np.uint16)
    x[0, 5] = 0x3F80                                # 1.0
    x[1, 5] = 0x4000                                # 2.0
    out = og.w8a16_gemv(w, s, x)
    vals = nx.bf16_decode(out)
    assert vals.tolist() == [[0.0, 224.0, 0.0], [0.0, 448.0, 0.0]]


def test_w8a16_scale_is_linear_and_rows_are_independent():
    rng = np.random.default_rng(5)
    w = _rand_e4m3_codes(rng, (16, 48))
    s = rng.uniform(1e-3, 4e-3, 16).astype(np.float32)
    x = _rand_bf16(rng, (4, 48))
    a = og.w8a16_gemv(w, s, x)
    b = og.w8a16_gemv(w, (s * 2).astype(np.float32), x)
    assert np.array_equal(nx.bf16_decode(a) * 2, nx.bf16_decode(b))
    for m in range(4):
        assert np.array_equal(og.w8a16_gemv(w, s, x[m:m + 1])[0], a[m])


def test_w8a8_quantize_matches_torch_cast():
    rng = np.random.default_rng(6)
    x = _rand_bf16(rng, (5, 96), scale=3.0)
    x[3] = 0                                        # an all-zero row
    x[4] = 0
    x[4, 7] = 0xC0A0                                # a single -5.0
    q, sx = og.w8a8_quantize_rows(x)
    xv = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float()
    amax = xv.abs().amax(dim=1)
    assert np.array_equal(sx, (amax / 448.0).numpy())   # float32 division in torch
    for m in range(3):
        ref = (xv[m] / torch.tensor(sx[m])).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(q[m], ref)
    assert sx[3] == 0 and not q[3].any()
    assert q[4, 7] == 0xFE and np.count_nonzero(q[4]) == 1


def test_w8a8_gemv_brute_force_exact():
    rng = np.random.default_rng(7)
    N, K, M = 4, 64, 2
    w = _rand_e4m3_codes(rng, (N, K))
    s = rng.uniform(1e-3, 4e-3, N).astype(np.float32)
    q = _rand_e4m3_codes(rng, (M, K))
    sx = rng.uniform(1e-3, 1e-2, M).astype(np.float32)
    out = og.w8a8_gemv(w, s, q, sx)
    for m in range(M):
        for n in range(N):
            r = sum(Fraction(_torch_e4m3(int(w[n, k]))) * Fraction(_torch_e4m3(int(q[m, k]))) for k in range(K))
            _assert_correctly_rounded_bf16(r * Fraction(float(s[n])) * Fraction(float(sx[m])), out[m, n])


def test_silu_product_matches_torch_silu():
    rng = np.random.default_rng(8)
    g = _rand_bf16(rng, (3, 200), scale=4.0)
    u = _rand_bf16(rng, (3, 200))
    h = og.silu_mul_bf16(g, u)
    gt = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).double()
    ut = torch.from_numpy(u.view(np.int16)).view(torch.bfloat16).double()
    p = (torch.nn.functional.silu(gt) * ut).numpy()
    got = nx.bf16_decode(h)
    # correctly rounded from the float64 product (ties and 1-ulp double differences aside)
    ref = torch.from_numpy(p).float().to(torch.bfloat16).double().numpy()
    close = np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7
    assert close.all()
    assert (got == ref).mean() > 0.999


def _finite_bf16_bits():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    return b[(b & 0x7F80) != 0x7F80]


def _mp_round_f32(v):
    """Nearest float32 to the mpmath value v (no ties: v is transcendental), inf on overflow."""
    import mpmath as mp

    if v > mp.mpf(float(np.finfo(np.float32).max)) * (1 + mp.mpf(2) ** -25):
        return math.inf
    c = np.float32(float(v))
    best, bd = None, None
    for cand in (np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))):
        if not np.isfinite(cand) or cand < 0:
            continue
        d = abs(v - mp.mpf(float(cand)))
        if bd is None or d < bd:
            best, bd = float(cand), d
    return best


def test_silu_exp_step_is_correctly_rounded_for_every_bf16():
    # e^-g rounded to float32, for every finite BF16 g, against a 200-bit mpmath evaluation
    import mpmath as mp

    gb = _finite_bf16_bits()
    g = nx.bf16_decode(gb)
    got = og.silu_exp_neg_f32(g)
    mp.mp.prec = 200
    for gi, e in zip(g, got):
        if gi > 104.0:                      # e^-g < 2^-150: rounds to +0
            assert e == 0.0, gi
        elif gi < -89.0:                    # e^-g > float32 max: inf
            assert e == math.inf, gi
        else:
            assert e == _mp_round_f32(mp.exp(-mp.mpf(float(gi)))), gi


def test_silu_agrees_with_float64_definition_off_midpoints():
    # The float32 chain (four correctly rounded steps, relative error < 2^-22) must round to
    # the BF16 of the float64 definition wherever that is farther than 2^-20 from a midpoint.
    rng = np.random.default_rng(81)
    gb = _finite_bf16_bits()
    g = nx.bf16_decode(gb)
    keep = np.abs(g) < 60.0
    gb, g = gb[keep], g[keep]
    ub = _rand_bf16(rng, gb.shape)
    u = nx.bf16_decode(ub)
    h = nx.bf16_decode(og.silu_mul_bf16(gb, ub))
    p = g / (1.0 + np.exp(-g)) * u                      # float64 definition
    a = np.abs(p)
    _, ex = np.frexp(a)
    quantum = np.ldexp(1.0, np.maximum(ex - 1, -126) - 7)
    frac = a / quantum - np.floor(a / quantum)
    near = (np.abs(frac - 0.5) * quantum <= a * 2.0 ** -20) & (a > 0)
    ref = torch.from_numpy(p).float().to(torch.bfloat16).double().numpy()
    # torch rounds float64 -> float32 -> BF16; off midpoints that is the BF16 of p
    assert np.array_equal(h[~near], ref[~near])
    # for large g, silu(g)*u is nearly the exact product of two 8-bit significands, which
    # lands on a BF16 midpoint about once in 128; the band stays a small minority
    assert near.mean() < 0.03
    ulp = np.ldexp(1.0, np.maximum(np.frexp(np.abs(ref))[1] - 1, -126) - 7)
    assert np.all(np.abs(h[near] - ref[near]) <= ulp[near])


def test_silu_special_values():
    one = np.array([0x3F80], np.uint16)
    def h(gbits, ubits=one):
        return nx.bf16_decode(og.silu_mul_bf16(np.array([gbits], np.uint16), np.asarray(ubits, np.uint16)))[0]
    assert h(0x0000) == 0.0                               # silu(0) = 0
    assert h(0x42C8) == 100.0                             # e^-100 is far below half an ulp of 1
    z = h(0xC2C8)                                         # g = -100: e^100 overflows float32 -> -0
    assert z == 0.0 and math.copysign(1.0, z) < 0
    assert h(0x3F80) == 0.73046875                        # silu(1) = 0.7310585786...
    assert h(0xBF80) == -0.26953125                       # silu(-1) = -0.2689414214...
    assert h(0x4000, np.array([0xC000], np.uint16)) == -3.515625  # silu(2) * -2 = -3.5231883...


def test_w4a16_brute_force_exact():
    rng = np.random.default_rng(9)
    N, K, M = 3, 64, 2
    wp = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    S = torch.from_numpy(rng.uniform(0.5, 4.0, (N, K // 16)).astype(np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()
    g = np.float32(1.0) / np.float32(448.0)
    x = _rand_bf16(rng, (M, K))
    out = og.w4a16_gemv(wp, S, g, x)
    table = {int(c): float(v) for c, v in _golden_rows("e2m1_table.txt")}
    for m in range(M):
        for n in range(N):
            r = Fraction(0)
            for k in range(K):
                byte = int(wp[n, k // 2])
                code = (byte & 0xF) if k % 2 == 0 else (byte >> 4)
                r += Fraction(table[code]) * Fraction(_torch_e4m3(int(S[n, k // 16]))) * _bf16_val(int(x[m, k]))
            _assert_correctly_rounded_bf16(r * Fraction(float(g)), out[m, n])


def test_w4a16_unit_scales_reduce_to_e2m1_matmul():
    rng = np.random.default_rng(10)
    N, K = 4, 32
    wp = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    S = np.full((N, K // 16), 0x38, np.uint8)        # E4M3 1.0
    x = np.full((1, K), 0x3F80, np.uint16)           # all ones
    out = nx.bf16_decode(og.w4a16_gemv(wp, S, np.float32(1.0), x))[0]
    table = {int(c): float(v) for c, v in _golden_rows("e2m1_table.txt")}
    for n in range(N):
        tot = sum(table[int(b) & 0xF] + table[int(b) >> 4] for b in wp[n])
        assert out[n] == tot       # small sums of halves: exact in bf16


def test_q8_1_hand_cases():
    K = 64
    x = np.zeros((1, K), np.float32)
    x[0, 0] = 127.0
    x[0, 1:6] = [2.5, -2.5, 0.5, 1.5, -0.5]          # d = 1: exact ties -> away from zero
    # block 1 stays zero
    xb = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    q8 = og.q8_1_quantize_rows(xb)
    assert q8.shape == (1, 2, 36)
    b0 = q8[0, 0]
    assert b0[0:2].view(np.uint16)[0] == 0x3C00      # d = 1.0 in f16
    qs = b0[4:].view(np.int8)
    assert qs[:6].tolist() == [127, 3, -3, 1, 2, -1]
    assert not qs[6:].any()
    assert b0[2:4].view(np.uint16)[0] == np.float16(129.0).view(np.uint16)   # s = d * sum(qs)
    assert not q8[0, 1].any()                          # all-zero block: d = s = 0, qs = 0


def test_q8_1_properties_random():
    rng = np.random.default_rng(11)
    x = _rand_bf16(rng, (3, 256))
    q8 = og.q8_1_quantize_rows(x)
    d, s, qs = og.q8_1_fields(q8)
    xv = nx.bf16_decode(x).reshape(3, 8, 32)
    qv = qs.reshape(3, 8, 32)
    assert np.abs(qv).max() <= 127
    imax = np.abs(xv).argmax(axis=2)
    for m in range(3):
        for b in range(8):
            assert abs(qv[m, b, imax[m, b]]) == 127
            dd = float(np.float32(np.abs(xv[m, b]).max()) / np.float32(127))
            assert np.all(np.abs(xv[m, b] - qv[m, b] * dd) <= dd * 0.5 * (1 + 1e-6))
            assert abs(d[m, b] - dd) <= dd * 2.0 ** -11


def _q6k_block(ql, qh, sc, d_bits):
    b = np.zeros(210, np.uint8)
    b[0:128] = ql
    b[128:192] = qh
    b[192:208] = np.asarray(sc, np.int8).view(np.uint8)
    b[208:210] = np.frombuffer(np.uint16(d_bits).tobytes(), np.uint8)
    return b


def test_q6k_uniform_blocks_decode_to_constant():
    for lo in (0, 5, 15):
        for hi in range(4):
            qh_byte = hi | hi << 2 | hi << 4 | hi << 6
            blk = _q6k_block(np.full(128, lo | lo << 4), np.full(64, qh_byte), np.arange(16) - 8, 0x3C00)
            q, sc, d = og.q6k_unpack(blk[None])
            assert np.all(q == (lo | hi << 4))
            assert sc[0].tolist() == list(range(-8, 8)) and d[0] == 1.0


def test_q6k_code_sum_is_order_free():
    rng = np.random.default_rng(12)
    for _ in range(20):
        ql = rng.integers(0, 256, 128)
        qh = rng.integers(0, 256, 64)
        blk = _q6k_block(ql, qh, np.zeros(16), 0)
        q, _, _ = og.q6k_unpack(blk[None])
        lows = int(np.sum(ql & 0xF) + np.sum(ql >> 4))
        highs = int(sum(((int(b) >> (2 * t)) & 3) for b in qh for t in range(4)))
        assert int(q.sum()) == lows + 16 * highs
        assert q.min() >= 0 and q.max() <= 63


def test_q6k_mmvq_integer_reduction():
    rng = np.random.default_rng(13)
    N, K = 3, 256 * 2
    blocks = np.stack([np.stack([_q6k_block(rng.integers(0, 256, 128), rng.integers(0, 256, 64),
                                            np.ones(16), 0x3C00) for _ in range(K // 256)]) for _ in range(N)])
    # q8_1 rows with d = 1 and a constant code c per row: the dot is order free
    M = 2
    q8 = np.zeros((M, K // 32, 36), np.uint8)
    consts = [3, -2]
    for m in range(M):
        q8[m, :, 0:2] = np.frombuffer(np.uint16(0x3C00).tobytes(), np.uint8)
        q8[m, :, 4:] = np.int8(consts[m]).view(np.uint8)
    out = og.q6k_mmvq(blocks, q8)
    for n in range(N):
        lows = int(np.sum(blocks[n, :, 0:128] & 0xF) + np.sum(blocks[n, :, 0:128] >> 4))
        highs = int(sum(((int(b) >> (2 * t)) & 3) for b in blocks[n, :, 128:192].ravel() for t in range(4)))
        total = lows + 16 * highs - 32 * K
        for m in range(M):
            _assert_correctly_rounded_bf16(Fraction(consts[m] * total), out[m, n])


def test_q6k_mmvq_brute_force_exact():
    rng = np.random.default_rng(14)
    N, K, M = 2, 256, 2
    blocks = np.stack([np.stack([_q6k_block(rng.integers(0, 256, 128), rng.integers(0, 256, 64),
                                            rng.integers(-32, 32, 16),
                                            np.float16(rng.uniform(1e-4, 1e-3)).view(np.uint16))])
                       for _ in range(N)])
    x = _rand_bf16(rng, (M, K))
    q8 = og.q8_1_quantize_rows(x)
    out = og.q6k_mmvq(blocks, q8)
    for n in range(N):
        q, sc, dw = og.q6k_unpack(blocks[n, 0])
        for m in range(M):
            r = Fraction(0)
            for i in range(K):
                blk = q8[m, i // 32]
                dx = Fraction(float(blk[0:2].view(np.float16)[0]))
                qsv = int(blk[4 + i % 32:5 + i % 32].view(np.int8)[0])
                r += Fraction(float(dw)) * int(sc[i // 16]) * dx * (int(q[i]) - 32) * qsv
            _assert_correctly_rounded_bf16(r, out[m, n])


def _q6k_values(blocks, unpack=og.q6k_unpack):
    q, sc, d = unpack(blocks)
    return d[..., None] * np.repeat(sc, 16, axis=-1) * (q - 32)


def test_q6k_element_map_hand_probes():
    # tests/golden/q6k_single_byte_probes.txt: one byte (or a few) set at a time, the 256
    # expected values derived by hand from the public GGUF Q6_K layout; every nibble, qh bit
    # pair, half, scale index and the position of d is probed
    from q6k_probes import load

    probes = load()
    assert len(probes) == 15
    for name, blk, exp in probes:
        got = _q6k_values(blk[None])[0]
        bad = np.flatnonzero(got != exp)
        assert bad.size == 0, f"{name}: elements {bad[:8].tolist()} got {got[bad[:8]].tolist()}"


def _gguf_q6k():
    gq = pytest.importorskip("gguf.quants")
    from gguf import GGMLQuantizationType

    return lambda b: gq.dequantize(np.ascontiguousarray(b, np.uint8), GGMLQuantizationType.Q6_K)


def test_q6k_element_map_matches_gguf_library():
    # gguf.quants is an independent implementation of the public Q6_K block format (a library
    # routine).  Its float32 result is d * sc * (q - 32) rounded once (d*sc is exact in f32),
    # so the oracle's float64 value rounded to f32 must equal it bit for bit.  Blocks: every
    # byte value in ql and qh, every int8 scale, several d.
    deq = _gguf_q6k()
    rng = np.random.default_rng(16)
    b = rng.integers(0, 256, (256, 210)).astype(np.uint8)
    b[:, 0] = np.arange(256)                       # every ql byte value (low/high nibble pairs)
    b[:, 128] = np.arange(256)[::-1]               # every qh byte value (all bit pairs)
    b[:, 192] = np.arange(256)                     # every int8 scale
    d = np.concatenate([rng.uniform(1e-4, 1e-3, 200), rng.uniform(0.5, 4.0, 56)])
    b[:, 208:210] = np.frombuffer(np.float16(d).tobytes(), np.uint8).reshape(256, 2)
    ref = deq(b)
    got = _q6k_values(b).astype(np.float32)
    assert ref.shape == got.shape == (256, 256)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # the hand probes agree with the library too
    from q6k_probes import load

    for name, blk, exp in load():
        assert np.array_equal(deq(blk[None])[0].astype(np.float64), exp), name


def test_q6k_element_map_pins_catch_a_nibble_swap():
    # a plausible slip: values 32..63 of each half from the high nibble of ql[64h + l] and
    # values 64..95 from the low nibble of ql[64h + 32 + l] (t = 1 and t = 2 swapped).  Both
    # pins above must reject it.
    def swapped_unpack(blocks):
        q, sc, d = og.q6k_unpack(blocks)
        q2 = q.copy()
        for h in range(2):
            o = 128 * h
            q2[..., o + 32:o + 64], q2[..., o + 64:o + 96] = q[..., o + 64:o + 96], q[..., o + 32:o + 64]
        return q2, sc, d

    from q6k_probes import load

    probes = load()
    assert any(not np.array_equal(_q6k_values(blk[None], swapped_unpack)[0], exp) for _, blk, exp in probes)
    deq = _gguf_q6k()
    rng = np.random.default_rng(17)
    b = rng.integers(0, 256, (8, 210)).astype(np.uint8)
    b[:, 208:210] = np.frombuffer(np.float16(np.full(8, 1e-3)).tobytes(), np.uint8).reshape(8, 2)
    assert not np.array_equal(_q6k_values(b, swapped_unpack).astype(np.float32), deq(b))


def test_row_invariance_all_formats():
    rng = np.random.default_rng(15)
    N, K, M = 8, 256, 5
    x = _rand_bf16(rng, (M, K))
    w = _rand_e4m3_codes(rng, (N, K))
    s = rng.uniform(1e-3, 4e-3, N).astype(np.float32)
    wp = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    S = np.full((N, K // 16), 0x40, np.uint8)
    blocks = rng.integers(0, 256, (N, 1, 210)).astype(np.uint8)
    blocks[:, :, 208:210] = np.frombuffer(np.float16(5e-4).tobytes(), np.uint8)
    fulls = [og.w8a16_gemv(w, s, x), og.w8a8_proj(w, s, x), og.w4a16_gemv(wp, S, np.float32(1 / 448), x),
             og.q6k_mmvq(blocks, og.q8_1_quantize_rows(x))]
    for m in range(M):
        one = x[m:m + 1]
        singles = [og.w8a16_gemv(w, s, one), og.w8a8_proj(w, s, one), og.w4a16_gemv(wp, S, np.float32(1 / 448), one),
                   og.q6k_mmvq(blocks, og.q8_1_quantize_rows(one))]
        for f, sgl in zip(fulls, singles):
            assert np.array_equal(f[m], sgl[0])


# ---------------------------------------------------------------------------
# host plan
# ---------------------------------------------------------------------------


def test_chunk_plan_covers_rows_in_order():
    for width in (8, 16, 128):
        for rows in range(0, 300):
            p = op.chunk_plan(rows, width)
            assert sum(c for _, c in p) == rows
            assert all(1 <= c <= width for _, c in p)
            assert [o for o, _ in p] == [sum(c for _, c in p[:i]) for i in range(len(p))]
            assert all(c == width for _, c in p[:-1])
    assert op.chunk_plan(17, 16) == [(0, 16), (16, 1)]
    assert len(op.chunk_plan(128, 16)) == 8


def test_select_tier_properties_exhaustive():
    widths = [4, 5, 6, 7, 8]
    for mask in range(32):
        present = [(mask >> i) & 1 == 1 for i in range(5)]
        for m in range(0, 12):
            i = op.select_tier(m, widths, present)
            cover = [j for j in range(5) if present[j] and widths[j] >= m]
            if m == 0 or not cover:
                assert i is None
            else:
                assert present[i] and widths[i] >= m
                assert widths[i] == min(widths[j] for j in cover)
