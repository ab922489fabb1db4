"""Pins of the oracle's load-time FP4 dequant (fp8_lut.rs, dequant_nvfp4_to_bf16 and
dequant_nvfp4_e8m0_to_bf16) against an independent restatement: plain Python floats, the
float32 rounding of `struct` (the C double -> float conversion) and a round-to-nearest-even
of the float32 bits to BF16 in integer arithmetic.  Exhaustive over all 16 E2M1 codes x all
256 scale codes, for both global conventions and for E8M0; plus the flat-index grouping."""

import math
import struct

import numpy as np
import pytest

from oracle import gemv as og
from oracle import numerics as nx

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0]


def f32_bits(v):
    """Nearest float32 of a Python float as its bit pattern (overflow -> inf)."""
    try:
        return struct.unpack("<I", struct.pack("<f", v))[0]
    except OverflowError:
        return 0x7F800000 | (0x80000000 if v < 0 else 0)


def bf16_of_f32_bits(b):
    """Round-to-nearest-even of float32 bits to BF16 bits (no NaN occurs here)."""
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) & 0xFFFF


def e4m3(code):
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 7
    if e == 0:
        return s * m / 8.0 * 2.0 ** -6
    return s * (1 + m / 8.0) * 2.0 ** (e - 7)


def test_nvfp4_dequant_exhaustive_both_conventions():
    codes = np.arange(16, dtype=np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)          # 16 codes in 8 bytes
    for stored, reciprocal in [(1.0, False), (0.25, False), (1.0 / 3.0, False), (448.0, True), (3.0, True),
                               (0.0, True)]:
        g = np.float32(0.0) if (reciprocal and stored == 0.0) else (
            np.float32(1.0) / np.float32(stored) if reciprocal else np.float32(stored))
        for sc in range(256):
            if sc & 0x7F == 0x7F:
                continue                                                   # NaN scale: outside the data
            got = og.nvfp4_dequant_bf16(packed[None, :], np.array([[sc]], np.uint8), stored, reciprocal)[0]
            for c in range(16):
                want = bf16_of_f32_bits(f32_bits(E2M1[c] * e4m3(sc) * float(g)))
                assert got[c] == want, (stored, reciprocal, sc, c)


def test_reciprocal_global_matches_direct_and_zero_gives_zero():
    rng = np.random.default_rng(21)
    packed = rng.integers(0, 256, (4, 32), dtype=np.uint8)
    scale = rng.integers(0, 0x7E, (4, 4), dtype=np.uint8)
    a = og.nvfp4_dequant_bf16(packed, scale, 4.0, True)
    b = og.nvfp4_dequant_bf16(packed, scale, 0.25, False)
    assert np.array_equal(a, b)
    z = og.nvfp4_dequant_bf16(packed, scale, 0.0, True)
    assert not nx.bf16_decode(z).any()


def test_e8m0_dequant_exhaustive():
    codes = np.arange(16, dtype=np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    for e in range(256):
        got = og.e8m0_fp4_dequant_bf16(packed, np.array([e], np.uint8), 1, 16)[0]
        scale = 0.0 if e in (0, 255) else math.ldexp(1.0, e - 127)
        for c in range(16):
            want = bf16_of_f32_bits(f32_bits(E2M1[c] * scale))
            assert got[c] == want, (e, c)


def test_e8m0_groups_follow_flat_indices_across_rows():
    # n=3, k=20: 60 values, 5 groups of 12 -> groups straddle row boundaries
    rng = np.random.default_rng(22)
    n, k = 3, 20
    packed = rng.integers(0, 256, n * k // 2, dtype=np.uint8)
    scales = np.array([120, 127, 130, 0, 140], dtype=np.uint8)
    got = og.e8m0_fp4_dequant_bf16(packed, scales, n, k)
    for f in range(n * k):
        byte = int(packed[f // 2])
        code = byte & 0xF if f % 2 == 0 else byte >> 4
        e = int(scales[f // 12])
        scale = 0.0 if e in (0, 255) else math.ldexp(1.0, e - 127)
        assert got[f // k, f % k] == bf16_of_f32_bits(f32_bits(E2M1[code] * scale)), f
    with pytest.raises(ValueError):
        og.e8m0_fp4_dequant_bf16(packed, scales[:4], n, k + 2)
