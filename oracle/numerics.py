"""Number formats of the method, decoded and encoded from their definitions.

Test infrastructure (see the package docstring); float64 numpy throughout.

Sources on the pages:
* E4M3 decode is imported by ``fp8_lut.rs`` (``FP8_E4M3_LUT``,
  ``fp8_e4m3_to_f32``) without its body.  Reading: OCP FP8 E4M3 ("FN"):
  1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals
  ``2^-6 * m/8``, no infinities, magnitude code 0x7F is NaN, max 448.
* ``f32_to_bf16`` is imported by ``fp8_lut.rs`` without its body.  Reading:
  IEEE round-to-nearest-even.  This oracle rounds a float64 value to BF16
  once, never through float32.
* E2M1 values: the table printed in ``fp8_lut.rs``,
  ``dequant_nvfp4_e8m0_to_bf16`` (``e2m1_table``).
* E8M0 values: ``fp8_lut.rs``, ``FP8_E8M0_LUT``: ``2^(e-127)`` for
  e = 1..254, and 0 for e = 0 and e = 255.
* The E4M3 encode used for activations is not printed.  Reading:
  round-to-nearest-even, with saturation: a magnitude above 448 becomes 448.
"""

import numpy as np

# ----------------------------------------------------------------------------
# generic "round a float64 to a binary format" helper
# ----------------------------------------------------------------------------


def _round_to_format(v, mant_bits, emin, max_finite, overflow_to_inf):
    """Round float64 ``v`` to nearest-even in a binary format.

    ``mant_bits`` stored mantissa bits, ``emin`` exponent of the smallest
    normal, ``max_finite`` largest finite magnitude.  Subnormals keep the
    quantum ``2^(emin - mant_bits)``.  Returns float64 values of the format
    (or +-inf on overflow when ``overflow_to_inf``, else +-max_finite).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, e = np.frexp(a)            # a = f * 2^e, 0.5 <= f < 1 -> exponent of a is e-1
    e = e.astype(np.int64) - 1
    e = np.maximum(e, emin)       # subnormal range shares the quantum of emin
    quantum = np.ldexp(1.0, e - mant_bits)
    r = np.rint(a / quantum) * quantum   # rint: ties to even; division by 2^n is exact
    r = np.where(a == 0, 0.0, r)
    if overflow_to_inf:
        r = np.where(r > max_finite, np.inf, r)
    else:
        r = np.minimum(r, max_finite)
    return np.copysign(r, v)


# ----------------------------------------------------------------------------
# BF16 / F16 / F32
# ----------------------------------------------------------------------------

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
F16_MAX = 65504.0


def bf16_decode(bits):
    """BF16 bit patterns (uint16) -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_rn(v):
    """float64 -> BF16 bits, round-to-nearest-even, overflow to inf."""
    r = _round_to_format(v, 7, -126, BF16_MAX, True)
    r32 = r.astype(np.float32)    # exact: every BF16 value is a float32 value
    return (np.atleast_1d(r32).view(np.uint32) >> 16).astype(np.uint16).reshape(np.shape(v))


def f16_decode(bits):
    """F16 bit patterns (uint16) -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def f16_rn(v):
    """float64 -> F16 bits, round-to-nearest-even, overflow to inf."""
    r = _round_to_format(v, 10, -14, F16_MAX, True)
    return np.atleast_1d(r.astype(np.float16)).view(np.uint16).reshape(np.shape(v))


def f32(v):
    """float64 -> nearest float32 value, returned as float64 (numpy's cast is RNE)."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# FP8 E4M3 (OCP "FN" variant)
# ----------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_value(code):
    """Value of one E4M3 byte from the definition (NaN for 0x7F / 0xFF)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:
        return sign * (2.0 ** -6) * (man / 8.0)
    return sign * (2.0 ** (exp - 7)) * (1.0 + man / 8.0)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes):
    """E4M3 bytes (any integer array) -> float64."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


# the finite non-negative values in code order 0x00..0x7E (increasing), used
# to map a rounded value back to its byte
_E4M3_POS = E4M3_TABLE[:0x7F]


def e4m3_rn_sat(v):
    """Values (float64, typically float32-exact) -> E4M3 bytes.

    Round-to-nearest-even on the E4M3 grid (3 mantissa bits, subnormal
    quantum 2^-9), then saturate: magnitudes above 448 give 448.  A negative
    value that rounds to zero gives -0 (0x80).  NaN input is outside the
    contract.
    """
    v = np.asarray(v, dtype=np.float64)
    r = _round_to_format(v, 3, -6, E4M3_MAX, False)
    mag = np.abs(r)
    code = np.searchsorted(_E4M3_POS, mag)
    if not np.array_equal(_E4M3_POS[np.minimum(code, 0x7E)], mag):
        raise AssertionError("rounded value is not on the E4M3 grid")
    return (code.astype(np.uint8) | np.where(np.signbit(r), 0x80, 0).astype(np.uint8)).astype(np.uint8)


# ----------------------------------------------------------------------------
# FP4 E2M1 and E8M0
# ----------------------------------------------------------------------------

# fp8_lut.rs, dequant_nvfp4_e8m0_to_bf16: the printed e2m1_table (code -> value)
E2M1_TABLE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
                       -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0], dtype=np.float64)


def e2m1_decode(codes):
    """4-bit E2M1 codes (0..15) -> float64."""
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_rn_sat(v):
    """Values (float64, typically float32-exact) -> 4-bit E2M1 codes (0..15).

    Round-to-nearest-even on the E2M1 grid (1 mantissa bit, subnormal quantum
    0.5: 0, 0.5, 1, 1.5, 2, 3, 4, 6), then saturate: magnitudes above 6 give
    6.  A negative value that rounds to zero gives -0 (code 8).  NaN input is
    outside the contract.
    """
    v = np.asarray(v, dtype=np.float64)
    r = _round_to_format(v, 1, 0, 6.0, False)
    mag = np.abs(r)
    code = np.searchsorted(E2M1_TABLE[:8], mag)
    if not np.array_equal(E2M1_TABLE[np.minimum(code, 7)], mag):
        raise AssertionError("rounded value is not on the E2M1 grid")
    return (code.astype(np.uint8) | np.where(np.signbit(r), 8, 0).astype(np.uint8)).astype(np.uint8)


def pack_nibbles(codes):
    """Codes [..., K] (0..15) -> packed bytes [..., K/2], even index in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    """Packed FP4 bytes [..., K/2] -> codes [..., K].

    fp8_lut.rs, dequant_nvfp4_e8m0_to_bf16: an even flat index is the low
    nibble of byte index/2, an odd one the high nibble.
    """
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


def e8m0_value(code):
    """fp8_lut.rs, FP8_E8M0_LUT: 2^(e-127) for e in 1..254; e = 0 and e = 255 give 0."""
    code = int(code) & 0xFF
    if code == 0 or code == 255:
        return 0.0
    return 2.0 ** (code - 127)


E8M0_TABLE = np.array([e8m0_value(c) for c in range(256)], dtype=np.float64)


def nvfp4_fold_global(global_scale, is_reciprocal):
    """fp8_lut.rs, dequant_nvfp4_to_bf16: one multiplier from the stored global.

    compressed-tensors stores a reciprocal (value = E2M1 * scale / global), so
    the multiplier is 1/global, with a zero global giving 0; ModelOpt stores a
    direct multiplier.  Computed in float32, as the loader does.
    """
    g = np.float32(global_scale)
    if is_reciprocal:
        return np.float32(0.0) if g == 0 else np.float32(1.0) / g
    return g
