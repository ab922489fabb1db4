"""The W8A16 tensor-core reading, checked on the CPU: a BF16 row scaled by a power of two
into [2^7, 2^8) splits into two E4M3 terms hi = e4m3(x'), lo = e4m3(16 (x' - hi)) with
hi + lo / 16 == x' exactly for every |x'| >= 2^-6, and an error of at most 2^-14 below.

Exhaustive over all positive finite BF16 values below 2^8 (the scaled range), using the
oracle's E4M3 rounding (round-to-nearest-even on the E4M3 grid).
"""

import numpy as np

from oracle import numerics as nx


def _split(v):
    hi = nx.e4m3_decode(nx.e4m3_rn_sat(v))
    lo = nx.e4m3_decode(nx.e4m3_rn_sat((v - hi) * 16.0))
    return hi, lo


def _all_bf16_below(limit):
    bits = np.arange(1, 0x7F80, dtype=np.uint32)
    v = (bits << 16).view(np.float32).astype(np.float64)
    return v[v < limit]


def test_two_term_split_exact_within_range():
    v = _all_bf16_below(256.0)
    for sign in (1.0, -1.0):
        hi, lo = _split(sign * v)
        rec = hi + lo / 16.0
        err = np.abs(rec - sign * v)
        big = v >= 2.0 ** -6
        assert np.all(err[big] == 0.0)
        assert err[~big].max() <= 2.0 ** -14
        assert np.all(np.abs(hi) <= 256.0)  # far from the 448 saturation point


def test_split_terms_are_each_finite_e4m3():
    v = _all_bf16_below(256.0)
    codes_hi = nx.e4m3_rn_sat(v)
    hi = nx.e4m3_decode(codes_hi)
    codes_lo = nx.e4m3_rn_sat((v - hi) * 16.0)
    assert not np.any((codes_hi & 0x7F) == 0x7F)
    assert not np.any((codes_lo & 0x7F) == 0x7F)
    # the residual carries at most 4 significant bits: |lo| <= 8 ulp(x') * 16 / 16
    assert np.all(np.abs(nx.e4m3_decode(codes_lo)) <= 16.0 * np.abs(v - hi) + 2.0 ** -10)


def test_row_exponent_rule_places_max_in_range():
    # e = 7 - floor(log2(amax)) puts max|x| * 2^e in [2^7, 2^8)
    rng = np.random.default_rng(13)
    amax = np.exp(rng.uniform(-80, 80, 2000))
    e = 7 - np.floor(np.log2(amax))
    scaled = amax * 2.0 ** e
    assert np.all((scaled >= 128.0) & (scaled < 256.0))
