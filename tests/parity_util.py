"""Shared helpers of the GPU parity tests (comparison rules, no arithmetic of the method)."""

import numpy as np

from oracle import numerics as nx

TOL_REL = 2.0 ** -7
TOL_RMS = 1e-3


def bf16_tolerance_report(got_bits, ref_bits):
    """Elements outside |err| <= 2^-7 |ref| + 1e-3 rms(ref), rms over the whole call output."""
    got = nx.bf16_decode(np.asarray(got_bits))
    ref = nx.bf16_decode(np.asarray(ref_bits))
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(got - ref)
    tol = TOL_REL * np.abs(ref) + TOL_RMS * rms
    bad = ~(err <= tol)
    return bad, err, tol, rms


def assert_bf16_close(got_bits, ref_bits, what="", rms_ref_bits=None):
    bad, err, tol, rms = bf16_tolerance_report(got_bits, ref_bits)
    if rms_ref_bits is not None:  # sampled outputs: use the rms of a larger reference sample
        ref = nx.bf16_decode(np.asarray(ref_bits))
        rr = nx.bf16_decode(np.asarray(rms_ref_bits))
        rms = float(np.sqrt(np.mean(rr * rr)))
        tol = TOL_REL * np.abs(ref) + TOL_RMS * rms
        bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        got = nx.bf16_decode(np.asarray(got_bits))
        ref = nx.bf16_decode(np.asarray(ref_bits))
        detail = ", ".join(f"{tuple(i)}: got {got[tuple(i)]!r} ref {ref[tuple(i)]!r}" for i in idx)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outputs outside tolerance "
                             f"(rms(ref)={rms:.4g}); first: {detail}")
