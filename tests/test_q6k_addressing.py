"""Host restatement of the streamed 8-row Q6_K kernel's shared-memory addressing.

The kernel (q6k_rows8_kernel<true, true>) reads each 210-byte super-block of a staged weight
row with 32-bit shared loads: single loads when every lane's super-block is 4-byte aligned,
otherwise from one aligned base and a funnel shift (a row with an odd super-block count puts
both alignments in one warp).  This test re-derives, for the shapes the tests and the bench
use, the host's stage choice (rows per stage, ring depth) and every shared read the lanes make,
and checks that each is aligned to its width and lies inside its super-block (two bytes before
it at most, for the 2-mod-4 case), and that the ring fits the shared memory.  It also shows that
the scale load an earlier version used (five words from 2 bytes before the scales, whatever the
lane's alignment) is misaligned at k = 1280.
"""

import pytest

SMS, OPTIN = 148, 232448
RED = 2 * 16 * 32 * 4 * 4


def _rup(x, m):
    return (x + m - 1) // m * m


def _slice_begin(nsb, w):
    q, r = divmod(nsb, 16)
    return w * q + min(w, r)


def _config(k):
    nsb = k // 256
    reg = (nsb + 15) // 16 <= 2
    base = (k // 32) * 8 * 4 + (k // 16) * 8 * 4 + RED
    ring_off = _rup(base, 128)
    limit = OPTIN - 2048
    best, best_t = None, 1.0
    if reg:
        for sr in (8, 4):
            if (sr * nsb * 210) % 16:
                continue
            stride = _rup(sr * nsb * 210, 128)
            spt = 16 // sr
            ns = min((limit - ring_off) // stride if limit > ring_off else 0, 2 * spt, 16)
            if ns / spt > best_t + 1e-9:
                best, best_t = (ns, sr, stride), ns / spt
    return ring_off, best


def _reads(a, t, aligned, old_scales=False):
    if aligned:
        r = [(a + 4 * t + 16 * q, 4) for q in range(8)] + [(a + 4 * t + 128 + 16 * q, 4) for q in range(4)]
        r += [(a + 192 + 4 * q, 4) for q in range(4)]
    else:
        b, sh = a & ~3, (a & 3) * 8
        r = []
        for q in range(8):
            r += [(b + 4 * t + 16 * q, 4), (b + 4 * t + 16 * q + 4, 4)]
        for q in range(4):
            r += [(b + 4 * t + 128 + 16 * q, 4), (b + 4 * t + 128 + 16 * q + 4, 4)]
        if old_scales:
            r += [(a + 190 + 4 * q, 4) for q in range(5)]
        else:
            r += [(b + 192 + 4 * q, 4) for q in range(4)] + [(b + (208 if sh else 204), 4)]
    return r + [(a + 208, 2)]


def _check(n, k, old_scales=False):
    nsb, row_bytes = k // 256, (k // 256) * 210
    ring_off, best = _config(k)
    assert best is not None, "streamed kernel expected"
    ns, sr, stride = best
    spt = 16 // sr
    assert ring_off + ns * stride + 256 <= OPTIN
    ntiles = (n + 15) // 16
    grid = min(ntiles, SMS)
    bad = 0
    for b in (0, grid // 2, grid - 1):
        t0, t1 = b * ntiles // grid, (b + 1) * ntiles // grid
        for i in range(min(t1 - t0, 3)):
            tile = t0 + i
            for w in range(16):
                for sb in range(_slice_begin(nsb, w), _slice_begin(nsb, w + 1)):
                    lanes = []
                    for lane in range(32):
                        g, t = lane >> 2, lane & 3
                        sa, sbb = spt * i + g // sr, spt * i + (g + 8) // sr
                        ba = ring_off + (sa % ns) * stride + (g % sr) * row_bytes + 210 * sb
                        bb = ring_off + (sbb % ns) * stride + ((g + 8) % sr) * row_bytes + 210 * sb
                        lanes.append((ba, tile * 16 + g < n, t))
                        lanes.append((bb, tile * 16 + g + 8 < n, t))
                    aligned = all(a % 4 == 0 for a, _, _ in lanes)
                    for a, valid, t in lanes:
                        if not valid:
                            continue
                        for addr, width in _reads(a, t, aligned, old_scales):
                            bad += addr % width != 0
                            assert a - 2 <= addr and addr + width <= a + 210
    return bad


@pytest.mark.parametrize("n,k", [(1000, 7168), (45, 1280), (1000, 8192), (129280, 7168), (15, 256), (256, 1024)])
def test_streamed_q6k_reads_are_aligned_and_inside_their_super_block(n, k):
    assert _check(n, k) == 0


def test_the_earlier_scale_load_is_caught():
    assert _check(45, 1280, old_scales=True) > 0
    assert _check(1000, 7168, old_scales=True) == 0  # even super-block counts never mix alignments
