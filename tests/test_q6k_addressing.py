"""Host restatement of the streamed 8-row Q6_K kernel's shared-memory addressing.

The kernel (q6k_rows8_kernel<true, true, *>) reads each 210-byte super-block of a staged weight
row with 32-bit shared loads: single loads when every lane's super-block is 4-byte aligned,
otherwise from one aligned base and a funnel shift (a row with an odd super-block count puts
both alignments in one warp).  This test re-derives, for the shapes the tests and the bench use, the host's stage choice (rows
per stage, ring depth, lane row map, slot padding) and every shared read the lanes make, and
checks that each is aligned to its width and lies inside its super-block (two bytes before it
at most, for the 2-mod-4 case), and that the ring fits the shared memory.  It also shows that
the scale load an earlier version used (five words from 2 bytes before the scales, whatever the
lane's alignment) is misaligned at k = 1280, and restates the activation tables' layout of the
8-row kernels and the wide kernel's regrouped activation stage.
"""

import pytest

SMS, OPTIN = 148, 232448
RED = 2 * 16 * 32 * 4 * 4


def _rup(x, m):
    return (x + m - 1) // m * m


def _slice_begin(nsb, w):
    q, r = divmod(nsb, 16)
    return w * q + min(w, r)


def _rows(row_pair, g):
    """Tile rows of MMA rows g and g + 8 of lane (g, t)."""
    return (2 * g, 2 * g + 1) if row_pair else (g, g + 8)


def _bank_cost(row_bytes, sr, stride, row_pair):
    cost = 0
    for odd in (0, 1):
        for half in (0, 1):
            banks = {}
            for g in range(8):
                lr = _rows(row_pair, g)[half]
                off = (lr // sr) * stride + (lr % sr) * row_bytes + 210 * odd
                for t in range(4):
                    w = (off >> 2) + t
                    banks.setdefault(w & 31, set()).add(w)
            cost += max(len(v) for v in banks.values())
    return cost


def _bank_layout(row_bytes, sr):
    base, best = _rup(sr * row_bytes, 128), None
    for rp in (0, 1):
        for pad in range(0, 128, 16):
            c = _bank_cost(row_bytes, sr, base + pad, rp)
            if best is None or c < best[0]:
                best = (c, rp, pad)
    return best[1], best[2]


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
            row_pair, pad = _bank_layout(nsb * 210, sr)
            stride = _rup(sr * nsb * 210, 128) + pad
            spt = 16 // sr
            ns = min((limit - ring_off) // stride if limit > ring_off else 0, 2 * spt, 16)
            if ns / spt > best_t + 1e-9:
                best, best_t = (ns, sr, stride, row_pair), ns / spt
    return ring_off, best


def _scale_reads(a):
    """The scales and d of a 4-byte aligned super-block at a."""
    return [(a + 192 + 4 * q, 4) for q in range(4)] + [(a + 208, 2)]


def _reads(a, t, aligned, old_scales=False):
    if aligned:
        r = [(a + 4 * t + 16 * q, 4) for q in range(8)] + [(a + 4 * t + 128 + 16 * q, 4) for q in range(4)]
        return r + _scale_reads(a)
    else:
        b, sh = a & ~3, (a & 3) * 8
        r = []
        for q in range(8):
            r += [(b + 4 * t + 16 * q, 4), (b + 4 * t + 16 * q + 4, 4)]
        for q in range(4):
            r += [(b + 4 * t + 128 + 16 * q, 4), (b + 4 * t + 128 + 16 * q + 4, 4)]
        if old_scales:
            return r + [(a + 190 + 4 * q, 4) for q in range(5)] + [(a + 208, 2)]
        # the five words from b + 192 (the fifth only when sh != 0, else the fourth again)
        r += [(b + 192 + 4 * q, 4) for q in range(4)] + [(b + (208 if sh else 204), 4)]
        return r + [(a + 208, 2)]


def _check(n, k, old_scales=False):
    nsb, row_bytes = k // 256, (k // 256) * 210
    ring_off, best = _config(k)
    assert best is not None, "streamed kernel expected"
    ns, sr, stride, row_pair = best
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
                        lra, lrb = _rows(row_pair, g)
                        sa, sbb = spt * i + lra // sr, spt * i + lrb // sr
                        ba = ring_off + (sa % ns) * stride + (lra % sr) * row_bytes + 210 * sb
                        bb = ring_off + (sbb % ns) * stride + (lrb % sr) * row_bytes + 210 * sb
                        lanes.append((ba, tile * 16 + lra < n, t))
                        lanes.append((bb, tile * 16 + lrb < n, t))
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


def test_bank_layout_at_k7168_is_conflict_free():
    # rows 5880 bytes apart: the plain map has 2-way conflicts on every fragment load, rows 2g
    # and 2g + 1 with 64 bytes of slot padding none (one distinct word per bank per load)
    assert _bank_cost(5880, 8, _rup(8 * 5880, 128), 0) == 8
    assert _bank_layout(5880, 8) == (1, 64)
    assert _bank_cost(5880, 8, _rup(8 * 5880, 128) + 64, 1) == 4


@pytest.mark.parametrize("k", [512, 1280, 7168, 8192])
def test_activation_tables_read_back_what_was_staged(k):
    # staging: d of (block b, column m) at dxs[(b >> 1) * 16 + (m >> 1) * 4 + (b & 1) * 2 + (m & 1)],
    # the correction of (sub-block 2b + e, column m) at cor[b * 16 + (m >> 1) * 4 + e * 2 + (m & 1)];
    # lane t reads 16 bytes at dxs + 16 t + 256 sb + 64 (blk >> 1) and cor + 16 t + 512 sb + 64 blk
    nb32 = k // 32
    dxs, cor = {}, {}
    for b in range(nb32):
        for m in range(8):
            o = (b >> 1) * 16 + (m >> 1) * 4 + (b & 1) * 2 + (m & 1)
            assert o not in dxs and 0 <= o < nb32 * 8
            dxs[o] = (b, m)
            for e in range(2):
                o = b * 16 + (m >> 1) * 4 + e * 2 + (m & 1)
                assert o not in cor and 0 <= o < nb32 * 16
                cor[o] = (2 * b + e, m)
    for sb in range(k // 256):
        for blk in range(8):
            for t in range(4):
                a = (16 * t + 256 * sb + 64 * (blk >> 1)) // 4
                got = [dxs[a + c] for c in range(4)]
                b = 8 * sb + blk
                # components x, y: even block; z, w: odd block; columns 2t, 2t + 1
                assert got[2 * (blk & 1)] == (b, 2 * t) and got[2 * (blk & 1) + 1] == (b, 2 * t + 1)
                a = (16 * t + 512 * sb + 64 * blk) // 4
                got = [cor[a + c] for c in range(4)]
                j0 = 16 * sb + 2 * blk
                assert got == [(j0, 2 * t), (j0, 2 * t + 1), (j0 + 1, 2 * t), (j0 + 1, 2 * t + 1)]


@pytest.mark.parametrize("nt,rows", [(2, 9), (2, 16), (4, 17), (4, 32), (8, 33), (8, 64)])
def test_wide_activation_stage_reads_back_what_was_copied(nt, rows):
    # the wide kernel's producer copies code word w (bytes 4w..4w+3 of a block's 32 codes) of
    # block b of row m to word (((b NT + m / 8) 8 + m % 8) 4 + w % 4) 2 + w / 4 of the stage,
    # and the (d, s) word of block b of row m to word ((b NT + m / 8) 4 + (m % 8) / 2) 2 + m % 2
    # after 8 NT 32 8 bytes of codes; lane (g, t) of column group ct reads 8 bytes at
    # (((blk NT + ct) 8 + g) 4 + t) 8 (its B words of sub-blocks 2 blk, 2 blk + 1) and at
    # codes_bytes + ((blk NT + ct) 4 + t) 8 (the d of columns 2t, 2t + 1)
    codes_words = 8 * nt * 32 * 8 // 4
    stage = {}
    for m in range(rows):
        for b in range(8):
            for w in range(8):
                o = (((b * nt + (m >> 3)) * 8 + (m & 7)) * 4 + (w & 3)) * 2 + (w >> 2)
                assert o not in stage and 0 <= o < codes_words
                stage[o] = ("code", m, b, w)
            o = codes_words + ((b * nt + (m >> 3)) * 4 + ((m & 7) >> 1)) * 2 + (m & 1)
            assert o not in stage and o < codes_words + 256 * nt // 4
            stage[o] = ("ds", m, b)
    for blk in range(8):
        for ct in range(nt):
            for g in range(8):
                for t in range(4):
                    m = 8 * ct + g
                    a = ((((blk * nt + ct) * 8 + g) * 4 + t) * 8) // 4
                    want = [("code", m, blk, t), ("code", m, blk, 4 + t)] if m < rows else [None, None]
                    assert [stage.get(a), stage.get(a + 1)] == want  # padding rows read the zeroed stage
                    a = codes_words + (((blk * nt + ct) * 4 + t) * 8) // 4
                    want = [("ds", c, blk) if c < rows else None for c in (8 * ct + 2 * t, 8 * ct + 2 * t + 1)]
                    assert [stage.get(a), stage.get(a + 1)] == want
