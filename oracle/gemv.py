"""The hot-path operations, restated plainly in float64.

Test infrastructure (see the package docstring).  Every function takes and
returns raw bit patterns as numpy arrays: BF16 and F16 as uint16, E4M3 /
packed E2M1 / Q6_K / q8_1 as uint8, scales as float32.  Each dot product is
evaluated in float64 from exactly decoded operands and rounded once to BF16
at the end (``numerics.bf16_rn``); every elementwise product below is exact
in float64, so the only rounding before the final one is the float64
summation of the matmul.
"""

import numpy as np

from . import numerics as nx

# ----------------------------------------------------------------------------
# a1  FP8 E4M3 weight x BF16 rows (W8A16)
# ----------------------------------------------------------------------------


def w8a16_gemv(w, w_scale, x):
    """``out[m, n] = bf16_rn(s[n] * sum_k e4m3(W[n, k]) * x[m, k])``.

    lm_head_fp8_rows.rs, module doc and ``lm_head_fp8_run``: an FP8 E4M3 head
    with one float32 scale per output row (``Fp8Weight``,
    ``WeightQuantFormat::Fp8PerRow``) applied to BF16 hidden rows, BF16
    logits out.  w: uint8 [N, K]; w_scale: float32 [N]; x: uint16 [M, K].
    Returns uint16 [M, N].
    """
    W = nx.e4m3_decode(w)
    X = nx.bf16_decode(x)
    acc = X @ W.T
    return nx.bf16_rn(acc * np.asarray(w_scale, dtype=np.float32).astype(np.float64)[None, :])


# ----------------------------------------------------------------------------
# a2  per-row dynamic E4M3 activation quantize, a3 fused SiLU quantize
# ----------------------------------------------------------------------------


def w8a8_quantize_rows(x):
    """Per-row dynamic E4M3 quantize of BF16 rows.

    w8a8_layer.rs, ``W8a8Ctx::proj`` (quantized activations of up to
    ``W8A8_MAX_ROWS`` rows in the shared scratch) with the scale rule
    ``amax / 448``: per row, ``amax = max_k |x|``, ``sx = amax / 448`` as a
    float32 division, and ``q = e4m3_rn_sat(x / sx)`` with ``x / sx`` a
    float32 division.  A row whose ``sx`` is 0 gets all-zero codes.
    x: uint16 [M, K] -> (q uint8 [M, K], sx float32 [M]).
    """
    xv = nx.bf16_decode(x).astype(np.float32)          # exact
    amax = np.max(np.abs(xv), axis=1) if xv.shape[1] else np.zeros(xv.shape[0], np.float32)
    sx = (amax.astype(np.float32) / np.float32(448.0)).astype(np.float32)
    q = np.zeros(xv.shape, dtype=np.uint8)
    for m in range(xv.shape[0]):
        if sx[m] != 0:
            ratio = (xv[m] / sx[m]).astype(np.float32)    # float32 division, RN
            q[m] = nx.e4m3_rn_sat(ratio.astype(np.float64))
    return q, sx


def silu_exp_neg_f32(g):
    """``e^-g`` correctly rounded to float32, as float64 values.

    The float64 exp (error below one float64 ulp) is rounded once to float32; this is the
    correctly rounded float32 value unless e^-g lies within a float64 ulp of a float32
    rounding midpoint (``tests/test_oracle_pins.py`` checks every finite BF16 g against a
    60-digit evaluation).  Overflow gives inf, as in float32.
    """
    with np.errstate(over="ignore"):
        return nx.f32(np.exp(-np.asarray(g, dtype=np.float64)))


def silu_mul_bf16(gate, up):
    """``h = bf16_rn(silu(gate) * up)``, ``silu(g) = g / (1 + e^-g)``, in float32 steps.

    w8a8_layer.rs, ``W8a8Ctx::silu_proj`` (``ops::w8a8_act_quant_silu``): the down
    projection's input is ``bf16(silu(gate) * up)`` of BF16 gate and up rows, computed by
    the fused quantize kernel.  h decides the E4M3 codes, so it is evaluated in that
    kernel's float32: ``e = rn32(e^-g)`` (``silu_exp_neg_f32``), ``d = rn32(1 + e)``,
    ``s = rn32(g / d)``, ``p = rn32(s * u)``, then one round-to-nearest-even to BF16.
    Each float32 step is the float64 operation rounded once to float32, which equals the
    IEEE float32 operation (53 >= 2*24 + 2 bits: double rounding is innocuous for
    +, -, *, /).  Returns uint16.
    """
    g = nx.bf16_decode(gate)
    u = nx.bf16_decode(up)
    e = silu_exp_neg_f32(g)
    d = nx.f32(1.0 + e)
    with np.errstate(invalid="ignore"):
        s = nx.f32(g / d)
    return nx.bf16_rn(nx.f32(s * u))


def silu_quantize_rows(gate, up):
    """a3: the SiLU product of each row, quantized per row as in a2."""
    return w8a8_quantize_rows(silu_mul_bf16(gate, up))


# ----------------------------------------------------------------------------
# a4  W8A8 GEMV
# ----------------------------------------------------------------------------


def w8a8_gemv(w, w_scale, q, sx):
    """``out[m, n] = bf16_rn(s[n] * sx[m] * sum_k e4m3(W[n, k]) * e4m3(q[m, k]))``.

    lm_head_fp8_rows.rs, module doc and the W8A8 branch of
    ``lm_head_fp8_run``; w8a8_layer.rs, ``W8a8Ctx::proj``.
    w uint8 [N, K], w_scale float32 [N], q uint8 [M, K], sx float32 [M].
    """
    W = nx.e4m3_decode(w)
    Q = nx.e4m3_decode(q)
    acc = Q @ W.T
    s = np.asarray(w_scale, dtype=np.float32).astype(np.float64)
    t = np.asarray(sx, dtype=np.float32).astype(np.float64)
    return nx.bf16_rn(acc * s[None, :] * t[:, None])


def w8a8_proj(w, w_scale, x):
    """a2 then a4 on BF16 rows."""
    q, sx = w8a8_quantize_rows(x)
    return w8a8_gemv(w, w_scale, q, sx)


def w8a8_silu_proj(w, w_scale, gate, up):
    """a3 then a4."""
    q, sx = silu_quantize_rows(gate, up)
    return w8a8_gemv(w, w_scale, q, sx)


# ----------------------------------------------------------------------------
# a5  NVFP4 W4A16
# ----------------------------------------------------------------------------

NVFP4_BLOCK = 16


def nvfp4_dequant(w_packed, w_block_scale):
    """Decoded weight (float64 [N, K]) without the global factor.

    fp8_lut.rs, ``dequant_nvfp4_to_bf16`` / ``dequant_nvfp4_e8m0_to_bf16``:
    E2M1 codes two per byte, even index in the low nibble; one E4M3 scale per
    16 consecutive K elements of a row.
    """
    codes = nx.unpack_nibbles(w_packed)
    vals = nx.e2m1_decode(codes)
    S = nx.e4m3_decode(w_block_scale)
    return vals * np.repeat(S, NVFP4_BLOCK, axis=1)


def w4a16_gemv(w_packed, w_block_scale, global_scale, x):
    """``out[m, n] = bf16_rn(g * sum_b e4m3(S[n, b]) * sum_{k in b} e2m1(W[n, k]) * x[m, k])``.

    w4a16_gemv_tiers.rs (the W4A16 row tiers) over the NVFP4 layout of
    fp8_lut.rs; ``g`` is the folded float32 global multiplier.
    w_packed uint8 [N, K/2], w_block_scale uint8 [N, K/16], x uint16 [M, K].
    """
    Wd = nvfp4_dequant(w_packed, w_block_scale)
    X = nx.bf16_decode(x)
    acc = X @ Wd.T
    return nx.bf16_rn(acc * float(np.float32(global_scale)))


# ----------------------------------------------------------------------------
# NEXT 4  NVFP4 W4A4: FP4 activations for the wider row edge
# ----------------------------------------------------------------------------

NVFP4_ACT_GLOBAL_DIV = 2688.0   # 6 (largest E2M1) x 448 (largest E4M3)


def nvfp4_quantize_rows(x):
    """Per-row dynamic NVFP4 quantize of BF16 rows (the W4A4 activations).

    w4a16_gemv_tiers.rs, ``W4a16BatchmTiers`` (``a4_rows``, ``w4a4_proj``): a
    weight that declares FP4 activations runs its narrow projections W4A4 up
    to ``W4A4_MAX_M`` rows; the NVFP4 layout is fp8_lut.rs's (E2M1 pairs,
    even index in the low nibble, one E4M3 scale per 16 values, a float32
    global).  The pages do not print the quantize; this is the plain NVFP4
    recipe, every decision in float32 as the kernel takes it:
      g     = amax(row) / 2688                      (IEEE float32 division)
      s_b   = e4m3_rn_sat( amax(block b) / rn32(6 g) )
      S_b   = rn32( e4m3(s_b) * g )
      code  = e2m1_rn_sat( rn32(x / S_b) ),  0 where S_b == 0.
    Returns (codes packed uint8 [M, K/2], block scales uint8 [M, K/16],
    globals float32 [M]).  x: uint16 [M, K], K % 16 == 0.
    """
    X = nx.bf16_decode(x)
    M, K = X.shape
    if K % NVFP4_BLOCK:
        raise ValueError("K must be a multiple of 16")
    g = nx.f32(np.abs(X).max(axis=1) / NVFP4_ACT_GLOBAL_DIV) if K else np.zeros(M)
    B = np.abs(X).reshape(M, K // NVFP4_BLOCK, NVFP4_BLOCK).max(axis=2)
    d6 = nx.f32(6.0 * g)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        sf = np.where(d6 > 0, nx.f32(B / np.where(d6 > 0, d6, 1.0)), 0.0)
    s_code = nx.e4m3_rn_sat(sf)
    S = nx.f32(nx.e4m3_decode(s_code) * g[:, None])
    S_full = np.repeat(S, NVFP4_BLOCK, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(S_full > 0, nx.f32(X / np.where(S_full > 0, S_full, 1.0)), 0.0)
    codes = np.where(S_full > 0, nx.e2m1_rn_sat(q), 0).astype(np.uint8)
    return nx.pack_nibbles(codes), s_code, g.astype(np.float32)


def w4a4_gemv(w_packed, w_block_scale, global_scale, xq, x_block_scale, x_global):
    """``out[m, n] = bf16_rn(g_w * g_x[m] * sum_b e4m3(S[n, b]) e4m3(s[m, b]) sum_{k in b} e2m1(W) e2m1(X))``.

    The W4A4 projection (w4a16_gemv_tiers.rs, ``w4a4_proj``): both operands
    NVFP4, decoded exactly, the dot in float64, the two globals applied once,
    one BF16 rounding.  xq uint8 [M, K/2], x_block_scale uint8 [M, K/16],
    x_global float32 [M].
    """
    Wd = nvfp4_dequant(w_packed, w_block_scale)
    Xd = nvfp4_dequant(xq, x_block_scale)
    acc = Xd @ Wd.T
    gx = np.asarray(x_global, dtype=np.float32).astype(np.float64)[:, None]
    return nx.bf16_rn(acc * float(np.float32(global_scale)) * gx)


def w4a4_proj(w_packed, w_block_scale, global_scale, x):
    """BF16 rows -> nvfp4_quantize_rows -> w4a4_gemv."""
    q, s, g = nvfp4_quantize_rows(x)
    return w4a4_gemv(w_packed, w_block_scale, global_scale, q, s, g)


# ----------------------------------------------------------------------------
# NEXT 3  load-time FP4 dequant to BF16 (the step before the path)
# ----------------------------------------------------------------------------


def nvfp4_dequant_bf16(w_packed, w_block_scale, global_scale, is_reciprocal):
    """BF16 bits [N, K] of ``e2m1(W) * e4m3(S) * g``.

    fp8_lut.rs, ``dequant_nvfp4_to_bf16``: the stored global is folded into one
    float32 multiplier ``g`` (compressed-tensors: ``1 / global``, a zero global
    giving 0; ModelOpt: ``global``), and one BF16 value is written per weight.
    The kernel body is not printed; the reading is float32 arithmetic:
    ``e2m1 * e4m3`` is exact in float32 (at most 6 significant bits), its
    product with ``g`` is rounded once to float32, then to BF16 (nearest-even).
    w_packed uint8 [N, K/2], w_block_scale uint8 [N, K/16] -> uint16 [N, K].
    """
    g = float(nx.nvfp4_fold_global(global_scale, is_reciprocal))
    v = nvfp4_dequant(w_packed, w_block_scale)      # exact float64
    with np.errstate(over="ignore"):
        return nx.bf16_rn(nx.f32(v * g))


def e8m0_fp4_dequant_bf16(w_packed, scales, n, k):
    """BF16 bits [N, K] of ``e2m1(W) * e8m0(scale[group])``.

    fp8_lut.rs, ``dequant_nvfp4_e8m0_to_bf16``: two E2M1 values per byte (an
    even flat index is the low nibble), one E8M0 byte per group, the group size
    ``block = N*K / #scales`` over flat (row-major) indices, no global scale;
    ``f32_to_bf16(e2m1_table[code] * block_scale)``: a float32 product (exact
    unless it leaves the float32 range) rounded to BF16.  E8M0 codes 0 and 255
    decode to 0 (``FP8_E8M0_LUT``, pinned by ``tests/golden``).
    w_packed uint8 [N*K/2] (any shape), scales uint8 [#scales] -> uint16 [N, K].
    """
    total = n * k
    scales = np.asarray(scales, dtype=np.uint8).reshape(-1)
    if scales.size == 0 or total % scales.size != 0:
        raise ValueError("N*K must be a multiple of the number of E8M0 scales")
    block = total // scales.size
    codes = nx.unpack_nibbles(np.asarray(w_packed, dtype=np.uint8).reshape(-1))
    vals = nx.e2m1_decode(codes) * nx.E8M0_TABLE[np.repeat(scales, block)]
    with np.errstate(over="ignore"):
        return nx.bf16_rn(nx.f32(vals)).reshape(n, k)


# ----------------------------------------------------------------------------
# a6  block_q8_1 row quantize
# ----------------------------------------------------------------------------

Q8_1_BLOCK = 32
Q8_1_BYTES = 36


def q8_1_quantize_rows(x):
    """BF16 rows -> ``block_q8_1`` blocks of 32 values (36 bytes each).

    lm_head_q6k.rs, ``lm_head_q6k_run`` (``kquant_q8_1_rows_bf16`` quantises
    the hidden rows to ``block_q8_1``).  The block layout is not printed.
    Reading: ``{f16 d; f16 s; int8 qs[32]}``, little-endian; per block
    ``amax = max |x|``, ``d = amax / 127`` (float32 division), ``qs =
    round_half_away(x / d)`` (float32 division; all 0 when d is 0), ``d``
    stored round-to-nearest-even to f16, ``s = f16_rn(d * float(sum qs))``
    with the float32 d and a float32 product.
    x: uint16 [M, K] -> uint8 [M, K/32, 36].
    """
    xv = nx.bf16_decode(x).astype(np.float32)
    M, K = xv.shape
    nb = K // Q8_1_BLOCK
    out = np.zeros((M, nb, Q8_1_BYTES), dtype=np.uint8)
    for m in range(M):
        for b in range(nb):
            blk = xv[m, b * 32:(b + 1) * 32]
            amax = np.float32(np.max(np.abs(blk)))
            d = np.float32(amax / np.float32(127.0))
            if d == 0:
                qs = np.zeros(32, dtype=np.int64)
            else:
                r = (blk / d).astype(np.float32).astype(np.float64)
                qs = (np.sign(r) * np.floor(np.abs(r) + 0.5)).astype(np.int64)
            ssum = np.float32(np.float32(d) * np.float32(qs.sum()))
            d_bits = nx.f16_rn(np.float64(d))
            s_bits = nx.f16_rn(np.float64(ssum))
            out[m, b, 0:2] = np.frombuffer(np.uint16(d_bits).tobytes(), dtype=np.uint8)
            out[m, b, 2:4] = np.frombuffer(np.uint16(s_bits).tobytes(), dtype=np.uint8)
            out[m, b, 4:36] = qs.astype(np.int8).view(np.uint8)
    return out


def q8_1_fields(q8):
    """uint8 [M, K/32, 36] -> (d float64 [M, K/32], s float64 [M, K/32], qs int64 [M, K])."""
    q8 = np.ascontiguousarray(q8, dtype=np.uint8)
    M, nb, _ = q8.shape
    d = nx.f16_decode(q8[:, :, 0:2].copy().view(np.uint16)[..., 0])
    s = nx.f16_decode(q8[:, :, 2:4].copy().view(np.uint16)[..., 0])
    qs = q8[:, :, 4:36].copy().view(np.int8).astype(np.int64).reshape(M, nb * 32)
    return d, s, qs


# ----------------------------------------------------------------------------
# a7  Q6_K super-blocks x block_q8_1 rows
# ----------------------------------------------------------------------------

Q6K_VALUES = 256
Q6K_BYTES = 210


def q6k_unpack(blocks):
    """Q6_K super-blocks [..., 210] -> (q int64 [..., 256] in 0..63, sc int64 [..., 16], d float64 [...]).

    lm_head_q6k.rs, ``LmHeadQ6k``: 210-byte super-blocks of 256 values.  The
    byte map is not printed.  Reading (the public GGUF Q6_K layout): ``ql[128]``
    at 0, ``qh[64]`` at 128, ``int8 scales[16]`` at 192, ``f16 d`` at 208.
    For half h in {0, 1} and l in 0..31, element ``128h + 32t + l`` takes the
    low 4 bits from ``ql[64h + l]`` (t = 0: low nibble, t = 2: high nibble) or
    ``ql[64h + 32 + l]`` (t = 1: low nibble, t = 3: high nibble), and its top 2
    bits from bits 2t..2t+1 of ``qh[32h + l]``.  Element i uses ``scales[i // 16]``.
    The pages print no element order; it is pinned by hand-derived single-byte
    probes (tests/golden/q6k_single_byte_probes.txt) and by bit-exact agreement
    with the gguf library's independent Q6_K dequantizer on blocks covering every
    byte value of ql, qh and the scales (tests/test_oracle_pins.py).
    """
    b = np.asarray(blocks, dtype=np.uint8)
    ql = b[..., 0:128].astype(np.int64)
    qh = b[..., 128:192].astype(np.int64)
    sc = b[..., 192:208].view(np.int8).astype(np.int64)
    d = nx.f16_decode(b[..., 208:210].copy().view(np.uint16)[..., 0])
    q = np.empty(b.shape[:-1] + (Q6K_VALUES,), dtype=np.int64)
    for h in range(2):
        for t in range(4):
            src = ql[..., 64 * h + 32 * (t & 1): 64 * h + 32 * (t & 1) + 32]
            low = (src & 0xF) if t < 2 else (src >> 4)
            high = (qh[..., 32 * h: 32 * h + 32] >> (2 * t)) & 0x3
            q[..., 128 * h + 32 * t: 128 * h + 32 * t + 32] = low | (high << 4)
    return q, sc, d


def q6k_mmvq(blocks, q8):
    """``out[m, n] = bf16_rn(sum_sb sum_j d_w * sc_j * d_x(blk) * sum_{i in j} (q_i - 32) * qs_i)``.

    lm_head_q6k.rs, ``lm_head_q6k_run``: raw Q6_K blocks ``[vocab][hidden/256]``
    against ``block_q8_1`` rows, BF16 logits.  Sub-block j (16 values) lies in
    q8_1 block ``j // 2``; its integer dot is exact, then scaled by the f16
    super-block d, the int8 sub-scale and the stored f16 q8_1 d, in float64.
    blocks uint8 [N, K/256, 210]; q8 uint8 [M, K/32, 36] -> uint16 [M, N].
    """
    q, sc, dw = q6k_unpack(blocks)                 # [N, nsb, 256], [N, nsb, 16], [N, nsb]
    N, nsb, _ = q.shape
    K = nsb * Q6K_VALUES
    dx, _, qs = q8_1_fields(q8)                    # [M, K/32], [M, K]
    M = qs.shape[0]
    wq = (q - 32).reshape(N, K).astype(np.float64)
    wscale = (dw[:, :, None] * sc).reshape(N, K // 16)        # d_w * sc_j, exact
    xq = qs.astype(np.float64)
    acc = np.zeros((M, N), dtype=np.float64)
    for j in range(K // 16):
        isum = xq[:, 16 * j:16 * j + 16] @ wq[:, 16 * j:16 * j + 16].T   # exact integers
        acc += isum * wscale[None, :, j] * dx[:, j // 2][:, None]
    return nx.bf16_rn(acc)
