// Row-tile GEMV on warp MMAs: one weight pass for up to 8*NT activation rows.
//
// Work decomposition (one persistent 512-thread CTA per SM):
//   * the weight is cut into tiles of 16 consecutive rows x the full K; CTA c owns the
//     contiguous tile range [c*T/G, (c+1)*T/G), so the per-SM load differs by at most
//     one tile;
//   * a tile's K is split into 64-byte "k-blocks" of every row (64 FP8 or 128 FP4 values);
//     warp w of 16 owns k-blocks w, w+16, w+32, ... (summed in that order);
//   * inside a warp, lane (g = lane/4, t = lane%4) loads bytes [16t, 16t+16) of rows g and
//     g+8 of every k-block with one 128-bit streaming load each, through a register ring
//     that runs PF k-blocks ahead (across tile boundaries);
//   * the 16 bytes are decoded in registers into MMA A fragments; the activation rows sit
//     in shared memory in the matching fragment order, staged once per CTA;
//   * at the end of a tile the 16 warps' partial sums are added in warp order through
//     shared memory (fixed order, independent of the row count: every output row gets the
//     same bits whatever the number of rows in the call).
//
// K permutation: an MMA sums over its k index, so any bijection between physical k and
// the MMA's logical k is allowed as long as A and B use the same one.  Lane t feeds the
// MMA with its own 16 contiguous bytes, and the activation tile in shared memory stores,
// for each k-block, lane t's elements in the order its MMAs consume them.
#pragma once

#include "dlmh_common.cuh"

namespace dlmh {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kTileRows = 16;
constexpr int kKBlockBytes = 64;  // weight bytes of one row in one k-block

struct RowTileParams {
  const uint8_t* w;        // weight rows, row stride w_row_bytes
  int64_t w_row_bytes;     // bytes per weight row (k for FP8, k/2 for FP4)
  const float* w_scale;    // FP8: per-row float32 scale
  const uint8_t* w_bscale; // FP4: per-16 E4M3 block scales [n, k/16]
  float gscale;            // FP4: folded global multiplier
  int n, k;                // output rows, reduction length (elements)
  const void* x;           // activations (bf16 for A16, e4m3 codes for W8A8)
  int64_t ldx;             // elements
  const float* x_scale;    // W8A8: per-row activation scale; W4A4: per-row NVFP4 global
  const uint8_t* x_bscale; // W4A4: per-16 E4M3 activation block scales [rows, k/16]
  int rows;                // activation rows in this pass (<= 8*NT)
  uint16_t* out;           // bf16 out [rows, ldc]
  int64_t ldc;
  int early_w;             // streamed kernel: 1 when the preceding kernel on the stream is this
                           // library's activation pre-pass (writes neither weights nor outputs), so
                           // the weight ring may fill before that kernel completes
};

// ---------------------------------------------------------------------------------------
// formats
// ---------------------------------------------------------------------------------------

// FP8 E4M3 weight x BF16 activation: E4M3 -> f16 (exact), x -> f16 after a per-row power
// of two, f16 MMA with f32 accumulation.
struct FmtW8A16 {
  static constexpr int kElemsPerKB = 64;   // one byte per value
  static constexpr int kXBytes = 2;        // f16 activations in shared memory
  static constexpr int kXChunks = 2;       // 16-byte chunks of x per lane per k-block
  static constexpr bool kBlockScale = false;
};

// NVFP4: E2M1 x E4M3 block scale -> f16 (exact), f16 MMA.
struct FmtW4A16 {
  static constexpr int kElemsPerKB = 128;  // two values per byte
  static constexpr int kXBytes = 2;
  static constexpr int kXChunks = 4;
  static constexpr bool kBlockScale = true;
};

// NVFP4 weight x NVFP4 activations (W4A4): both operands E2M1 x E4M3 block scale -> f16
// (exact: at most 6 significant bits, range 2^-10 .. 2688), f16 MMA; the activation codes stay
// packed in registers (kXBytes == 0) and are decoded per MMA step.  Streamed kernel only.
struct FmtW4A4 {
  static constexpr int kElemsPerKB = 128;
  static constexpr int kXBytes = 0;
  static constexpr int kXChunks = 1;
  static constexpr bool kBlockScale = true;
};

// FP8 weight x FP8 activation codes: raw bytes into an E4M3 MMA, f32 accumulation.
struct FmtW8A8 {
  static constexpr int kElemsPerKB = 64;
  static constexpr int kXBytes = 1;
  static constexpr int kXChunks = 1;
  static constexpr bool kBlockScale = false;
};

template <class F>
struct XLayout {
  static constexpr int kKBBytes = F::kXChunks * 64;  // x bytes of one row per k-block
  // row stride in bytes with stride % 128 == 64: the two rows read by one quarter-warp
  // land on disjoint bank groups
  static __host__ __device__ int row_stride(int kb_total) {
    int s = kb_total * kKBBytes;
    int r = s % 128;
    return s + ((64 - r) + 128) % 128;
  }
};

template <class F>
__host__ __device__ inline int kblocks_of(int k) { return (k + F::kElemsPerKB - 1) / F::kElemsPerKB; }

// Reduction buffers: two (a tile's partials are written while the previous tile's are
// still being read) except for the 32-row tier, where one buffer and a second barrier
// leave room for a 5120-wide activation tile.
template <int NT>
__host__ __device__ constexpr int red_buffers() { return NT >= 4 ? 1 : 2; }

template <class F, int NT>
__host__ __device__ inline size_t rowtile_smem_bytes(int k) {
  const int mt = 8 * NT;
  size_t x = (size_t)mt * XLayout<F>::row_stride(kblocks_of<F>(k));
  size_t red = (size_t)red_buffers<NT>() * kWarps * kTileRows * mt * sizeof(float);
  size_t mul = 64 * sizeof(float);
  return x + red + mul;
}

// ---------------------------------------------------------------------------------------
// activation staging (once per CTA)
// ---------------------------------------------------------------------------------------

// A16: BF16 rows -> f16 * 2^e(row) in fragment order; rowmul[m] = 2^-e(row).
template <class F, int NT>
__device__ void stage_x_a16(const RowTileParams& p, uint8_t* xs, int rs, float* rowmul, int kb_total) {
  constexpr int MT = 8 * NT;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int rowexp[MT];
  const uint16_t* x = static_cast<const uint16_t*>(p.x);
  // 1. per-row max |x|
  for (int m = warp; m < MT; m += kWarps) {
    float amax = 0.f;
    if (m < p.rows) {
      const uint16_t* xr = x + (int64_t)m * p.ldx;
#pragma unroll 4
      for (int k8 = lane * 8; k8 < p.k; k8 += 32 * 8) {
        uint4 v = ldg_nc(xr + k8);
        uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          amax = fmaxf(amax, fabsf(bf16_bits_to_f32(wv[i] & 0xffffu)));
          amax = fmaxf(amax, fabsf(bf16_bits_to_f32(wv[i] >> 16)));
        }
      }
    }
    amax = warp_max(amax);
    if (lane == 0) {
      int e = f16_row_exponent(amax);
      rowexp[m] = e;
      rowmul[m] = __int_as_float((127 - e) << 23);  // 2^-e, exact
    }
  }
  __syncthreads();
  // 2. convert 8-element groups
  constexpr int EL = F::kElemsPerKB / 4;   // elements owned by one lane per k-block
  const int groups_per_row = kb_total * (F::kElemsPerKB / 8);
#pragma unroll 4
  for (int it = threadIdx.x; it < MT * groups_per_row; it += kThreads) {
    const int m = it / groups_per_row;
    const int g8 = it - m * groups_per_row;
    const int k0 = g8 * 8;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (m < p.rows && k0 < p.k) {
      const uint4 v = ldg_nc(x + (int64_t)m * p.ldx + k0);
      const float mul = __int_as_float((127 + rowexp[m]) << 23);  // 2^e
      uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      uint32_t ov[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t lo = f32_to_f16_bits(bf16_bits_to_f32(wv[i] & 0xffffu) * mul);
        uint32_t hi = f32_to_f16_bits(bf16_bits_to_f32(wv[i] >> 16) * mul);
        ov[i] = lo | (hi << 16);
      }
      o = make_uint4(ov[0], ov[1], ov[2], ov[3]);
    }
    const int kb = k0 / F::kElemsPerKB;
    const int e = k0 % F::kElemsPerKB;
    const int t = e / EL;
    const int q = (e % EL) / 8;
    const uint32_t off = m * rs + kb * XLayout<F>::kKBBytes + q * 64 + t * 16;
    sts128(smem_u32(xs + off), o);
  }
}

// W8A8: E4M3 code rows copied in fragment order; rowmul[m] = sx[m].
template <class F, int NT>
__device__ void stage_x_a8(const RowTileParams& p, uint8_t* xs, int rs, float* rowmul, int kb_total) {
  constexpr int MT = 8 * NT;
  const uint8_t* x = static_cast<const uint8_t*>(p.x);
  if (threadIdx.x < MT) rowmul[threadIdx.x] = threadIdx.x < p.rows ? p.x_scale[threadIdx.x] : 0.f;
  const int groups_per_row = kb_total * 4;   // 16-byte groups
#pragma unroll 4
  for (int it = threadIdx.x; it < MT * groups_per_row; it += kThreads) {
    const int m = it / groups_per_row;
    const int g16 = it - m * groups_per_row;
    const int k0 = g16 * 16;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (m < p.rows && k0 < p.k) o = ldg_nc(x + (int64_t)m * p.ldx + k0);
    const int kb = k0 / 64;
    const int t = (k0 % 64) / 16;
    sts128(smem_u32(xs + m * rs + kb * 64 + t * 16), o);
  }
}

// ---------------------------------------------------------------------------------------
// per-k-block MMA work
// ---------------------------------------------------------------------------------------

template <int NT>
__device__ __forceinline__ void kblock_w8a16(float (&acc)[NT][4], const uint4& ra, const uint4& rb,
                                             uint32_t xrow_saddr, int rs) {
  const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
  const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
  uint4 xc[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int q = 0; q < 2; ++q) xc[nt][q] = lds128(xrow_saddr + nt * 8 * rs + q * 64);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)(wa[j] & 0xffff));
    const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)(wa[j] >> 16));
    const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)(wb[j] & 0xffff));
    const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)(wb[j] >> 16));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const uint4& c = xc[nt][j >> 1];
      const uint32_t b0 = (j & 1) ? c.z : c.x;
      const uint32_t b1 = (j & 1) ? c.w : c.y;
      mma_f16_16816(acc[nt], a0, a1, a2, a3, b0, b1);
    }
  }
}

template <int NT>
__device__ __forceinline__ void kblock_w8a8(float (&acc)[NT][4], const uint4& ra, const uint4& rb,
                                            uint32_t xrow_saddr, int rs) {
  uint4 xc[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) xc[nt] = lds128(xrow_saddr + nt * 8 * rs);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mma_e4m3_16832(acc[nt], ra.x, rb.x, ra.y, rb.y, xc[nt].x, xc[nt].y);
    mma_e4m3_16832(acc[nt], ra.z, rb.z, ra.w, rb.w, xc[nt].z, xc[nt].w);
  }
}

// FP4: 16 bytes = 32 values per row; s2a/s2b = the two E4M3 block scales of rows g / g+8.
template <int NT>
__device__ __forceinline__ void kblock_w4a16(float (&acc)[NT][4], const uint4& ra, const uint4& rb, uint32_t s2a,
                                             uint32_t s2b, uint32_t xrow_saddr, int rs) {
  const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
  const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
  const uint32_t sa = e4m3x2_to_f16x2((uint16_t)s2a);  // (scale block 0, scale block 1) of row g
  const uint32_t sb = e4m3x2_to_f16x2((uint16_t)s2b);
  const uint32_t sa0 = __byte_perm(sa, 0, 0x1010), sa1 = __byte_perm(sa, 0, 0x3232);
  const uint32_t sb0 = __byte_perm(sb, 0, 0x1010), sb1 = __byte_perm(sb, 0, 0x3232);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 xc[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) xc[nt] = lds128(xrow_saddr + nt * 8 * rs + q * 64);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = 2 * q + h;                  // MMA step: bytes 2j, 2j+1 of the lane's 16
      const uint32_t word_a = wa[j >> 1], word_b = wb[j >> 1];
      const int sh = (j & 1) * 16;
      const uint32_t ssa = (j < 4) ? sa0 : sa1;
      const uint32_t ssb = (j < 4) ? sb0 : sb1;
      const uint32_t a0 = hmul2(e2m1x2_to_f16x2((word_a >> sh) & 0xff), ssa);
      const uint32_t a2 = hmul2(e2m1x2_to_f16x2((word_a >> (sh + 8)) & 0xff), ssa);
      const uint32_t a1 = hmul2(e2m1x2_to_f16x2((word_b >> sh) & 0xff), ssb);
      const uint32_t a3 = hmul2(e2m1x2_to_f16x2((word_b >> (sh + 8)) & 0xff), ssb);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t b0 = h ? xc[nt].z : xc[nt].x;
        const uint32_t b1 = h ? xc[nt].w : xc[nt].y;
        mma_f16_16816(acc[nt], a0, a1, a2, a3, b0, b1);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------

template <class F, int NT, int PF>
__global__ void __launch_bounds__(kThreads, 1) rowtile_gemv_kernel(const RowTileParams p) {
  constexpr int MT = 8 * NT;
  extern __shared__ __align__(128) uint8_t smem[];
  const int kb_total = kblocks_of<F>(p.k);
  const int rs = XLayout<F>::row_stride(kb_total);
  uint8_t* xs = smem;
  float* red = reinterpret_cast<float*>(smem + (size_t)MT * rs);
  float* rowmul = red + red_buffers<NT>() * kWarps * kTileRows * MT;

  const int ntiles = (p.n + kTileRows - 1) / kTileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  if (T0 >= T1) return;  // uniform over the CTA

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nkb = (kb_total + kWarps - 1) / kWarps;          // k-blocks per warp (uniform)
  // Warp w owns k-blocks w, w + 16, w + 32, ... in that order: the same split, and so the
  // same summation order, as the streamed kernel (rowtile_tma.cuh), so that every tier of
  // every kernel gives a row the same bits.
  const int nvalid = max(0, min(nkb, (kb_total - warp + kWarps - 1) / kWarps));
  const int64_t wrb = p.w_row_bytes;
  const int lane_col = warp * kKBlockBytes + 16 * t;          // byte column of the lane's first slot
  constexpr int kSlotBytes = kWarps * kKBlockBytes;           // column step between a warp's slots
  // bit j: slot j is inside K for this warp and the lane's 16 bytes lie inside the row
  uint32_t colmask = 0;
  for (int j = 0; j < nvalid; ++j)
    if (lane_col + j * kSlotBytes < wrb) colmask |= 1u << j;
  const int nfull = p.n / kTileRows;  // tiles whose 16 rows all exist

  // ---- load side of the ring: running pointers, no per-load index arithmetic
  const int64_t row8 = 8 * wrb;
  const int64_t tile_jump = kTileRows * wrb - (int64_t)nkb * kSlotBytes;
  const uint8_t* lp = p.w + ((int64_t)T0 * kTileRows + g) * wrb + lane_col;
  const int64_t srb = p.k / 16;  // FP4: block-scale bytes per row; a lane takes 2 per k-block
  const int64_t s_row8 = 8 * srb;
  const int64_t s_tile_jump = kTileRows * srb - (int64_t)nkb * kWarps * 8;
  const uint8_t* sp = nullptr;
  if constexpr (F::kBlockScale) sp = p.w_bscale + ((int64_t)T0 * kTileRows + g) * srb + warp * 8 + 2 * t;
  int ltile = T0, lkb = 0;
  auto issue = [&](uint4& ra, uint4& rb, uint32_t& sa, uint32_t& sb) {
    ra = make_uint4(0, 0, 0, 0);
    rb = ra;
    sa = sb = 0;
    if (ltile < T1 && ((colmask >> lkb) & 1u)) {
      const bool full = ltile < nfull;
      const int r = ltile * kTileRows + g;
      if (full || r < p.n) {
        ra = ldg_stream(lp);
        if constexpr (F::kBlockScale) sa = ldg_u16(sp);
      }
      if (full || r + 8 < p.n) {
        rb = ldg_stream(lp + row8);
        if constexpr (F::kBlockScale) sb = ldg_u16(sp + s_row8);
      }
    }
    lp += kSlotBytes;
    if constexpr (F::kBlockScale) sp += kWarps * 8;
    if (++lkb == nkb) {
      lkb = 0;
      ++ltile;
      lp += tile_jump;
      if constexpr (F::kBlockScale) sp += s_tile_jump;
    }
  };

  uint4 bufa[PF], bufb[PF];
  uint32_t bsa[PF], bsb[PF];
#pragma unroll
  for (int s = 0; s < PF; ++s) issue(bufa[s], bufb[s], bsa[s], bsb[s]);

  // Stage the activation rows while the first PF k-blocks of weight are in flight.
  if constexpr (F::kXBytes == 2)
    stage_x_a16<F, NT>(p, xs, rs, rowmul, kb_total);
  else
    stage_x_a8<F, NT>(p, xs, rs, rowmul, kb_total);
  __syncthreads();

  // The reducing threads (one output each per tile) hold the row scale of their output
  // for the current tile and fetch the next tile's one tile ahead, off the critical path.
  const int red_rr = threadIdx.x % kTileRows, red_cc = threadIdx.x / kTileRows;
  const bool reducer = threadIdx.x < kTileRows * MT;
  float wscale_cur = 0.f;
  if constexpr (!F::kBlockScale) {
    const int row = T0 * kTileRows + red_rr;
    if (reducer && row < p.n) wscale_cur = p.w_scale[row];
  }

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.f;

  const uint32_t xs_lane = smem_u32(xs) + g * rs + t * 16 + warp * XLayout<F>::kKBBytes;
  uint32_t xa = xs_lane;
  int tile = T0, kb = 0, parity = 0;

  while (tile < T1) {
#pragma unroll
    for (int s = 0; s < PF; ++s) {
      if (tile < T1) {
        const uint4 ra = bufa[s], rb = bufb[s];
        const uint32_t sa = bsa[s], sb = bsb[s];
        issue(bufa[s], bufb[s], bsa[s], bsb[s]);
        if (kb < nvalid) {
          if constexpr (F::kBlockScale)
            kblock_w4a16<NT>(acc, ra, rb, sa, sb, xa, rs);
          else if constexpr (F::kXBytes == 1)
            kblock_w8a8<NT>(acc, ra, rb, xa, rs);
          else
            kblock_w8a16<NT>(acc, ra, rb, xa, rs);
        }
        xa += kWarps * XLayout<F>::kKBBytes;
        if (++kb == nkb) {
          // ---- end of tile: fixed-order cross-warp reduction
          float* rb_ = red + parity * (kWarps * kTileRows * MT);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float4 v = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
            reinterpret_cast<float4*>(rb_)[(warp * NT + nt) * 32 + lane] = v;
            acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
          }
          __syncthreads();
          if (reducer) {
            const int rr = red_rr, cc = red_cc;
            const int row = tile * kTileRows + rr;
            float wsc = 0.f;
            if constexpr (!F::kBlockScale) {
              wsc = wscale_cur;
              const int nrow = row + kTileRows;
              if (tile + 1 < T1 && nrow < p.n) wscale_cur = p.w_scale[nrow];
            }
            if (cc < p.rows && row < p.n) {
              const int gg = rr & 7, up = rr >> 3;
              const int nt = cc >> 3, cl = cc & 7;
              const int ln = gg * 4 + (cl >> 1), comp = up * 2 + (cl & 1);
              float sum = 0.f;
#pragma unroll
              for (int ww = 0; ww < kWarps; ++ww) sum += rb_[((ww * NT + nt) * 32 + ln) * 4 + comp];
              // weight-side scale first: sum * 2^-e alone can leave the f32 range for
              // rows with |x| near the BF16 limits, sum * s cannot
              float y;
              if constexpr (F::kBlockScale)
                y = (sum * p.gscale) * rowmul[cc];
              else
                y = (sum * wsc) * rowmul[cc];
              p.out[(int64_t)cc * p.ldc + row] = f32_to_bf16_bits(y);
            }
          }
          if constexpr (red_buffers<NT>() == 1) __syncthreads();
          else parity ^= 1;
          kb = 0;
          xa = xs_lane;
          ++tile;
        }
      }
    }
  }
}

}  // namespace dlmh
