// Q6_K super-blocks x block_q8_1 rows on int8 warp MMAs.
//
// Per 16-value sub-block j one m16n8k16 integer MMA gives the exact int32 dot
//   D_j = sum_{i in j} (q_i - 32) * qs_i
// for 16 weight rows x 8 activation columns.  Per q8_1 block (sub-blocks 2b, 2b+1) the two
// dots are weighted by their int8 sub-scales in int32 (exact: |sum| < 2^24, so its float
// conversion is exact too) and accumulated in float over the super-block's 8 blocks with the
// block's q8_1 d:  t = fma(float(D_2b sc_2b + D_2b+1 sc_2b+1), d8(b), t)  from t = 0; the
// super-block then adds  acc = fma(t, d(super-block), acc).  The super-blocks of a row are cut
// into 16 K-slices (q6k_slices.h); each slice is accumulated alone from 0 and the slices are
// added in order.  Every kernel below takes exactly these steps for every output, so a row's
// bits do not depend on which kernel, or how many rows, served it.
//
// Two exact ways to the same D_j:
//   - 8-row kernels: the MMA multiplies the unsigned codes q (u8 x s8) and its accumulator
//     starts at -32 * sum_{i in j} qs_i, from a table built once per CTA;
//   - wide kernel (several 8-column groups share one weight fragment): the codes are turned
//     into (q - 32) as signed bytes once (bit tricks, no table) and every MMA starts from 0.
//
// Super-block byte map (210 bytes): ql[128] @0, qh[64] @128, int8 scales[16] @192, f16 d @208.
// Value i = 128h + 32u + l (h < 2, u < 4, l < 32): low 4 bits from ql[64h + 32(u&1) + l] (low
// nibble for u < 2, high for u >= 2), top 2 bits from bits 2u..2u+1 of qh[32h + l]; sub-block
// j = i / 16 uses scales[j].  Lane (g, t) feeds the MMA with values 4t..4t+3 of every sub-block,
// i.e. the 4 consecutive ql / qh bytes at l = 16(j&1) + 4t, for the weight rows of MMA rows g
// and g + 8 (tile rows g and g + 8, or 2g and 2g + 1: see the 8-row kernels).
#include "dlmh_common.cuh"
#include "gemv_launch.h"
#include "q6k_slices.h"
#include "umma_common.cuh"

namespace dlmh {
namespace {

constexpr int kQ6Warps = 16;
constexpr int kQ6Threads = kQ6Warps * 32;
constexpr int kQ6TileRows = 16;
constexpr int kQ6MaxRows = 8;  // q8_1 rows of the 8-row kernels (one 8-column MMA tile)

static_assert(kQ6Warps == kQ6Slices, "one K-slice per warp of the 8-row kernels");

// ---------------------------------------------------------------------------------------
// The shared arithmetic
// ---------------------------------------------------------------------------------------

// One weight row's super-block as lane (g, t) needs it: ql bytes 16i + 4t (i < 8), qh bytes
// 128 + 16i + 4t (i < 4), the 16 scale bytes, and d.
struct Q6W {
  uint32_t ql[8], qh[4], sc[4];
  float d;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// The four 6-bit codes q (one per byte, 0..63) of sub-block j, values 4t..4t+3.
__device__ __forceinline__ uint32_t q6_codes_u8(const Q6W& w, int j) {
  const int h = j >> 3, u = (j & 7) >> 1, e = j & 1;
  const uint32_t qlw = w.ql[4 * h + 2 * (u & 1) + e];
  const uint32_t qhw = w.qh[2 * h + e];
  const uint32_t lo = u >= 2 ? qlw >> 4 : qlw;
  const uint32_t hi = u == 0 ? qhw << 4 : u == 1 ? qhw << 2 : u == 2 ? qhw : qhw >> 2;
  return (lo & 0x0f0f0f0fu) | (hi & 0x30303030u);
}

// The same codes as (q - 32) in signed bytes: flipping bit 5 gives the 6-bit two's complement,
// then bit 5 is copied into bits 6 and 7 (adding 6 * 0x20 sets them; they are 0, so no carry).
__device__ __forceinline__ uint32_t q6_codes_s8(const Q6W& w, int j) {
  const uint32_t a = q6_codes_u8(w, j) ^ 0x20202020u;
  return a + (a & 0x20202020u) * 6u;
}

// Sub-scale j of the row, sign-extended (prmt: byte j&3, its sign replicated into the others).
__device__ __forceinline__ int q6_scale(const Q6W& w, int j) {
  const uint32_t q = (uint32_t)(j & 3);
  return (int)prmt(w.sc[j >> 2], 0u, q | ((8u | q) << 4) | ((8u | q) << 8) | ((8u | q) << 12));
}

// D = A (u8) x B (s8) + C, C given as two values per row pair (columns 2t, 2t+1).
__device__ __forceinline__ void mma_u8s8_c(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0, int c0, int c1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%8,%7,%8};"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(a0), "r"(a1), "r"(b0), "r"(c0), "r"(c1));
}
// D = A (s8) x B (s8), accumulator from zero (one zero register for all of C).
__device__ __forceinline__ void mma_s8s8_z(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(a0), "r"(a1), "r"(b0), "r"(0));
}

// One q8_1 block of one 8-column group: t[i] += float(D0[i] sc0 + D1[i] sc1) * d8(column).
// Outputs i: 0 = (row g, column 2t), 1 = (g, 2t+1), 2 = (g+8, 2t), 3 = (g+8, 2t+1).
// kCol0: only column 0 is live (one activation row), the odd columns are left alone.
template <bool kCol0 = false>
__device__ __forceinline__ void q6_block_step(float (&tsb)[4], const int (&d0)[4], const int (&d1)[4], int ra0, int ra1,
                                              int rb0, int rb1, float dx0, float dx1) {
  tsb[0] = __fmaf_rn((float)(d0[0] * ra0 + d1[0] * ra1), dx0, tsb[0]);
  if (!kCol0) tsb[1] = __fmaf_rn((float)(d0[1] * ra0 + d1[1] * ra1), dx1, tsb[1]);
  tsb[2] = __fmaf_rn((float)(d0[2] * rb0 + d1[2] * rb1), dx0, tsb[2]);
  if (!kCol0) tsb[3] = __fmaf_rn((float)(d0[3] * rb0 + d1[3] * rb1), dx1, tsb[3]);
}

// End of a super-block: acc += t * d(row).
template <bool kCol0 = false>
__device__ __forceinline__ void q6_superblock_end(float (&acc)[4], const float (&tsb)[4], float da, float db) {
  acc[0] = __fmaf_rn(tsb[0], da, acc[0]);
  if (!kCol0) acc[1] = __fmaf_rn(tsb[1], da, acc[1]);
  acc[2] = __fmaf_rn(tsb[2], db, acc[2]);
  if (!kCol0) acc[3] = __fmaf_rn(tsb[3], db, acc[3]);
}

// ---- weight fragment loads

__device__ __forceinline__ uint32_t lds_u32(uint32_t saddr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(saddr));
  return v;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t saddr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(saddr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t saddr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(saddr));
  return v;
}

// Super-block at shared address `ba`: kAligned only when ba is 4-byte aligned; the other path
// takes any even ba (the lanes of one warp may mix both alignments when a row holds an odd
// number of super-blocks).  It reads the aligned words that cover each field, all inside
// [ba - 2, ba + 210).
template <bool kAligned>
__device__ __forceinline__ void q6_load_smem(Q6W& w, bool valid, uint32_t ba, int t) {
  if (!valid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) w.ql[i] = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) w.qh[i] = w.sc[i] = 0u;
    w.d = 0.f;
    return;
  }
  if (kAligned) {
    const uint32_t a = ba + 4 * t;
#pragma unroll
    for (int i = 0; i < 8; ++i) w.ql[i] = lds_u32(a + 16 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) w.qh[i] = lds_u32(a + 128 + 16 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) w.sc[i] = lds_u32(ba + 192 + 4 * i);
  } else {
    // every field starts at ba plus a multiple of 4: one aligned base, one shift for all
    const uint32_t b = ba & ~3u, sh = (ba & 3u) * 8u;
    const uint32_t a = b + 4 * t;
#pragma unroll
    for (int i = 0; i < 8; ++i) w.ql[i] = __funnelshift_r(lds_u32(a + 16 * i), lds_u32(a + 16 * i + 4), sh);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w.qh[i] = __funnelshift_r(lds_u32(a + 128 + 16 * i), lds_u32(a + 128 + 16 * i + 4), sh);
    uint32_t v[5];  // the 16 scale bytes: five aligned words (the fifth only matters when sh != 0)
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = lds_u32(b + 192 + 4 * i);
    v[4] = lds_u32(b + (sh ? 208u : 204u));  // never past the super-block's last byte
#pragma unroll
    for (int i = 0; i < 4; ++i) w.sc[i] = __funnelshift_r(v[i], v[i + 1], sh);
  }
  w.d = f16_bits_to_f32(lds_u16(ba + 208));
}

__device__ __forceinline__ uint32_t ldg_u32_a2(const uint8_t* p) {  // 2-byte aligned 32-bit load
  return ldg_u16(p) | (ldg_u16(p + 2) << 16);
}

__device__ __forceinline__ void q6_load_global(Q6W& w, bool valid, const uint8_t* b, int t) {
#pragma unroll
  for (int i = 0; i < 8; ++i) w.ql[i] = valid ? ldg_u32_a2(b + 16 * i + 4 * t) : 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    w.qh[i] = valid ? ldg_u32_a2(b + 128 + 16 * i + 4 * t) : 0u;
    w.sc[i] = valid ? ldg_u32_a2(b + 192 + 4 * i) : 0u;
  }
  w.d = valid ? f16_bits_to_f32(ldg_u16(b + 208)) : 0.f;
}

// ---------------------------------------------------------------------------------------
// 8-row kernels (1..8 q8_1 rows, one 8-column MMA group)
// ---------------------------------------------------------------------------------------
//
// One persistent 512-thread CTA per SM over 16-row weight tiles; warp w runs K-slice w of every
// tile (q6_slice_begin), and the 16 slices of a tile are summed in warp order through shared
// memory.  Activations:
//   - the q8_1 d of block b and column c (float32, dxs) and -32 * (sum of the 16 codes of
//     sub-block 2b + e of column c) (int32, cor), staged once per CTA in the order lane (g, t)
//     reads them, 16 bytes at a time: dxs [b / 2][c / 2][b % 2][c % 2] (two blocks per load),
//     cor [b][c / 2][e][c % 2] (one block per load);
//   - the B fragments (4 codes of column g, values 4t..4t+3 of each sub-block): for K <= 8192
//     (at most 2 super-blocks per slice) each warp keeps the 32 words of its own slice in
//     registers, loaded once; beyond that the codes are staged whole, xs [8][rs] with
//     rs % 128 == 64, value k of super-block sb of column c at
//     c rs + 256 sb + 64 (k >> 6) + 16 ((k >> 2) & 3) + 4 ((k >> 4) & 3) + (k & 3),
//     so that lane (g, t) reads the fragments of sub-blocks 4q..4q+3 as one 16-byte word
//     (the 8 lanes of each phase on 8 distinct 16-byte bank groups).
// Padding columns (rows <= c < 8) are zero.
// Weights: either 1-D bulk copies (TMA) of stages of SR = 8 or 4 consecutive rows into a ring
// of shared memory (blocks 16-byte aligned; SR rows are 210 SR (k / 256) bytes, a multiple of
// 16 for SR = 8 always and for SR = 4 when k / 256 is even; a ragged last stage copies its
// 16-byte-multiple prefix in bulk and its last bytes with plain loads), or 16-bit global loads
// (blocks only 2-byte aligned).  A tile's stages are released at the tile's reduction barrier,
// so the ring holds two tiles when it can: one computed, the next one landing.
// MMA rows g and g + 8 of lane (g, t) are tile rows (g, g + 8) or (2g, 2g + 1), and the stage
// slots are padded, as the host finds fewest shared-memory bank conflicts for the weight
// fragment loads: rows 5880 bytes apart (K = 7168) put rows g and g + 1 on overlapping banks,
// rows 2g with 64 bytes of slot padding spread the 8 rows of one load over all 32 banks.

struct Q6Params {
  const uint8_t* blocks;
  int n, k;
  const uint8_t* q8;
  int rows;
  uint16_t* out;
  int64_t ldc;
};

constexpr int kQ6RegSlice = 2;    // super-blocks per slice whose B fragments stay in registers
constexpr int kQ6MaxStages = 16;
static __device__ int q6_fault_word = 0;

struct Q6RowsParams {
  Q6Params q;
  int ns;            // ring stages (streamed)
  int stage_rows;    // SR: 4 or 8
  int stage_stride;  // bytes per stage slot (>= SR rows, multiple of 128)
  int ring_offset;   // byte offset of the ring in dynamic shared memory
  int row_pair;      // 1: MMA rows g, g + 8 are tile rows 2g, 2g + 1; 0: tile rows g, g + 8
  int early_w;       // the preceding kernel is this library's q8_1 quantize: weight copies may start before it ends
};

__host__ __device__ __forceinline__ int q6_act_stride(int k) { return k + ((64 - k % 128) + 128) % 128; }
__host__ __device__ __forceinline__ bool q6_reg_acts(int k) { return (k / 256 + kQ6Slices - 1) / kQ6Slices <= kQ6RegSlice; }
constexpr size_t kQ6RedBytes = 2ull * kQ6Warps * 32 * 4 * 4;  // [2][warps][32 lanes][4 floats]
// dxs, cor, then (smem activations) xs, then the reduction buffer.
__host__ __device__ __forceinline__ size_t q6_dx_bytes(int k) { return (size_t)(k / 32) * kQ6MaxRows * 4; }
__host__ __device__ __forceinline__ size_t q6_cor_bytes(int k) { return (size_t)(k / 16) * kQ6MaxRows * 4; }
__host__ __device__ __forceinline__ size_t q6_base_bytes(int k, bool reg_acts) {
  return q6_dx_bytes(k) + q6_cor_bytes(k) + (reg_acts ? 0 : (size_t)kQ6MaxRows * q6_act_stride(k)) + kQ6RedBytes;
}

// Stage dxs and cor (and, without register fragments, xs).
__device__ void q6_stage_acts(const Q6Params& p, uint8_t* smem, bool stage_codes) {
  const int nb32 = p.k / 32;
  const int rs = q6_act_stride(p.k);
  float* dxs = reinterpret_cast<float*>(smem);
  int* cor = reinterpret_cast<int*>(smem + q6_dx_bytes(p.k));
  uint8_t* xs = smem + q6_dx_bytes(p.k) + q6_cor_bytes(p.k);
  for (int it = threadIdx.x; it < kQ6MaxRows * nb32; it += blockDim.x) {
    const int m = it / nb32, b = it % nb32;
    const uint32_t* bw = reinterpret_cast<const uint32_t*>(p.q8 + ((int64_t)m * nb32 + b) * 36);
    dxs[(b >> 1) * 16 + (m >> 1) * 4 + (b & 1) * 2 + (m & 1)] = m < p.rows ? f16_bits_to_f32(bw[0] & 0xffffu) : 0.f;
    int s0 = 0, s1 = 0;
    if (m < p.rows) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s0 = __dp4a((int)bw[1 + i], 0x01010101, s0);
        s1 = __dp4a((int)bw[5 + i], 0x01010101, s1);
      }
    }
    cor[b * 16 + (m >> 1) * 4 + (m & 1)] = -32 * s0;
    cor[b * 16 + (m >> 1) * 4 + 2 + (m & 1)] = -32 * s1;
    if (!stage_codes) continue;
    uint8_t* dst = xs + m * rs + (b >> 3) * 256;
    const int kb = (b & 7) * 32;  // first value of this block inside its super-block
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = kb + 4 * i;
      *reinterpret_cast<uint32_t*>(dst + 64 * (k >> 6) + 16 * ((k >> 2) & 3) + 4 * ((k >> 4) & 3)) =
          m < p.rows ? bw[1 + i] : 0u;
    }
  }
}

// B fragment of lane (g, t) for sub-block j of super-block sb, straight from the q8_1 rows.
__device__ __forceinline__ uint32_t q6_bfrag(const Q6Params& p, int col, int sb, int j, int t) {
  if (col >= p.rows) return 0u;
  const int nb32 = p.k / 32;
  return *reinterpret_cast<const uint32_t*>(p.q8 + ((int64_t)col * nb32 + 8 * sb + (j >> 1)) * 36 + 4 +
                                            16 * (j & 1) + 4 * t);
}

// One super-block of the 16-row tile (MMA rows g: wa, g+8: wb) against the 8 columns: bw[j] is
// the lane's B fragment of sub-block j; dxs and cor point at the super-block's staged values
// (256 and 512 bytes a super-block) plus 16 t.
template <bool kCol0>
__device__ __forceinline__ void q6_superblock_8(float (&acc)[4], const Q6W& wa, const Q6W& wb, const uint32_t (&bw)[16],
                                                uint32_t dxs, uint32_t cor) {
  float tsb[4] = {0.f, 0.f, 0.f, 0.f};
  uint4 dx;
#pragma unroll
  for (int blk = 0; blk < 8; ++blk) {
    const int j0 = 2 * blk, j1 = j0 + 1;
    const uint4 c = lds128(cor + 64 * blk);  // columns 2t, 2t + 1 of sub-blocks j0, j1
    int d0[4], d1[4];
    mma_u8s8_c(d0, q6_codes_u8(wa, j0), q6_codes_u8(wb, j0), bw[j0], (int)c.x, (int)c.y);
    mma_u8s8_c(d1, q6_codes_u8(wa, j1), q6_codes_u8(wb, j1), bw[j1], (int)c.z, (int)c.w);
    if ((blk & 1) == 0) dx = lds128(dxs + 64 * (blk >> 1));  // blocks blk, blk + 1
    q6_block_step<kCol0>(tsb, d0, d1, q6_scale(wa, j0), q6_scale(wa, j1), q6_scale(wb, j0), q6_scale(wb, j1),
                         __uint_as_float((blk & 1) ? dx.z : dx.x), __uint_as_float((blk & 1) ? dx.w : dx.y));
  }
  q6_superblock_end<kCol0>(acc, tsb, wa.d, wb.d);
}

// Fixed-order sum over the 16 warps' partials of a tile, one BF16 store per output; run by the
// 128 threads of warps 12..15 (the K-slices are split with the longer ones first, so these
// warps never have more super-blocks than the others), thread r of them output r.
constexpr int kQ6RedWarp0 = kQ6Warps - 4;
__device__ __forceinline__ void q6_reduce_tile(const Q6Params& p, const float* red, int tile, int row_pair) {
  const int o = threadIdx.x - kQ6RedWarp0 * 32;
  const int rr = o % kQ6TileRows, cc = o / kQ6TileRows;
  const int row = tile * kQ6TileRows + rr;
  if (cc < p.rows && row < p.n) {
    const int gg = row_pair ? rr >> 1 : rr & 7, up = row_pair ? rr & 1 : rr >> 3;  // lane row, MMA half
    const int ln = gg * 4 + (cc >> 1), comp = up * 2 + (cc & 1);
    float sum = 0.f;
#pragma unroll
    for (int ww = 0; ww < kQ6Warps; ++ww) sum = __fadd_rn(sum, red[(ww * 32 + ln) * 4 + comp]);
    p.out[(int64_t)cc * p.ldc + row] = f32_to_bf16_bits(sum);
  }
}

// kCol0: one activation row (column 0 only; the other columns' sums are never formed).
template <bool kStream, bool kRegActs, bool kCol0>
__global__ void __launch_bounds__(kQ6Threads, 1) q6k_rows8_kernel(const Q6RowsParams sp) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full[kQ6MaxStages];
  grid_dependents_launch();
  const Q6Params& p = sp.q;
  const int nsb = p.k / 256;
  const int rs = q6_act_stride(p.k);
  const int64_t row_bytes = (int64_t)nsb * 210;
  float* red = reinterpret_cast<float*>(smem + q6_base_bytes(p.k, kRegActs) - kQ6RedBytes);
  const uint32_t ring = smem_u32(smem + sp.ring_offset);
  const uint32_t full0 = smem_u32(full);
  const int SR = kStream ? sp.stage_rows : 8, spt = kQ6TileRows / SR;

  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  const int nstages = spt * (T1 - T0);

  // Stage s of this CTA: rows [16 (T0 + s / spt) + SR (s % spt), +SR) clipped to n, slot s % NS.
  auto produce = [&](int s) {
    const int slot = s % sp.ns;
    const int64_t r0 = (int64_t)(T0 + s / spt) * kQ6TileRows + (s % spt) * SR;
    const int64_t nr = r0 >= p.n ? 0 : (p.n - r0 < SR ? p.n - r0 : SR);
    const uint32_t bytes = (uint32_t)(nr * row_bytes);
    const uint32_t bulk = bytes & ~15u;
    const uint32_t dst = ring + (uint32_t)slot * sp.stage_stride;
    const uint8_t* src = p.blocks + r0 * row_bytes;
    for (uint32_t o = bulk; o < bytes; o += 2) {  // ragged tail: at most 7 half-words
      const uint32_t v = ldg_u16(src + o);
      asm volatile("st.shared.u16 [%0], %1;" ::"r"(dst + o), "h"((unsigned short)v) : "memory");
    }
    umma::expect_tx(full0 + 8u * slot, bulk);
    if (bulk) umma::bulk_load(dst, src, bulk, full0 + 8u * slot, umma::l2_policy_evict_first());
  };

  if (kStream && threadIdx.x == 0) {
    for (int i = 0; i < sp.ns; ++i) umma::bar_init(full0 + 8u * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // Weight copies before the dependency wait only when the preceding kernel is this library's
    // q8_1 quantize (it writes neither the weights nor the ragged tail's source).
    if (sp.early_w)
      for (int s = 0; s < sp.ns && s < nstages; ++s) produce(s);
  }
  grid_dependency_wait();  // q8, and the blocks unless early_w, follow the preceding kernel
  if (kStream && threadIdx.x == 0 && !sp.early_w)
    for (int s = 0; s < sp.ns && s < nstages; ++s) produce(s);
  q6_stage_acts(p, smem, !kRegActs);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sb_begin = q6_slice_begin(nsb, warp), sb_end = q6_slice_begin(nsb, warp + 1);
  const uint32_t dx0 = smem_u32(smem) + (uint32_t)(16 * t);
  const uint32_t co0 = smem_u32(smem) + (uint32_t)(q6_dx_bytes(p.k) + 16 * t);
  const uint32_t xs0 = smem_u32(smem) + (uint32_t)(q6_dx_bytes(p.k) + q6_cor_bytes(p.k) + g * rs + 16 * t);
  uint32_t bfr[kQ6RegSlice][16];
  if (kRegActs) {
#pragma unroll
    for (int s = 0; s < kQ6RegSlice; ++s)
#pragma unroll
      for (int j = 0; j < 16; ++j) bfr[s][j] = sb_begin + s < sb_end ? q6_bfrag(p, g, sb_begin + s, j, t) : 0u;
  }
  __syncthreads();

  const int lra = sp.row_pair ? 2 * g : g, lrb = sp.row_pair ? 2 * g + 1 : g + 8;  // tile rows of MMA rows g, g+8
  const int sa_off = lra / SR, sb_off = lrb / SR;  // their stages within a tile
  for (int i = 0; T0 + i < T1; ++i) {
    const int tile = T0 + i;
    const int ra = tile * kQ6TileRows + lra, rb = tile * kQ6TileRows + lrb;
    const bool va = ra < p.n, vb = rb < p.n;
    uint32_t base_a = 0, base_b = 0;
    if (kStream) {
      bool ok = true;
      for (int q = 0; q < spt; ++q) {
        const int s = spt * i + q;
        ok &= umma::wait(full0 + 8u * (s % sp.ns), (s / sp.ns) & 1);
      }
      if (!ok) atomicOr(&q6_fault_word, 1);
      const int s_a = spt * i + sa_off, s_b = spt * i + sb_off;
      base_a = ring + (uint32_t)(s_a % sp.ns) * sp.stage_stride + (uint32_t)((lra % SR) * row_bytes);
      base_b = ring + (uint32_t)(s_b % sp.ns) * sp.stage_stride + (uint32_t)((lrb % SR) * row_bytes);
    }
    // the previous tile's reduction, on the warps with the shortest slices, while the others
    // start this tile
    if (warp >= kQ6RedWarp0 && i > 0) q6_reduce_tile(p, red + ((i - 1) & 1) * (kQ6Warps * 32 * 4), tile - 1, sp.row_pair);
    const uint8_t* ga = p.blocks + (int64_t)ra * row_bytes;
    const uint8_t* gb = p.blocks + (int64_t)rb * row_bytes;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    auto one = [&](int sb, const uint32_t (&bw)[16]) {
      Q6W wa, wb;
      if (kStream) {
        const uint32_t ba = base_a + (uint32_t)sb * 210u, bb = base_b + (uint32_t)sb * 210u;
        if (__all_sync(0xffffffffu, ((ba | bb) & 3u) == 0)) {
          q6_load_smem<true>(wa, va, ba, t);
          q6_load_smem<true>(wb, vb, bb, t);
        } else {
          q6_load_smem<false>(wa, va, ba, t);
          q6_load_smem<false>(wb, vb, bb, t);
        }
      } else {
        q6_load_global(wa, va, ga + (int64_t)sb * 210, t);
        q6_load_global(wb, vb, gb + (int64_t)sb * 210, t);
      }
      q6_superblock_8<kCol0>(acc, wa, wb, bw, dx0 + 256u * sb, co0 + 512u * sb);
    };
    if (kRegActs) {
#pragma unroll
      for (int s = 0; s < kQ6RegSlice; ++s)
        if (sb_begin + s < sb_end) one(sb_begin + s, bfr[s]);
    } else {
      for (int sb = sb_begin; sb < sb_end; ++sb) {
        uint32_t bw[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = lds128(xs0 + 256u * sb + 64 * q);
          bw[4 * q] = v.x, bw[4 * q + 1] = v.y, bw[4 * q + 2] = v.z, bw[4 * q + 3] = v.w;
        }
        one(sb, bw);
      }
    }
    // publish the partial sums; after the barrier the tile's stages are free, and its sums are
    // reduced during the next tile (the buffer of parity i & 1 is written again two tiles on,
    // after the next barrier, by when that reduction has read it)
    reinterpret_cast<float4*>(red + (i & 1) * (kQ6Warps * 32 * 4))[warp * 32 + lane] =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (kStream && threadIdx.x == 0)
      for (int q = 0; q < spt; ++q)
        if (spt * i + q + sp.ns < nstages) produce(spt * i + q + sp.ns);
  }
  if (warp >= kQ6RedWarp0 && T1 > T0) q6_reduce_tile(p, red + ((T1 - T0 - 1) & 1) * (kQ6Warps * 32 * 4), T1 - 1, sp.row_pair);
}

// ---------------------------------------------------------------------------------------
// Wide variant: 9..64 q8_1 rows in one weight pass.  Whole activation rows no longer fit in
// shared memory (64 rows of codes at K = 7168 take 458 KB), so the loop order is turned
// around: a CTA takes its 16-row weight tiles in row-blocks of up to W tiles, one tile per
// consumer warp, and the row-block walks K one super-block at a time.
//   - Activations: a producer warp copies each super-block's q8_1 blocks of every activation
//     row into a ring shared by the row-block's warps, with 4-byte cp.async into the order the
//     lanes read them (below) and one mbarrier arrival per lane; the activations are re-read
//     (from L2) once per row-block, not once per tile.
//   - Weights: every consumer warp streams its own tile through a private ring of `depth`
//     stages with 16-byte cp.async: per row the 16-byte aligned span that covers the
//     super-block's 210 bytes (at most 224; super-blocks are only 2-byte aligned), read back
//     at the span's offset.  The buffer's last bytes past its last 16-byte boundary are stored
//     with plain loads, so no copy reads past the weight buffer.
// Each consumer warp decodes a weight fragment once per sub-block ((q - 32) as signed bytes)
// and runs NT 8-column MMAs on it.  The K-slices of the 8-row kernels are kept: each slice is
// accumulated alone from 0 and added to the total at the slice's end (q6_slice_ends).
// NT <= 4: 15 consumer warps + 1 producer (128 registers a thread); NT = 8: 11 + 1 (168, a
// small spill; 7 warps of 228 registers left the schedulers short of warps: 1040 against
// 881 us for 64 rows on a 129280 x 7168 head).
constexpr int kQWSpan = 240;       // staged bytes per weight row and super-block (>= 224)
constexpr int kQWTileBytes = kQ6TileRows * kQWSpan;
constexpr int kQWMaxActStages = 4;
// An activation stage holds one super-block of the NT * 8 q8_1 rows, regrouped for the lanes:
//   - codes: [block b][8-column group ct][g][t] x (codes 4t..4t+3, codes 16+4t..16+4t+3) of
//     row 8 ct + g: lane (g, t)'s B words of sub-blocks 2b and 2b + 1 in one 8-byte load (the
//     32 lanes read 256 contiguous bytes);
//   - then (f16 d, f16 s): [block b][ct][t][column 2t, 2t + 1]: both of lane (g, t)'s columns'
//     d in one 8-byte load.
template <int NT>
constexpr uint32_t qw_codes_bytes() {
  return (uint32_t)(8 * NT * 32 * 8);
}
template <int NT>
constexpr uint32_t qw_act_bytes() {
  return qw_codes_bytes<NT>() + (uint32_t)(256 * NT);
}

template <int NT>
struct QW {
  static constexpr int kWarps = NT >= 8 ? 11 : 15;  // consumer warps
  static constexpr int kThreads = (kWarps + 1) * 32;
};

struct Q6WideParams {
  Q6Params q;
  int act_stages;  // activation ring stages of qw_act_bytes<NT>() bytes
  int depth;       // weight stages per consumer warp (>= 2)
  int early_w;     // the preceding kernel is this library's q8_1 quantize (see Q6RowsParams)
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// The mbarrier receives one arrival when this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// One super-block of one warp's 16-row tile against NT 8-column groups of the staged chunk at
// `xs` (the regrouped codes, then d and s; see qw_act_bytes).
template <int NT>
__device__ __forceinline__ void q6_superblock_wide(float (&acc)[NT][4], const Q6W& wa, const Q6W& wb, uint32_t xs,
                                                   int g, int t) {
  float tsb[NT][4];
#pragma unroll
  for (int ct = 0; ct < NT; ++ct)
#pragma unroll
    for (int i = 0; i < 4; ++i) tsb[ct][i] = 0.f;
#pragma unroll
  for (int blk = 0; blk < 8; ++blk) {
    const int j0 = 2 * blk, j1 = j0 + 1;
    const uint32_t a00 = q6_codes_s8(wa, j0), a01 = q6_codes_s8(wb, j0);
    const uint32_t a10 = q6_codes_s8(wa, j1), a11 = q6_codes_s8(wb, j1);
    const int ra0 = q6_scale(wa, j0), ra1 = q6_scale(wa, j1), rb0 = q6_scale(wb, j0), rb1 = q6_scale(wb, j1);
#pragma unroll
    for (int ct = 0; ct < NT; ++ct) {
      const uint2 bw = lds_u64(xs + (uint32_t)((((blk * NT + ct) * 8 + g) * 4 + t) * 8));
      int d0[4], d1[4];
      mma_s8s8_z(d0, a00, a01, bw.x);
      mma_s8s8_z(d1, a10, a11, bw.y);
      const uint2 dd = lds_u64(xs + qw_codes_bytes<NT>() + (uint32_t)(((blk * NT + ct) * 4 + t) * 8));
      const float dx0 = f16_bits_to_f32(dd.x & 0xffffu), dx1 = f16_bits_to_f32(dd.y & 0xffffu);
      q6_block_step(tsb[ct], d0, d1, ra0, ra1, rb0, rb1, dx0, dx1);
    }
  }
#pragma unroll
  for (int ct = 0; ct < NT; ++ct) q6_superblock_end(acc[ct], tsb[ct], wa.d, wb.d);
}

// Stage super-block sb of the 16 rows of tile `tile` into `dst` (row i at i * kQWSpan) with
// this lane's share of the 16-byte pieces; rows at or past n are skipped.
__device__ __forceinline__ void q6_stage_tile(const Q6Params& p, int64_t row_bytes, uintptr_t buf_end, int tile,
                                              int sb, uint32_t dst, int lane) {
  for (int c = lane; c < kQ6TileRows * (kQWSpan / 16); c += 32) {
    const int i = c / (kQWSpan / 16), piece = c % (kQWSpan / 16);
    const int row = tile * kQ6TileRows + i;
    if (row >= p.n) continue;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p.blocks) + (uintptr_t)((int64_t)row * row_bytes + 210 * sb);
    const uintptr_t a16 = a & ~uintptr_t(15);
    const uintptr_t src = a16 + 16u * piece;
    if (src >= a + 210) continue;  // past the span
    const uint32_t d = dst + (uint32_t)(i * kQWSpan + 16 * piece);
    if (src + 16 <= buf_end) {
      cp_async16(d, reinterpret_cast<const void*>(src));
    } else {  // the buffer's last bytes: plain 16-bit loads up to its end
      for (uintptr_t o = src; o < buf_end; o += 2)
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(d + (uint32_t)(o - src)),
                     "h"((unsigned short)ldg_u16(reinterpret_cast<const void*>(o)))
                     : "memory");
    }
  }
}

template <int NT>
__global__ void __launch_bounds__(QW<NT>::kThreads, 1) q6k_wide_kernel(const Q6WideParams wp) {
  constexpr int kWarps = QW<NT>::kWarps;
  extern __shared__ __align__(128) uint8_t smem[];
  grid_dependents_launch();
  // launched early (programmatic): q8, blocks and out follow the preceding kernel; with early_w
  // only the consumers' first weight stages are requested before the wait
  if (!wp.early_w) grid_dependency_wait();
  __shared__ __align__(8) uint64_t full[kQWMaxActStages], empty[kQWMaxActStages];
  const Q6Params& p = wp.q;
  const int nsb = p.k / 256;
  const int nb32 = p.k / 32;
  const int64_t row_bytes = (int64_t)nsb * 210;
  const uintptr_t buf_end = reinterpret_cast<uintptr_t>(p.blocks) + (uintptr_t)((int64_t)p.n * row_bytes);
  constexpr uint32_t kActBytes = qw_act_bytes<NT>();
  const int ns = wp.act_stages, depth = wp.depth;
  const uint32_t act_ring = smem_u32(smem);
  const uint32_t w_rings = act_ring + (uint32_t)ns * kActBytes;
  const uint32_t full0 = smem_u32(full), empty0 = smem_u32(empty);

  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  const int nt = T1 - T0;
  const int nrb = (nt + kWarps - 1) / kWarps;  // row-blocks, as even as possible
  const int nchunks = nrb * nsb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the activation ring starts zero: the padding rows [rows, kRows) are never copied
  for (int i = threadIdx.x; i < ns * (int)(kActBytes / 4); i += blockDim.x) reinterpret_cast<uint32_t*>(smem)[i] = 0u;
  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      umma::bar_init(full0 + 8u * i, 32);  // one arrival per producer lane, when its copies land
      umma::bar_init(empty0 + 8u * i, kWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---------------- producer: chunk c = (row-block c / nsb, super-block c % nsb)
    if (wp.early_w) grid_dependency_wait();
    for (int c = 0; c < nchunks; ++c) {
      const int slot = c % ns, sb = c % nsb;
      if (c >= ns && !umma::wait(empty0 + 8u * slot, ((c / ns) - 1) & 1)) atomicOr(&q6_fault_word, 4);
      __syncwarp();
      const uint32_t st = act_ring + (uint32_t)slot * kActBytes;
      for (int q = lane; q < p.rows * 64; q += 32) {  // code word w of block b of row m
        const int m = q >> 6, b = (q >> 3) & 7, w = q & 7;
        cp_async4(st + (uint32_t)(((((b * NT + (m >> 3)) * 8 + (m & 7)) * 4 + (w & 3)) * 2 + (w >> 2)) * 4),
                  p.q8 + ((int64_t)m * nb32 + 8 * sb + b) * 36 + 4 + 4 * w);
      }
      for (int q = lane; q < p.rows * 8; q += 32) {  // (d, s) of block b of row m
        const int m = q >> 3, b = q & 7;
        cp_async4(st + qw_codes_bytes<NT>() + (uint32_t)((((b * NT + (m >> 3)) * 4 + ((m & 7) >> 1)) * 2 + (m & 1)) * 4),
                  p.q8 + ((int64_t)m * nb32 + 8 * sb + b) * 36);
      }
      cp_async_arrive(full0 + 8u * slot);
    }
    cp_async_wait<0>();  // nothing of this thread in flight at exit
    return;
  }

  // ---------------- consumers
  const int g = lane >> 2, t = lane & 3;
  const uint32_t my_ring = w_rings + (uint32_t)(warp * depth * kQWTileBytes);
  int c = 0;
  for (int r = 0; r < nrb; ++r) {
    const int tb0 = T0 + (int)((int64_t)r * nt / nrb), tb1 = T0 + (int)((int64_t)(r + 1) * nt / nrb);
    const int tile = tb0 + warp;
    const bool active = tile < tb1;
    const int r0 = tile * kQ6TileRows + g;
    const bool va = active && r0 < p.n, vb = active && r0 + 8 < p.n;
    // weight pipeline: stages 0 .. depth-2 in flight before the loop (one group each)
    for (int s = 0; s < depth - 1; ++s) {
      if (active && s < nsb) q6_stage_tile(p, row_bytes, buf_end, tile, s, my_ring + (uint32_t)(s * kQWTileBytes), lane);
      cp_async_commit();
    }
    if (wp.early_w && r == 0) grid_dependency_wait();
    float tot[NT][4], sl[NT][4];
#pragma unroll
    for (int ct = 0; ct < NT; ++ct)
#pragma unroll
      for (int i = 0; i < 4; ++i) tot[ct][i] = sl[ct][i] = 0.f;
    for (int sb = 0; sb < nsb; ++sb, ++c) {
      const int slot = c % ns;
      const uint32_t st = act_ring + (uint32_t)slot * kActBytes;
      // keep depth - 1 weight stages in flight: issue sb + depth - 1, wait for sb
      {
        const int s2 = sb + depth - 1;
        if (active && s2 < nsb)
          q6_stage_tile(p, row_bytes, buf_end, tile, s2, my_ring + (uint32_t)((s2 % depth) * kQWTileBytes), lane);
        cp_async_commit();
      }
      if (depth == 3) cp_async_wait<2>(); else cp_async_wait<1>();
      __syncwarp();
      if (!umma::wait(full0 + 8u * slot, (c / ns) & 1)) atomicOr(&q6_fault_word, 2);
      if (active) {
        const uint32_t wbase = my_ring + (uint32_t)((sb % depth) * kQWTileBytes);
        const uint32_t ba = wbase + (uint32_t)(g * kQWSpan) +
                            (uint32_t)((reinterpret_cast<uintptr_t>(p.blocks) + (uintptr_t)((int64_t)r0 * row_bytes + 210 * sb)) & 15u);
        const uint32_t bb = wbase + (uint32_t)((g + 8) * kQWSpan) +
                            (uint32_t)((reinterpret_cast<uintptr_t>(p.blocks) + (uintptr_t)((int64_t)(r0 + 8) * row_bytes + 210 * sb)) & 15u);
        Q6W wa, wb;
        if (__all_sync(0xffffffffu, ((ba | bb) & 3u) == 0)) {
          q6_load_smem<true>(wa, va, ba, t);
          q6_load_smem<true>(wb, vb, bb, t);
        } else {
          q6_load_smem<false>(wa, va, ba, t);
          q6_load_smem<false>(wb, vb, bb, t);
        }
        q6_superblock_wide<NT>(sl, wa, wb, st, g, t);
      }
      __syncwarp();  // the weight stage and the activation slot are read
      if (lane == 0) umma::arrive(empty0 + 8u * slot);
      // end of a slice of the 8-row kernels: add it to the total and restart
      if (q6_slice_ends(nsb, sb)) {
#pragma unroll
        for (int ct = 0; ct < NT; ++ct)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            tot[ct][i] = __fadd_rn(tot[ct][i], sl[ct][i]);
            sl[ct][i] = 0.f;
          }
      }
    }
    cp_async_wait<0>();
    __syncwarp();
    // empty slices (nsb < 16: idle warps of the 8-row kernels) add +0
    for (int w = nsb < kQ6Warps ? nsb : kQ6Warps; w < kQ6Warps; ++w)
#pragma unroll
      for (int ct = 0; ct < NT; ++ct)
#pragma unroll
        for (int i = 0; i < 4; ++i) tot[ct][i] = __fadd_rn(tot[ct][i], 0.f);
    if (active) {
#pragma unroll
      for (int ct = 0; ct < NT; ++ct) {
        const int m0 = 8 * ct + 2 * t;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = m0 + (i & 1), row = r0 + 8 * (i >> 1);
          if (m < p.rows && row < p.n) p.out[(int64_t)m * p.ldc + row] = f32_to_bf16_bits(tot[ct][i]);
        }
      }
    }
  }
}

}  // namespace

namespace {

template <int NT>
int launch_wide(const Q6Params& p, int sms, int smem_optin, cudaStream_t s, bool early_w) {
  constexpr int kWarps = QW<NT>::kWarps;
  const size_t act = qw_act_bytes<NT>();
  const size_t limit = (size_t)smem_optin > 1024 ? (size_t)smem_optin - 1024 : 0;  // static smem < 1 KB
  // three weight stages per warp when they fit beside at least two activation stages
  int depth = 3;
  if ((size_t)kWarps * depth * kQWTileBytes + 2 * act > limit) depth = 2;
  const size_t wbytes = (size_t)kWarps * depth * kQWTileBytes;
  if (wbytes + 2 * act > limit) return DLMH_ERR_UNSUPPORTED;
  int ns = (int)((limit - wbytes) / act);
  if (ns > kQWMaxActStages) ns = kQWMaxActStages;
  const size_t smem = (size_t)ns * act + wbytes;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(q6k_wide_kernel<NT>), (int)smem) != DLMH_OK)
    return DLMH_ERR_CUDA;
  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int grid = ntiles < sms ? ntiles : sms;
  return umma::launch_pdl(q6k_wide_kernel<NT>, dim3(grid), dim3(QW<NT>::kThreads), smem, s,
                          Q6WideParams{p, ns, depth, early_w ? 1 : 0});
}

template <bool kStream, bool kRegActs, bool kCol0 = false>
int launch_rows8(const Q6RowsParams& sp, int grid, size_t smem, cudaStream_t s) {
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(q6k_rows8_kernel<kStream, kRegActs, kCol0>), (int)smem) != DLMH_OK)
    return DLMH_ERR_CUDA;
  return umma::launch_pdl(q6k_rows8_kernel<kStream, kRegActs, kCol0>, dim3(grid), dim3(kQ6Threads), smem, s, sp);
}

}  // namespace

// Bank conflicts of the weight-fragment loads of the streamed 8-row kernel: for each of the
// two loads (MMA rows g and g + 8) of an even and an odd super-block, the largest number of
// distinct 4-byte words that the 32 lanes ask of one bank, summed.  Stage slot s starts at
// s * stride (the ring is 128-byte aligned); the tile's first slot stands for all.
static int q6_bank_cost(int64_t row_bytes, int sr, size_t stride, int row_pair) {
  int cost = 0;
  for (int odd = 0; odd < 2; ++odd)
    for (int half = 0; half < 2; ++half) {
      int64_t words[32][32];
      int nw[32] = {0}, ways = 0;
      for (int g = 0; g < 8; ++g) {
        const int lr = row_pair ? 2 * g + half : g + 8 * half;
        const int64_t off = (int64_t)(lr / sr) * (int64_t)stride + (lr % sr) * row_bytes + 210 * odd;
        for (int t = 0; t < 4; ++t) {
          const int64_t w = (off >> 2) + t;
          const int bank = (int)(w & 31);
          bool seen = false;
          for (int i = 0; i < nw[bank]; ++i) seen |= words[bank][i] == w;
          if (!seen) words[bank][nw[bank]++] = w;
          ways = nw[bank] > ways ? nw[bank] : ways;
        }
      }
      cost += ways;
    }
  return cost;
}

// The lane row map and the stage-slot padding (0, 16, ..., 112 bytes) with the fewest conflicts
// (ties: the plain map, then the least padding).
static void q6_bank_layout(int64_t row_bytes, int sr, int* row_pair, size_t* pad) {
  const size_t base = ((size_t)sr * (size_t)row_bytes + 127) / 128 * 128;
  int best = -1;
  for (int rp = 0; rp < 2; ++rp)
    for (size_t pd = 0; pd < 128; pd += 16) {
      const int c = q6_bank_cost(row_bytes, sr, base + pd, rp);
      if (best < 0 || c < best) best = c, *row_pair = rp, *pad = pd;
    }
}

int q6k_wide_rows(int rows) { return rows <= 8 ? 8 : rows <= 16 ? 16 : rows <= 32 ? 32 : 64; }

int q6k_mmvq_launch(const uint8_t* blocks, int n, int k, const uint8_t* q8, int rows, uint16_t* out, int64_t ldc,
                    cudaStream_t s, bool after_prepass) {
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  const Q6Params p{blocks, n, k, q8, rows, out, ldc};
  if (rows > kQ6MaxRows) {  // 9..64 rows (16-byte aligned blocks, q8_1 rows)
    if (rows > 64) return DLMH_ERR_ROWS;
    if ((reinterpret_cast<uintptr_t>(q8) & 15u) || (reinterpret_cast<uintptr_t>(blocks) & 15u)) return DLMH_ERR_ALIGN;
    if (rows <= 2 * kQ6MaxRows && q6_reg_acts(k)) {
      // 9..16 rows: two passes of the streamed 8-row kernel take less time than one of the
      // 16-row wide kernel (on a 129280 x 7168 head, 2 x ~183 against 416 us); same bits.  The
      // second pass follows the first, which writes neither the weights nor its q8_1 rows.
      const int rc = q6k_mmvq_launch(blocks, n, k, q8, kQ6MaxRows, out, ldc, s, after_prepass);
      if (rc != DLMH_OK) return rc;
      const int64_t q8_row = (int64_t)(k / 32) * 36;
      return q6k_mmvq_launch(blocks, n, k, q8 + kQ6MaxRows * q8_row, rows - kQ6MaxRows, out + kQ6MaxRows * ldc, ldc, s,
                             true);
    }
    switch (q6k_wide_rows(rows)) {
      case 16: return launch_wide<2>(p, di.sms, di.smem_optin, s, after_prepass);
      case 32: return launch_wide<4>(p, di.sms, di.smem_optin, s, after_prepass);
      default: return launch_wide<8>(p, di.sms, di.smem_optin, s, after_prepass);
    }
  }
  const bool reg = q6_reg_acts(k);
  const size_t base_smem = q6_base_bytes(k, reg);
  const int ntiles = (n + kQ6TileRows - 1) / kQ6TileRows;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  // Streamed when the B fragments stay in registers (K <= 8192: then the ring has room), the
  // blocks start 16-byte aligned (then every stage does) and the ring holds more than one tile:
  // the stage size (8 or 4 rows) that gives the most tiles in the ring, up to two (the next
  // tile lands while this one is computed).  Otherwise 16-bit global weight loads.
  const size_t ring_offset = (base_smem + 127) / 128 * 128;
  const size_t limit = (size_t)di.smem_optin > 2048 ? (size_t)di.smem_optin - 2048 : 0;
  const int nsb = k / 256;
  Q6RowsParams best{p, 0, 0, 0, (int)ring_offset, 0, after_prepass ? 1 : 0};
  double best_tiles = 1.0;
  for (int sr = 8; sr >= 4 && reg && (reinterpret_cast<uintptr_t>(blocks) & 15u) == 0; sr -= 4) {
    if (((size_t)sr * nsb * 210) % 16 != 0) continue;
    const int spt = kQ6TileRows / sr;
    int row_pair = 0;
    size_t pad = 0;
    q6_bank_layout((int64_t)nsb * 210, sr, &row_pair, &pad);
    const size_t stage_stride = ((size_t)sr * nsb * 210 + 127) / 128 * 128 + pad;
    int ns = limit > ring_offset ? (int)((limit - ring_offset) / stage_stride) : 0;
    if (ns > 2 * spt) ns = 2 * spt;
    if (ns > kQ6MaxStages) ns = kQ6MaxStages;
    const double tiles = (double)ns / spt;
    if (tiles > best_tiles + 1e-9) {
      best.ns = ns, best.stage_rows = sr, best.stage_stride = (int)stage_stride, best.row_pair = row_pair;
      best_tiles = tiles;
    }
  }
  if (best.ns > 0) {
    const size_t smem = ring_offset + (size_t)best.ns * best.stage_stride;
    return rows == 1 ? launch_rows8<true, true, true>(best, grid, smem, s) : launch_rows8<true, true>(best, grid, smem, s);
  }
  if (base_smem + 1024 > (size_t)di.smem_optin) return DLMH_ERR_UNSUPPORTED;
  const Q6RowsParams sp{p, 1, 8, 0, 0, 0, 0};
  return reg ? launch_rows8<false, true>(sp, grid, base_smem, s) : launch_rows8<false, false>(sp, grid, base_smem, s);
}

int q6k_fault(int reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, q6_fault_word, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(q6_fault_word, &zero, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  }
  return v;
}

}  // namespace dlmh
