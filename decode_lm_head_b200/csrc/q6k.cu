// Q6_K super-blocks x block_q8_1 rows on int8 warp MMAs.
//
// Same decomposition as the row-tile GEMV: one persistent 512-thread CTA per SM over
// 16-row weight tiles, the super-blocks of a tile split across 16 warps as evenly as
// possible (q6_slice_begin), a fixed-order
// cross-warp reduction at the end of each tile.  Per 16-value sub-block j a warp runs one
// s8 m16n8k16 MMA: the weight codes (q - 32) times the q8_1 codes, an exact int32 dot;
// the dot is then scaled in f32 by d(super-block) * scales[j] of the weight row, and
// every 32 values (one q8_1 block) by the row's q8_1 d.
//
// Super-block byte map (210 bytes): ql[128] @0, qh[64] @128, int8 scales[16] @192,
// f16 d @208.  Value i = 128h + 32u + l (h < 2, u < 4, l < 32): low 4 bits from
// ql[64h + 32(u&1) + l] (low nibble for u < 2, high nibble for u >= 2), top 2 bits from
// bits 2u..2u+1 of qh[32h + l]; sub-block j = i / 16 uses scales[j].
// Lane (g, t) of a warp feeds the MMA with values 4t..4t+3 of every sub-block, i.e. the
// 4 consecutive ql / qh bytes at l = 16(j&1) + 4t, for rows g and g+8.
// Super-blocks are only 2-byte aligned in the raw layout, so bytes are fetched with
// 16-bit read-only loads (each 32-byte sector still comes from DRAM once).
#include "dlmh_common.cuh"
#include "gemv_launch.h"
#include "q6k_slices.h"
#include "umma_common.cuh"

namespace dlmh {
namespace {

constexpr int kQ6Warps = 16;
constexpr int kQ6Threads = kQ6Warps * 32;
constexpr int kQ6TileRows = 16;
constexpr int kQ6MaxRows = 8;  // q8_1 rows per launch (one 8-column MMA tile)

__device__ __forceinline__ uint32_t ldg_u32_a2(const uint8_t* p) {  // 2-byte aligned 32-bit load
  return ldg_u16(p) | (ldg_u16(p + 2) << 16);
}

// (q - 32) as int8 for four 6-bit codes packed one per byte.
__device__ __forceinline__ uint32_t q6_to_s8x4(uint32_t q) {
  const uint32_t x = q ^ 0x20202020u;          // bit 5 set <=> q < 32
  const uint32_t s = x & 0x20202020u;
  return x | (s * 6u);                          // sign-extend bit 5 into bits 6, 7
}

// acc + (is * d) * dx with one rounding per step (a product, then a fused multiply-add), the
// same in every Q6_K kernel whatever the compiler would contract.
__device__ __forceinline__ float q6_block_step(float acc, int is, float d, float dx) {
  return __fmaf_rn(__fmul_rn((float)is, d), dx, acc);
}

// The K-slices (q6k_slices.h): warp w of the 8-row kernels runs slice w.
static_assert(kQ6Warps == kQ6Slices, "one K-slice per warp of the 8-row kernels");

// One super-block for rows g (a) and g+8 (b) of a 16-row tile against activation columns 2t
// and 2t+1 (acc[0..1]: row a, acc[2..3]: row b).  Per q8_1 block (sub-blocks j0, j1) the two
// exact int32 sub-block dots are scaled by their int8 sub-scales and summed in int32 -- exact,
// |sum| < 2^24 so its f32 conversion is exact too -- then multiplied by the super-block d and
// the q8_1 d in f32.  Shared by both Q6_K kernels so that they give the same bits.
__device__ __forceinline__ void q6_superblock(float (&acc)[4], const uint32_t (&qla)[8], const uint32_t (&qlb)[8],
                                              const uint32_t (&qha)[4], const uint32_t (&qhb)[4],
                                              const uint32_t (&sca)[4], const uint32_t (&scb)[4], float da, float db,
                                              const int8_t* xsb, const float* dx, int nb32, int sb, int t) {
#pragma unroll
  for (int blk = 0; blk < 8; ++blk) {  // q8_1 block = sub-blocks 2blk, 2blk+1
    int is0 = 0, is1 = 0, is2 = 0, is3 = 0;
#pragma unroll
    for (int hj = 0; hj < 2; ++hj) {
      const int j = 2 * blk + hj;
      const int h = j >> 3, u = (j & 7) >> 1;
      // ql word index: 64h + 32(u&1) + 16(j&1) -> q = 4h + 2(u&1) + (j&1); qh: 32h + 16(j&1)
      const int qi = 4 * h + 2 * (u & 1) + (j & 1);
      const int hi = 2 * h + (j & 1);
      const int nsh = (u >> 1) * 4, hsh = 2 * u;
      const uint32_t qa = ((qla[qi] >> nsh) & 0x0f0f0f0fu) | (((qha[hi] >> hsh) & 0x03030303u) << 4);
      const uint32_t qb = ((qlb[qi] >> nsh) & 0x0f0f0f0fu) | (((qhb[hi] >> hsh) & 0x03030303u) << 4);
      const uint32_t bx = *reinterpret_cast<const uint32_t*>(xsb + 16 * j + 4 * t);
      int d4[4] = {0, 0, 0, 0};
      mma_s8_16816(d4, q6_to_s8x4(qa), q6_to_s8x4(qb), bx);
      const int sha = 24 - 8 * (j & 3);  // sign-extend byte j&3 of the scale word
      const int ra = (int)(sca[j >> 2] << sha) >> 24;
      const int rb = (int)(scb[j >> 2] << sha) >> 24;
      is0 += d4[0] * ra;
      is1 += d4[1] * ra;
      is2 += d4[2] * rb;
      is3 += d4[3] * rb;
    }
    const int b32 = sb * 8 + blk;
    const float dx0 = dx[(2 * t) * nb32 + b32], dx1 = dx[(2 * t + 1) * nb32 + b32];
    acc[0] = q6_block_step(acc[0], is0, da, dx0);
    acc[1] = q6_block_step(acc[1], is1, da, dx1);
    acc[2] = q6_block_step(acc[2], is2, db, dx0);
    acc[3] = q6_block_step(acc[3], is3, db, dx1);
  }
}

struct Q6Params {
  const uint8_t* blocks;
  int n, k;
  const uint8_t* q8;
  int rows;
  uint16_t* out;
  int64_t ldc;
};

__device__ __forceinline__ int q6_row_stride(int k) {  // qs bytes per staged row, % 128 == 16
  int s = k;
  int r = s % 128;
  return s + ((16 - r) + 128) % 128;
}

__global__ void __launch_bounds__(kQ6Threads, 1) q6k_mmvq_kernel(const Q6Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_dependents_launch();
  grid_dependency_wait();  // launched early (programmatic): q8, blocks and out follow the preceding kernel
  const int nsb = p.k / 256;
  const int nb32 = p.k / 32;
  const int rs = q6_row_stride(p.k);
  int8_t* xs = reinterpret_cast<int8_t*>(smem);                              // [8][rs]
  float* dx = reinterpret_cast<float*>(smem + kQ6MaxRows * rs);              // [8][nb32]
  float* red = dx + kQ6MaxRows * nb32;                                       // [2][16 warps][32 lanes][4]

  // ---- stage the q8_1 rows: codes in natural order, d as f32
  for (int it = threadIdx.x; it < kQ6MaxRows * nb32; it += kQ6Threads) {
    const int m = it / nb32, b = it % nb32;
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float d = 0.f;
    if (m < p.rows) {
      const uint8_t* blk = p.q8 + ((int64_t)m * nb32 + b) * 36;
      const uint32_t* bw = reinterpret_cast<const uint32_t*>(blk);
      d = f16_bits_to_f32(bw[0] & 0xffff);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = bw[1 + i];
    }
    dx[m * nb32 + b] = d;
    uint4* dst = reinterpret_cast<uint4*>(xs + m * rs + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  __syncthreads();

  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sb_begin = q6_slice_begin(nsb, warp), sb_end = q6_slice_begin(nsb, warp + 1);
  const int64_t row_bytes = (int64_t)nsb * 210;
  const int8_t* xrow = xs + g * rs;  // B column g
  int parity = 0;

  for (int tile = T0; tile < T1; ++tile) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int r0 = tile * kQ6TileRows + g;
    const bool va = r0 < p.n, vb = r0 + 8 < p.n;
    for (int sb = sb_begin; sb < sb_end; ++sb) {
      const uint8_t* ba = p.blocks + (int64_t)r0 * row_bytes + (int64_t)sb * 210;
      const uint8_t* bb = ba + 8 * row_bytes;
      uint32_t qla[8], qlb[8], qha[4], qhb[4], sca[4], scb[4];
      float da = 0.f, db = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // ql bytes 16i + 4t (i = 4h + c: 64h + 16c)
        qla[i] = va ? ldg_u32_a2(ba + 16 * i + 4 * t) : 0u;
        qlb[i] = vb ? ldg_u32_a2(bb + 16 * i + 4 * t) : 0u;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // qh bytes 128 + 16i + 4t
        qha[i] = va ? ldg_u32_a2(ba + 128 + 16 * i + 4 * t) : 0u;
        qhb[i] = vb ? ldg_u32_a2(bb + 128 + 16 * i + 4 * t) : 0u;
        sca[i] = va ? ldg_u32_a2(ba + 192 + 4 * i) : 0u;
        scb[i] = vb ? ldg_u32_a2(bb + 192 + 4 * i) : 0u;
      }
      if (va) da = f16_bits_to_f32(ldg_u16(ba + 208));
      if (vb) db = f16_bits_to_f32(ldg_u16(bb + 208));

      q6_superblock(acc, qla, qlb, qha, qhb, sca, scb, da, db, xrow + sb * 256, dx, nb32, sb, t);
    }
    // ---- fixed-order reduction over warps
    float* rb_ = red + parity * (kQ6Warps * 32 * 4);
    reinterpret_cast<float4*>(rb_)[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (threadIdx.x < kQ6TileRows * kQ6MaxRows) {
      const int rr = threadIdx.x % kQ6TileRows, cc = threadIdx.x / kQ6TileRows;
      const int row = tile * kQ6TileRows + rr;
      if (cc < p.rows && row < p.n) {
        const int gg = rr & 7, up = rr >> 3;
        const int ln = gg * 4 + (cc >> 1), comp = up * 2 + (cc & 1);
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < kQ6Warps; ++ww) sum = __fadd_rn(sum, rb_[(ww * 32 + ln) * 4 + comp]);
        p.out[(int64_t)cc * p.ldc + row] = f32_to_bf16_bits(sum);
      }
    }
    parity ^= 1;
  }
}

// ---------------------------------------------------------------------------------------
// Streamed variant: the weight reaches shared memory through 1-D bulk copies (TMA) of 8-row
// stages.  8 rows of Q6_K are 8 * 210 * (k / 256) = 1680 * (k / 256) bytes, a multiple of 16,
// so every full stage starts and ends 16-byte aligned for any k; a ragged last stage copies
// its 16-byte-multiple prefix in bulk and its last few bytes with plain loads.  A 16-row MMA
// tile is two consecutive stages; the ring holds NS >= 3 stages, so the next tile is in
// flight while this one is computed.  Each lane reads its bytes from shared memory as aligned
// 32-bit pairs joined by a funnel shift (super-blocks are only 2-byte aligned).  The
// arithmetic, its order and the warp split are those of q6k_mmvq_kernel, so the two give the
// same bits.
constexpr int kQ6StageRows = 8;
constexpr int kQ6MaxStages = 6;
static __device__ int q6_fault_word = 0;

__device__ __forceinline__ uint32_t lds_u32_a2(uint32_t saddr) {  // 2-byte aligned 32-bit load
  const uint32_t a = saddr & ~3u;
  uint32_t w0, w1;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w0) : "r"(a));
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w1) : "r"(a + 4));
  return __funnelshift_r(w0, w1, (saddr & 3u) * 8u);
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t saddr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(saddr));
  return v;
}

struct Q6StreamParams {
  Q6Params q;
  int ns;             // ring stages
  int stage_stride;   // bytes per stage slot (>= 8 rows, multiple of 128)
  int ring_offset;    // byte offset of the ring in dynamic shared memory
};

__global__ void __launch_bounds__(kQ6Threads, 1) q6k_stream_kernel(const Q6StreamParams sp) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_dependents_launch();
  grid_dependency_wait();  // launched early (programmatic): q8, blocks and out follow the preceding kernel
  __shared__ __align__(8) uint64_t full[kQ6MaxStages];
  const Q6Params& p = sp.q;
  const int nsb = p.k / 256;
  const int nb32 = p.k / 32;
  const int rs = q6_row_stride(p.k);
  const int64_t row_bytes = (int64_t)nsb * 210;
  int8_t* xs = reinterpret_cast<int8_t*>(smem);                              // [8][rs]
  float* dx = reinterpret_cast<float*>(smem + kQ6MaxRows * rs);              // [8][nb32]
  float* red = dx + kQ6MaxRows * nb32;                                       // [2][16 warps][32 lanes][4]
  const uint32_t ring = smem_u32(smem + sp.ring_offset);
  const uint32_t full0 = smem_u32(full);

  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  const int nstages = 2 * (T1 - T0);

  // Stage s of this CTA: rows [16 (T0 + s/2) + 8 (s%2), +8) clipped to n, into slot s % NS.
  auto produce = [&](int s) {
    const int slot = s % sp.ns;
    const int64_t r0 = (int64_t)(T0 + s / 2) * kQ6TileRows + (s % 2) * kQ6StageRows;
    const int64_t nr = r0 >= p.n ? 0 : (p.n - r0 < kQ6StageRows ? p.n - r0 : kQ6StageRows);
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

  if (threadIdx.x == 0) {
    for (int i = 0; i < sp.ns; ++i) umma::bar_init(full0 + 8u * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int s = 0; s < sp.ns && s < nstages; ++s) produce(s);
  }

  // ---- stage the q8_1 rows (while the first weight stages are in flight)
  for (int it = threadIdx.x; it < kQ6MaxRows * nb32; it += kQ6Threads) {
    const int m = it / nb32, b = it % nb32;
    uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float d = 0.f;
    if (m < p.rows) {
      const uint8_t* blk = p.q8 + ((int64_t)m * nb32 + b) * 36;
      const uint32_t* bw = reinterpret_cast<const uint32_t*>(blk);
      d = f16_bits_to_f32(bw[0] & 0xffff);
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = bw[1 + i];
    }
    dx[m * nb32 + b] = d;
    uint4* dst = reinterpret_cast<uint4*>(xs + m * rs + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int sb_begin = q6_slice_begin(nsb, warp), sb_end = q6_slice_begin(nsb, warp + 1);
  const int8_t* xrow = xs + g * rs;  // B column g
  int parity = 0;

  for (int i = 0; T0 + i < T1; ++i) {
    const int tile = T0 + i;
    const int sa = 2 * i, sb2 = 2 * i + 1;
    const bool oka = umma::wait(full0 + 8u * (sa % sp.ns), (sa / sp.ns) & 1);
    const bool okb = umma::wait(full0 + 8u * (sb2 % sp.ns), (sb2 / sp.ns) & 1);
    if (!(oka && okb)) atomicOr(&q6_fault_word, 1);
    const uint32_t base_a = ring + (uint32_t)(sa % sp.ns) * sp.stage_stride + (uint32_t)(g * row_bytes);
    const uint32_t base_b = ring + (uint32_t)(sb2 % sp.ns) * sp.stage_stride + (uint32_t)(g * row_bytes);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int r0 = tile * kQ6TileRows + g;
    const bool va = r0 < p.n, vb = r0 + 8 < p.n;
    for (int sb = sb_begin; sb < sb_end; ++sb) {
      const uint32_t ba = base_a + (uint32_t)sb * 210u;
      const uint32_t bb = base_b + (uint32_t)sb * 210u;
      uint32_t qla[8], qlb[8], qha[4], qhb[4], sca[4], scb[4];
      float da = 0.f, db = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // ql bytes 16q + 4t
        qla[q] = va ? lds_u32_a2(ba + 16 * q + 4 * t) : 0u;
        qlb[q] = vb ? lds_u32_a2(bb + 16 * q + 4 * t) : 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // qh bytes 128 + 16q + 4t, scales 192 + 4q
        qha[q] = va ? lds_u32_a2(ba + 128 + 16 * q + 4 * t) : 0u;
        qhb[q] = vb ? lds_u32_a2(bb + 128 + 16 * q + 4 * t) : 0u;
        sca[q] = va ? lds_u32_a2(ba + 192 + 4 * q) : 0u;
        scb[q] = vb ? lds_u32_a2(bb + 192 + 4 * q) : 0u;
      }
      if (va) da = f16_bits_to_f32(lds_u16(ba + 208));
      if (vb) db = f16_bits_to_f32(lds_u16(bb + 208));

      q6_superblock(acc, qla, qlb, qha, qhb, sca, scb, da, db, xrow + sb * 256, dx, nb32, sb, t);
    }
    // ---- fixed-order reduction over warps; after its barrier the tile's stages are free
    float* rb_ = red + parity * (kQ6Warps * 32 * 4);
    reinterpret_cast<float4*>(rb_)[warp * 32 + lane] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (threadIdx.x == 0) {
      if (sa + sp.ns < nstages) produce(sa + sp.ns);
      if (sb2 + sp.ns < nstages) produce(sb2 + sp.ns);
    }
    if (threadIdx.x < kQ6TileRows * kQ6MaxRows) {
      const int rr = threadIdx.x % kQ6TileRows, cc = threadIdx.x / kQ6TileRows;
      const int row = tile * kQ6TileRows + rr;
      if (cc < p.rows && row < p.n) {
        const int gg = rr & 7, up = rr >> 3;
        const int ln = gg * 4 + (cc >> 1), comp = up * 2 + (cc & 1);
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < kQ6Warps; ++ww) sum = __fadd_rn(sum, rb_[(ww * 32 + ln) * 4 + comp]);
        p.out[(int64_t)cc * p.ldc + row] = f32_to_bf16_bits(sum);
      }
    }
    parity ^= 1;
  }
}

// ---------------------------------------------------------------------------------------
// Wide variant: 9..64 q8_1 rows in one weight pass.  Whole activation rows no longer fit in
// shared memory (64 rows of codes at K = 7168 take 458 KB), so the loop order is turned
// around: a CTA takes its 16-row weight tiles in row-blocks of up to kQWWarps tiles, one tile
// per consumer warp, and the row-block walks K one super-block at a time.
//   - Activations: a producer warp copies each super-block's q8_1 blocks of every activation
//     row (288 contiguous bytes per row) into a ring shared by the row-block's warps, with
//     16-byte cp.async and one mbarrier arrival per lane; the activations are re-read (from
//     L2) once per row-block, not once per tile.
//   - Weights: every consumer warp streams its own tile through a private ring of kQWDepth
//     stages with 16-byte cp.async (Ampere-style multistage pipeline, no registers held):
//     per row the 16-byte aligned span that covers the super-block's 210 bytes (at most 224;
//     super-blocks are only 2-byte aligned), read back at the span's offset with
//     funnel-shifted 32-bit shared loads.  The buffer's last bytes past its last 16-byte
//     boundary are stored with plain loads, so no copy reads past the weight buffer.
// Each consumer warp runs NT 8-column MMAs per sub-block on one decoded A fragment.
// The per-output arithmetic and its order are those of the 8-row kernels: K is cut into the
// same 16 slices (q6_slice_begin), each slice is accumulated alone from 0 with the same
// per-block step, and the slices are added to 0 in order -- so a row's bits do not depend on
// which kernel, or how many rows, served it.
// 15 consumer warps + 1 producer: 16 warps, 4 per SM sub-partition, so 128 registers a thread
constexpr int kQWWarps = 15;
constexpr int kQWThreads = (kQWWarps + 1) * 32;
constexpr int kQWRowBytes = 288;   // one super-block of one q8_1 row: 8 blocks
constexpr int kQWRowStride = 304;  // 76 words: the 8 B-fragment rows hit 32 banks
constexpr int kQWSpan = 240;       // staged bytes per weight row and super-block (>= 224)
constexpr int kQWTileBytes = kQ6TileRows * kQWSpan;
constexpr int kQWMaxActStages = 4;

struct Q6WideParams {
  Q6Params q;
  int act_stages;  // activation ring stages of NT * 8 * kQWRowStride bytes
  int depth;       // weight stages per consumer warp (>= 2)
};

__device__ __forceinline__ uint32_t lds_u32(uint32_t saddr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(saddr));
  return v;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
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
// `xs` (row stride kQWRowStride, block b of row m at m * stride + 36 b: f16 d, f16 s, 32 codes).
// Per (row, column) the same integer and float steps, in the same order, as q6_superblock.
template <int NT>
__device__ __forceinline__ void q6_superblock_wide(float (&acc)[NT][4], const uint32_t (&qla)[8],
                                                   const uint32_t (&qlb)[8], const uint32_t (&qha)[4],
                                                   const uint32_t (&qhb)[4], const uint32_t (&sca)[4],
                                                   const uint32_t (&scb)[4], float da, float db, uint32_t xs, int g,
                                                   int t) {
#pragma unroll
  for (int blk = 0; blk < 8; ++blk) {  // unrolled: the fragment arrays stay in registers
    uint32_t a0[2], a1[2];
    int ra[2], rb[2];
#pragma unroll
    for (int hj = 0; hj < 2; ++hj) {
      const int j = 2 * blk + hj;
      const int h = j >> 3, u = (j & 7) >> 1;
      const int qi = 4 * h + 2 * (u & 1) + (j & 1);
      const int hi = 2 * h + (j & 1);
      const int nsh = (u >> 1) * 4, hsh = 2 * u;
      a0[hj] = q6_to_s8x4(((qla[qi] >> nsh) & 0x0f0f0f0fu) | (((qha[hi] >> hsh) & 0x03030303u) << 4));
      a1[hj] = q6_to_s8x4(((qlb[qi] >> nsh) & 0x0f0f0f0fu) | (((qhb[hi] >> hsh) & 0x03030303u) << 4));
      const int sha = 24 - 8 * (j & 3);
      ra[hj] = (int)(sca[j >> 2] << sha) >> 24;
      rb[hj] = (int)(scb[j >> 2] << sha) >> 24;
    }
#pragma unroll
    for (int ct = 0; ct < NT; ++ct) {
      const uint32_t brow = xs + (uint32_t)((8 * ct + g) * kQWRowStride + 36 * blk + 4 + 4 * t);
      int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
      mma_s8_16816(d0, a0[0], a1[0], lds_u32(brow));
      mma_s8_16816(d1, a0[1], a1[1], lds_u32(brow + 16));
      const int is0 = d0[0] * ra[0] + d1[0] * ra[1];
      const int is1 = d0[1] * ra[0] + d1[1] * ra[1];
      const int is2 = d0[2] * rb[0] + d1[2] * rb[1];
      const int is3 = d0[3] * rb[0] + d1[3] * rb[1];
      const uint32_t drow = xs + (uint32_t)((8 * ct + 2 * t) * kQWRowStride + 36 * blk);
      const float dx0 = f16_bits_to_f32(lds_u16(drow));
      const float dx1 = f16_bits_to_f32(lds_u16(drow + kQWRowStride));
      acc[ct][0] = q6_block_step(acc[ct][0], is0, da, dx0);
      acc[ct][1] = q6_block_step(acc[ct][1], is1, da, dx1);
      acc[ct][2] = q6_block_step(acc[ct][2], is2, db, dx0);
      acc[ct][3] = q6_block_step(acc[ct][3], is3, db, dx1);
    }
  }
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
__global__ void __launch_bounds__(kQWThreads, 1) q6k_wide_kernel(const Q6WideParams wp) {
  extern __shared__ __align__(128) uint8_t smem[];
  grid_dependents_launch();
  grid_dependency_wait();  // launched early (programmatic): q8, blocks and out follow the preceding kernel
  __shared__ __align__(8) uint64_t full[kQWMaxActStages], empty[kQWMaxActStages];
  const Q6Params& p = wp.q;
  const int nsb = p.k / 256;
  const int nb32 = p.k / 32;
  const int64_t row_bytes = (int64_t)nsb * 210;
  const uintptr_t buf_end = reinterpret_cast<uintptr_t>(p.blocks) + (uintptr_t)((int64_t)p.n * row_bytes);
  constexpr int kRows = NT * 8;
  constexpr uint32_t kActBytes = kRows * kQWRowStride;
  const int ns = wp.act_stages, depth = wp.depth;
  const uint32_t act_ring = smem_u32(smem);
  const uint32_t w_rings = act_ring + (uint32_t)ns * kActBytes;
  const uint32_t full0 = smem_u32(full), empty0 = smem_u32(empty);

  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  const int nt = T1 - T0;
  const int nrb = (nt + kQWWarps - 1) / kQWWarps;  // row-blocks, as even as possible
  const int nchunks = nrb * nsb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // padding activation rows [rows, kRows) of every stage stay zero (never copied)
  for (int i = threadIdx.x; i < ns * (int)(kActBytes / 4); i += blockDim.x) {
    const int w = i % (int)(kActBytes / 4);
    if (w / (kQWRowStride / 4) >= p.rows) reinterpret_cast<uint32_t*>(smem)[i] = 0u;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < ns; ++i) {
      umma::bar_init(full0 + 8u * i, 32);  // one arrival per producer lane, when its copies land
      umma::bar_init(empty0 + 8u * i, kQWWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kQWWarps) {
    // ---------------- producer: chunk c = (row-block c / nsb, super-block c % nsb)
    constexpr int kPieces = kQWRowBytes / 16;
    for (int c = 0; c < nchunks; ++c) {
      const int slot = c % ns, sb = c % nsb;
      if (c >= ns && !umma::wait(empty0 + 8u * slot, ((c / ns) - 1) & 1)) atomicOr(&q6_fault_word, 4);
      __syncwarp();
      const uint32_t st = act_ring + (uint32_t)slot * kActBytes;
      for (int q = lane; q < p.rows * kPieces; q += 32) {
        const int m = q / kPieces, piece = q % kPieces;
        cp_async16(st + (uint32_t)(m * kQWRowStride + 16 * piece),
                   p.q8 + ((int64_t)m * nb32 + 8 * sb) * 36 + 16 * piece);
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
        uint32_t qla[8], qlb[8], qha[4], qhb[4], sca[4], scb[4];
        float da = 0.f, db = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          qla[q] = va ? lds_u32_a2(ba + 16 * q + 4 * t) : 0u;
          qlb[q] = vb ? lds_u32_a2(bb + 16 * q + 4 * t) : 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          qha[q] = va ? lds_u32_a2(ba + 128 + 16 * q + 4 * t) : 0u;
          qhb[q] = vb ? lds_u32_a2(bb + 128 + 16 * q + 4 * t) : 0u;
          sca[q] = va ? lds_u32_a2(ba + 192 + 4 * q) : 0u;
          scb[q] = vb ? lds_u32_a2(bb + 192 + 4 * q) : 0u;
        }
        if (va) da = f16_bits_to_f32(lds_u16(ba + 208));
        if (vb) db = f16_bits_to_f32(lds_u16(bb + 208));
        q6_superblock_wide<NT>(sl, qla, qlb, qha, qhb, sca, scb, da, db, st, g, t);
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

size_t q6k_smem_bytes(int k) {
  int rs = k + ((16 - k % 128) + 128) % 128;
  return (size_t)kQ6MaxRows * rs + (size_t)kQ6MaxRows * (k / 32) * 4 + 2ull * kQ6Warps * 32 * 4 * 4;
}

}  // namespace

namespace {

template <int NT>
int launch_wide(const Q6Params& p, int sms, int smem_optin, cudaStream_t s) {
  const size_t act = (size_t)NT * 8 * kQWRowStride;
  const size_t limit = (size_t)smem_optin > 1024 ? (size_t)smem_optin - 1024 : 0;  // static smem < 1 KB
  // three weight stages per warp when they fit beside at least two activation stages
  int depth = 3;
  if ((size_t)kQWWarps * depth * kQWTileBytes + 2 * act > limit) depth = 2;
  const size_t wbytes = (size_t)kQWWarps * depth * kQWTileBytes;
  if (wbytes + 2 * act > limit) return DLMH_ERR_UNSUPPORTED;
  int ns = (int)((limit - wbytes) / act);
  if (ns > kQWMaxActStages) ns = kQWMaxActStages;
  const size_t smem = (size_t)ns * act + wbytes;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(q6k_wide_kernel<NT>), (int)smem) != DLMH_OK)
    return DLMH_ERR_CUDA;
  const int ntiles = (p.n + kQ6TileRows - 1) / kQ6TileRows;
  const int grid = ntiles < sms ? ntiles : sms;
  return umma::launch_pdl(q6k_wide_kernel<NT>, dim3(grid), dim3(kQWThreads), smem, s, Q6WideParams{p, ns, depth});
}

}  // namespace

int q6k_wide_rows(int rows) { return rows <= 8 ? 8 : rows <= 16 ? 16 : rows <= 32 ? 32 : 64; }

int q6k_mmvq_launch(const uint8_t* blocks, int n, int k, const uint8_t* q8, int rows, uint16_t* out, int64_t ldc,
                    cudaStream_t s) {
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  if (rows > kQ6MaxRows) {  // 9..64 rows: one pass of the wide kernel (16-byte aligned blocks, q8_1 rows)
    if (rows > 64) return DLMH_ERR_ROWS;
    if ((reinterpret_cast<uintptr_t>(q8) & 15u) || (reinterpret_cast<uintptr_t>(blocks) & 15u)) return DLMH_ERR_ALIGN;
    const Q6Params p{blocks, n, k, q8, rows, out, ldc};
    switch (q6k_wide_rows(rows)) {
      case 16: return launch_wide<2>(p, di.sms, di.smem_optin, s);
      case 32: return launch_wide<4>(p, di.sms, di.smem_optin, s);
      default: return launch_wide<8>(p, di.sms, di.smem_optin, s);
    }
  }
  const size_t base_smem = q6k_smem_bytes(k);
  Q6Params p{blocks, n, k, q8, rows, out, ldc};
  const int ntiles = (n + kQ6TileRows - 1) / kQ6TileRows;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  // streamed variant when the ring holds at least three 8-row stages and the blocks start
  // 16-byte aligned (then every 8-row stage does); both variants give the same bits
  const size_t ring_offset = (base_smem + 127) / 128 * 128;
  const size_t stage_stride = ((size_t)kQ6StageRows * (k / 256) * 210 + 127) / 128 * 128;
  const size_t limit = (size_t)di.smem_optin > 2048 ? (size_t)di.smem_optin - 2048 : 0;
  int ns = limit > ring_offset ? (int)((limit - ring_offset) / stage_stride) : 0;
  if (ns > kQ6MaxStages) ns = kQ6MaxStages;
  if (ns >= 3 && (reinterpret_cast<uintptr_t>(blocks) & 15u) == 0) {
    const size_t smem = ring_offset + (size_t)ns * stage_stride;
    if (ensure_dynamic_smem(reinterpret_cast<const void*>(q6k_stream_kernel), (int)smem) != DLMH_OK)
      return DLMH_ERR_CUDA;
    Q6StreamParams sp{p, ns, (int)stage_stride, (int)ring_offset};
    return umma::launch_pdl(q6k_stream_kernel, dim3(grid), dim3(kQ6Threads), smem, s, sp);
  }
  if (base_smem + 1024 > (size_t)di.smem_optin) return DLMH_ERR_UNSUPPORTED;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(q6k_mmvq_kernel), (int)base_smem) != DLMH_OK)
    return DLMH_ERR_CUDA;
  return umma::launch_pdl(q6k_mmvq_kernel, dim3(grid), dim3(kQ6Threads), base_smem, s, p);
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
