// Q6_K super-blocks x block_q8_1 rows on int8 warp MMAs.
//
// Same decomposition as the row-tile GEMV: one persistent 512-thread CTA per SM over
// 16-row weight tiles, the super-blocks of a tile split across 16 warps, a fixed-order
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
  const int nsbw = (nsb + kQ6Warps - 1) / kQ6Warps;
  const int64_t row_bytes = (int64_t)nsb * 210;
  const int8_t* xrow = xs + g * rs;  // B column g
  int parity = 0;

  for (int tile = T0; tile < T1; ++tile) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const int r0 = tile * kQ6TileRows + g;
    const bool va = r0 < p.n, vb = r0 + 8 < p.n;
    for (int s = 0; s < nsbw; ++s) {
      const int sb = warp * nsbw + s;
      if (sb >= nsb) break;
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

      const int8_t* xsb = xrow + sb * 256;
#pragma unroll
      for (int blk = 0; blk < 8; ++blk) {  // q8_1 block = sub-blocks 2blk, 2blk+1
        float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hj = 0; hj < 2; ++hj) {
          const int j = 2 * blk + hj;
          const int h = j >> 3, u = (j & 7) >> 1;
          // ql word index: 64h + 32(u&1) + 16(j&1) -> i = 4h + 2(u&1) + (j&1)
          const int qi = 4 * h + 2 * (u & 1) + (j & 1);
          const int hi = 2 * h + (j & 1);  // qh: 32h + 16(j&1)
          const int nsh = (u >> 1) * 4, hsh = 2 * u;
          const uint32_t qa = ((qla[qi] >> nsh) & 0x0f0f0f0fu) | (((qha[hi] >> hsh) & 0x03030303u) << 4);
          const uint32_t qb = ((qlb[qi] >> nsh) & 0x0f0f0f0fu) | (((qhb[hi] >> hsh) & 0x03030303u) << 4);
          const uint32_t bx = *reinterpret_cast<const uint32_t*>(xsb + 16 * j + 4 * t);
          int d4[4] = {0, 0, 0, 0};
          mma_s8_16816(d4, q6_to_s8x4(qa), q6_to_s8x4(qb), bx);
          const float ra = da * (float)(int8_t)((sca[j >> 2] >> (8 * (j & 3))) & 0xff);
          const float rb = db * (float)(int8_t)((scb[j >> 2] >> (8 * (j & 3))) & 0xff);
          part[0] += (float)d4[0] * ra;
          part[1] += (float)d4[1] * ra;
          part[2] += (float)d4[2] * rb;
          part[3] += (float)d4[3] * rb;
        }
        const int b32 = sb * 8 + blk;
        const float dx0 = dx[(2 * t) * nb32 + b32], dx1 = dx[(2 * t + 1) * nb32 + b32];
        acc[0] += part[0] * dx0;
        acc[1] += part[1] * dx1;
        acc[2] += part[2] * dx0;
        acc[3] += part[3] * dx1;
      }
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
        for (int ww = 0; ww < kQ6Warps; ++ww) sum += rb_[(ww * 32 + ln) * 4 + comp];
        p.out[(int64_t)cc * p.ldc + row] = f32_to_bf16_bits(sum);
      }
    }
    parity ^= 1;
  }
}

size_t q6k_smem_bytes(int k) {
  int rs = k + ((16 - k % 128) + 128) % 128;
  return (size_t)kQ6MaxRows * rs + (size_t)kQ6MaxRows * (k / 32) * 4 + 2ull * kQ6Warps * 32 * 4 * 4;
}

}  // namespace

int q6k_mmvq_launch(const uint8_t* blocks, int n, int k, const uint8_t* q8, int rows, uint16_t* out, int64_t ldc,
                    cudaStream_t s) {
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  const size_t smem = q6k_smem_bytes(k);
  if (smem + 1024 > (size_t)di.smem_optin) return DLMH_ERR_UNSUPPORTED;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(q6k_mmvq_kernel), (int)smem) != DLMH_OK) return DLMH_ERR_CUDA;
  Q6Params p{blocks, n, k, q8, rows, out, ldc};
  const int ntiles = (n + kQ6TileRows - 1) / kQ6TileRows;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  q6k_mmvq_kernel<<<grid, kQ6Threads, smem, s>>>(p);
  return launch_status();
}

}  // namespace dlmh
