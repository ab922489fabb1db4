// Load-time FP4 dequant to BF16 (the step before the path; fp8_lut.rs):
//   - NVFP4:  out[n, k] = bf16( f32( e2m1(W[n, k]) * e4m3(S[n, k/16]) ) * g )   (g folded global)
//   - E8M0:   out[f]    = bf16( e2m1(W[f]) * 2^(e[f / block] - 127) )          (flat index f)
// Float32 arithmetic: the E2M1 x E4M3 product is exact (at most 6 significant bits), the
// product with g is one float32 rounding, the cast to BF16 rounds to nearest-even; the E8M0
// product is exact unless it leaves the float32 range.  NVFP4: a lane converts 8-element
// groups, one 4-byte load of codes and one 16-byte store each, laid out so that every load and
// store instruction of a warp covers one contiguous run.  E8M0: each thread converts 16
// consecutive elements of a row (one 8-byte load, two 16-byte stores), which measured faster
// for it than the warp-span layout (33 against 39 us on 14336 x 4096).
#include "dlmh_common.cuh"
#include "gemv_launch.h"

namespace dlmh {
namespace {

constexpr int kDqThreads = 256;

// Eight E2M1 codes (one 32-bit word, element 2i in the low nibble of byte i) times `scale`,
// times `g` when kGlobal, rounded to four BF16 pairs.
template <bool kGlobal>
__device__ __forceinline__ void fp4x8_to_bf16(uint32_t word, float scale, float g, uint32_t (&o)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h = e2m1x2_to_f16x2((word >> (8 * i)) & 0xffu);  // exact
    float a = f16_bits_to_f32(h & 0xffffu) * scale;                  // exact
    float b = f16_bits_to_f32(h >> 16) * scale;
    if (kGlobal) {
      a *= g;
      b *= g;
    }
    o[i] = (uint32_t)f32_to_bf16_bits(a) | ((uint32_t)f32_to_bf16_bits(b) << 16);
  }
}

// Work split: a flat sequence of 8-element groups (rows are k/8 groups long, k % 16 == 0, so a
// group never crosses a row).  A warp takes kDqSpan consecutive groups per step, lane l the
// groups l, l + 32, ...: every code load (4 bytes a lane) and every 16-byte output store of
// the warp covers one contiguous run, and all of a lane's loads are issued before its first
// conversion.  Index type: 32-bit when every index fits, 64-bit otherwise.
constexpr int kDqPerLane = 4;
constexpr int kDqSpan = 32 * kDqPerLane;

template <typename I>
__global__ void __launch_bounds__(kDqThreads) nvfp4_dequant_kernel(const uint8_t* __restrict__ packed,
                                                                   const uint8_t* __restrict__ bscale, float g,
                                                                   int n, int k, uint16_t* __restrict__ out,
                                                                   int64_t ldo) {
  const I per_row = k / 8;
  const I groups = (I)n * per_row;
  const int lane = threadIdx.x & 31;
  const I warp0 = ((I)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const I nwarps = ((I)gridDim.x * blockDim.x) >> 5;
  for (I base = warp0 * kDqSpan; base < groups; base += nwarps * kDqSpan) {
    uint32_t w[kDqPerLane];
    uint32_t sb[kDqPerLane];
#pragma unroll
    for (int j = 0; j < kDqPerLane; ++j) {
      const I g8 = base + lane + 32 * j;
      const bool ok = g8 < groups;
      w[j] = ok ? __ldg(reinterpret_cast<const unsigned int*>(packed) + g8) : 0u;
      sb[j] = ok ? (uint32_t)__ldg(bscale + (g8 >> 1)) : 0u;  // one scale per 16 values
    }
#pragma unroll
    for (int j = 0; j < kDqPerLane; ++j) {
      const I g8 = base + lane + 32 * j;
      if (g8 < groups) {
        uint32_t o[4];
        const float sc = f16_bits_to_f32(e4m3x2_to_f16x2((uint16_t)sb[j]) & 0xffffu);
        fp4x8_to_bf16<true>(w[j], sc, g, o);
        const I row = g8 / per_row;
        *reinterpret_cast<uint4*>(out + (int64_t)row * ldo + (int64_t)(g8 - row * per_row) * 8) =
            make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
}

__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  return (e == 0 || e == 255) ? 0.f : __int_as_float((int)(e << 23));  // 2^(e - 127)
}

// One chunk of 16 flat elements starting at f0 (within one row since k % 16 == 0).
template <typename I>
__device__ __forceinline__ void e8m0_chunk(const uint2 pk, I f0, int64_t block, const uint8_t* __restrict__ scales,
                                           uint32_t (&o)[8]) {
  if (block % 16 == 0) {  // the whole chunk lies in one scale group
    const float scale = e8m0_to_f32(scales[f0 / (I)block]);
    fp4x8_to_bf16<false>(pk.x, scale, 1.f, *reinterpret_cast<uint32_t(*)[4]>(&o[0]));
    fp4x8_to_bf16<false>(pk.y, scale, 1.f, *reinterpret_cast<uint32_t(*)[4]>(&o[4]));
    return;
  }
  I grp = f0 / (I)block, next = (grp + 1) * (I)block;
  float scale = e8m0_to_f32(scales[grp]);
#pragma unroll
  for (int i = 0; i < 8; ++i) {  // elements 2i, 2i+1
    const uint32_t word = i < 4 ? pk.x : pk.y;
    const uint32_t h = e2m1x2_to_f16x2((word >> (8 * (i & 3))) & 0xffu);
    float v[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const I f = f0 + 2 * i + j;
      if (f >= next) {  // the chunk crosses into another scale group
        grp = f / (I)block;
        next = (grp + 1) * (I)block;
        scale = e8m0_to_f32(scales[grp]);
      }
      v[j] = f16_bits_to_f32(j ? (h >> 16) : (h & 0xffffu)) * scale;
    }
    o[i] = (uint32_t)f32_to_bf16_bits(v[0]) | ((uint32_t)f32_to_bf16_bits(v[1]) << 16);
  }
}

template <typename I>
__global__ void __launch_bounds__(kDqThreads) e8m0_dequant_kernel(const uint8_t* __restrict__ packed,
                                                                  const uint8_t* __restrict__ scales,
                                                                  int64_t block, int n, int k,
                                                                  uint16_t* __restrict__ out, int64_t ldo) {
  const I chunks = (I)((int64_t)n * k / 16);
  const I per_row = k / 16;
  const I stride = (I)gridDim.x * blockDim.x;
  for (I c = (I)blockIdx.x * blockDim.x + threadIdx.x; c < chunks; c += 2 * stride) {
    const I c1 = c + stride;
    const bool has1 = c1 < chunks;
    const uint2 pk0 = *reinterpret_cast<const uint2*>(packed + (int64_t)c * 8);
    const uint2 pk1 = has1 ? *reinterpret_cast<const uint2*>(packed + (int64_t)c1 * 8) : make_uint2(0, 0);
    uint32_t o[8];
    e8m0_chunk<I>(pk0, c * 16, block, scales, o);
    I row = c / per_row;
    uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)row * ldo + (int64_t)(c - row * per_row) * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    if (has1) {
      e8m0_chunk<I>(pk1, c1 * 16, block, scales, o);
      row = c1 / per_row;
      dst = reinterpret_cast<uint4*>(out + (int64_t)row * ldo + (int64_t)(c1 - row * per_row) * 16);
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

// Blocks for the E8M0 kernel's `chunks` 16-element chunks: one per thread, capped at 16 blocks
// per SM.
int grid_for_chunks(int64_t chunks) {
  const DeviceInfo di = device_info();
  const int64_t want = (chunks + kDqThreads - 1) / kDqThreads;
  const int64_t cap = (int64_t)(di.sms > 0 ? di.sms : 148) * 16;
  return (int)(want < cap ? want : cap);
}

// Blocks for `groups` 8-element groups: enough warps for one span each, at most 8 resident
// blocks per SM (2048 threads).
int grid_for(int64_t groups) {
  const DeviceInfo di = device_info();
  const int64_t warps = (groups + kDqSpan - 1) / kDqSpan;
  const int64_t want = (warps + kDqThreads / 32 - 1) / (kDqThreads / 32);
  const int64_t cap = (int64_t)(di.sms > 0 ? di.sms : 148) * 8;
  return (int)(want < cap ? want : cap);
}

}  // namespace

int nvfp4_dequant_launch(const uint8_t* packed, const uint8_t* bscale, float g, int n, int k, uint16_t* out,
                         int64_t ldo, cudaStream_t s) {
  const int64_t groups = (int64_t)n * (k / 8);
  if (groups == 0) return DLMH_OK;
  if (groups * 8 + (int64_t)kDqSpan * 8 * 148 * 8 < ((int64_t)1 << 31))
    nvfp4_dequant_kernel<int32_t><<<grid_for(groups), kDqThreads, 0, s>>>(packed, bscale, g, n, k, out, ldo);
  else
    nvfp4_dequant_kernel<int64_t><<<grid_for(groups), kDqThreads, 0, s>>>(packed, bscale, g, n, k, out, ldo);
  return launch_status();
}

int e8m0_dequant_launch(const uint8_t* packed, const uint8_t* scales, int64_t block, int n, int k, uint16_t* out,
                        int64_t ldo, cudaStream_t s) {
  const int64_t chunks = (int64_t)n * k / 16;
  if (chunks == 0) return DLMH_OK;
  if (chunks * 16 < ((int64_t)1 << 31))
    e8m0_dequant_kernel<int32_t><<<grid_for_chunks(chunks), kDqThreads, 0, s>>>(packed, scales, block, n, k, out, ldo);
  else
    e8m0_dequant_kernel<int64_t><<<grid_for_chunks(chunks), kDqThreads, 0, s>>>(packed, scales, block, n, k, out, ldo);
  return launch_status();
}

}  // namespace dlmh
