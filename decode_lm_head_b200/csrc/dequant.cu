// Load-time FP4 dequant to BF16 (the step before the path; fp8_lut.rs):
//   - NVFP4:  out[n, k] = bf16( f32( e2m1(W[n, k]) * e4m3(S[n, k/16]) ) * g )   (g folded global)
//   - E8M0:   out[f]    = bf16( e2m1(W[f]) * 2^(e[f / block] - 127) )          (flat index f)
// Float32 arithmetic: the E2M1 x E4M3 product is exact (at most 6 significant bits), the
// product with g is one float32 rounding, the cast to BF16 rounds to nearest-even; the E8M0
// product is exact unless it leaves the float32 range.  Each thread converts 16 consecutive
// elements of a row: one 8-byte load of codes, one scale, two 16-byte stores, so loads and
// stores are coalesced across the warp and the kernel is a plain HBM stream.
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

// Index type: 32-bit when every chunk index fits (the usual case), 64-bit otherwise.
template <typename I>
__global__ void __launch_bounds__(kDqThreads) nvfp4_dequant_kernel(const uint8_t* __restrict__ packed,
                                                                   const uint8_t* __restrict__ bscale, float g,
                                                                   int n, int k, uint16_t* __restrict__ out,
                                                                   int64_t ldo) {
  const I per_row = k / 16;
  const I chunks = (I)n * per_row;
  const I stride = (I)gridDim.x * blockDim.x;
  // two chunks per iteration, both loads issued before either is converted
  for (I c = (I)blockIdx.x * blockDim.x + threadIdx.x; c < chunks; c += 2 * stride) {
    const I c1 = c + stride;
    const bool has1 = c1 < chunks;
    const I row0 = c / per_row, cb0 = c - row0 * per_row;
    const I row1 = has1 ? c1 / per_row : 0, cb1 = has1 ? c1 - row1 * per_row : 0;
    const uint2 pk0 = *reinterpret_cast<const uint2*>(packed + (int64_t)c * 8);
    const uint8_t s0 = bscale[c];
    uint2 pk1 = make_uint2(0, 0);
    uint8_t s1 = 0;
    if (has1) {
      pk1 = *reinterpret_cast<const uint2*>(packed + (int64_t)c1 * 8);
      s1 = bscale[c1];
    }
    uint32_t lo[4], hi[4];
    const float sc0 = f16_bits_to_f32(e4m3x2_to_f16x2((uint16_t)s0) & 0xffffu);
    fp4x8_to_bf16<true>(pk0.x, sc0, g, lo);
    fp4x8_to_bf16<true>(pk0.y, sc0, g, hi);
    uint4* dst = reinterpret_cast<uint4*>(out + (int64_t)row0 * ldo + (int64_t)cb0 * 16);
    dst[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    dst[1] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    if (has1) {
      const float sc1 = f16_bits_to_f32(e4m3x2_to_f16x2((uint16_t)s1) & 0xffffu);
      fp4x8_to_bf16<true>(pk1.x, sc1, g, lo);
      fp4x8_to_bf16<true>(pk1.y, sc1, g, hi);
      dst = reinterpret_cast<uint4*>(out + (int64_t)row1 * ldo + (int64_t)cb1 * 16);
      dst[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      dst[1] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
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

int grid_for(int64_t chunks) {
  const DeviceInfo di = device_info();
  const int64_t want = (chunks + kDqThreads - 1) / kDqThreads;
  const int64_t cap = (int64_t)(di.sms > 0 ? di.sms : 148) * 16;
  return (int)(want < cap ? want : cap);
}

}  // namespace

int nvfp4_dequant_launch(const uint8_t* packed, const uint8_t* bscale, float g, int n, int k, uint16_t* out,
                         int64_t ldo, cudaStream_t s) {
  const int64_t chunks = (int64_t)n * (k / 16);
  if (chunks == 0) return DLMH_OK;
  if (chunks * 16 < ((int64_t)1 << 31))
    nvfp4_dequant_kernel<int32_t><<<grid_for(chunks), kDqThreads, 0, s>>>(packed, bscale, g, n, k, out, ldo);
  else
    nvfp4_dequant_kernel<int64_t><<<grid_for(chunks), kDqThreads, 0, s>>>(packed, bscale, g, n, k, out, ldo);
  return launch_status();
}

int e8m0_dequant_launch(const uint8_t* packed, const uint8_t* scales, int64_t block, int n, int k, uint16_t* out,
                        int64_t ldo, cudaStream_t s) {
  const int64_t chunks = (int64_t)n * k / 16;
  if (chunks == 0) return DLMH_OK;
  if (chunks * 16 < ((int64_t)1 << 31))
    e8m0_dequant_kernel<int32_t><<<grid_for(chunks), kDqThreads, 0, s>>>(packed, scales, block, n, k, out, ldo);
  else
    e8m0_dequant_kernel<int64_t><<<grid_for(chunks), kDqThreads, 0, s>>>(packed, scales, block, n, k, out, ldo);
  return launch_status();
}

}  // namespace dlmh
