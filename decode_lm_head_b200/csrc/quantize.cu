// Activation quantize kernels: per-row dynamic E4M3 (W8A8), the fused SiLU variant, and
// block_q8_1 rows (Q6_K path).  Bytes are tiny next to the weight pass; these kernels aim
// for exact agreement with the definitions, not for bandwidth.
#include "dlmh_common.cuh"
#include "gemv_launch.h"

namespace dlmh {
namespace {

constexpr int kQThreads = 256;

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
    v = warp_max(v);
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  v = red[0];
  __syncthreads();
  return v;
}

// h = bf16(silu(g) * u): silu in f32 as g / (1 + e^-g) with an IEEE division, one product,
// one rounding to BF16.
__device__ __forceinline__ float silu_mul_bf16(float g, float u) {
  const float s = __fdiv_rn(g, 1.0f + expf(-g));
  return bf16_bits_to_f32(f32_to_bf16_bits(s * u));
}

// Quantize one row held as f32 values produced by `getv(k)` (k multiple of 16 groups).
template <class GetV>
__device__ void quantize_row(GetV getv, int k, uint8_t* q, float* sx_out, float* red) {
  float amax = 0.f;
  for (int k0 = threadIdx.x * 16; k0 < k; k0 += kQThreads * 16) {
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(getv(k0 + i)));
  }
  amax = block_max(amax, red);
  const float sx = __fdiv_rn(amax, 448.0f);
  if (threadIdx.x == 0) *sx_out = sx;
  for (int k0 = threadIdx.x * 16; k0 < k; k0 += kQThreads * 16) {
    uint32_t wv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t c0 = 0, c1 = 0;
      if (sx != 0.f) {
        c0 = f32x2_to_e4m3x2(__fdiv_rn(getv(k0 + 4 * i + 0), sx), __fdiv_rn(getv(k0 + 4 * i + 1), sx));
        c1 = f32x2_to_e4m3x2(__fdiv_rn(getv(k0 + 4 * i + 2), sx), __fdiv_rn(getv(k0 + 4 * i + 3), sx));
      }
      wv[i] = c0 | (c1 << 16);
    }
    *reinterpret_cast<uint4*>(q + k0) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
  }
}

__global__ void __launch_bounds__(kQThreads) w8a8_quantize_kernel(const uint16_t* __restrict__ x, int64_t ldx, int k,
                                                                  uint8_t* __restrict__ xq, int64_t ldq,
                                                                  float* __restrict__ sx) {
  __shared__ float red[32];
  grid_dependents_launch();  // a following tensor-core GEMV may start its weight loads
  const int m = blockIdx.x;
  const uint16_t* xr = x + (int64_t)m * ldx;
  quantize_row([&](int i) { return bf16_bits_to_f32(xr[i]); }, k, xq + (int64_t)m * ldq, sx + m, red);
}

// One CTA per row; the BF16 SiLU products of the row are kept in shared memory between the
// max pass and the quantize pass.
__global__ void __launch_bounds__(kQThreads) w8a8_silu_quantize_kernel(const uint16_t* __restrict__ gate,
                                                                       const uint16_t* __restrict__ up, int64_t ld,
                                                                       int k, uint8_t* __restrict__ xq, int64_t ldq,
                                                                       float* __restrict__ sx) {
  extern __shared__ __align__(16) float hbuf[];  // k floats (BF16-exact values)
  __shared__ float red[32];
  grid_dependents_launch();  // a following tensor-core GEMV may start its weight loads
  const int m = blockIdx.x;
  const uint16_t* gr = gate + (int64_t)m * ld;
  const uint16_t* ur = up + (int64_t)m * ld;
  for (int i = threadIdx.x; i < k; i += kQThreads)
    hbuf[i] = silu_mul_bf16(bf16_bits_to_f32(gr[i]), bf16_bits_to_f32(ur[i]));
  __syncthreads();
  quantize_row([&](int i) { return hbuf[i]; }, k, xq + (int64_t)m * ldq, sx + m, red);
}

// block_q8_1: one warp per 32-value block.  Layout {f16 d; f16 s; int8 qs[32]}.
__global__ void __launch_bounds__(kQThreads) q8_1_quantize_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                                  int rows, int k, uint8_t* __restrict__ q8) {
  const int nb = k / 32;
  const int64_t blk = (int64_t)blockIdx.x * (kQThreads / 32) + (threadIdx.x >> 5);
  if (blk >= (int64_t)rows * nb) return;
  const int lane = threadIdx.x & 31;
  const int m = (int)(blk / nb), b = (int)(blk % nb);
  const float v = bf16_bits_to_f32(x[(int64_t)m * ldx + b * 32 + lane]);
  const float amax = warp_max(fabsf(v));
  const float d = __fdiv_rn(amax, 127.0f);
  int q = 0;
  if (d != 0.f) q = (int)roundf(__fdiv_rn(v, d));  // roundf: half away from zero
  int sum = q;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  uint8_t* out = q8 + blk * 36;
  out[4 + lane] = (uint8_t)(int8_t)q;
  if (lane == 0) {
    const uint16_t dbits = f32_to_f16_bits(d);
    const uint16_t sbits = f32_to_f16_bits(__fmul_rn(d, (float)sum));
    *reinterpret_cast<uint32_t*>(out) = (uint32_t)dbits | ((uint32_t)sbits << 16);
  }
}

}  // namespace

int w8a8_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* xq, int64_t ldq, float* sx,
                         cudaStream_t s) {
  w8a8_quantize_kernel<<<rows, kQThreads, 0, s>>>(x, ldx, k, xq, ldq, sx);
  return launch_status();
}

int w8a8_silu_quantize_launch(const uint16_t* gate, const uint16_t* up, int64_t ld, int rows, int k, uint8_t* xq,
                              int64_t ldq, float* sx, cudaStream_t s) {
  const size_t smem = (size_t)k * sizeof(float);
  if (smem > 200 * 1024) return DLMH_ERR_UNSUPPORTED;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(w8a8_silu_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return DLMH_ERR_CUDA;
  w8a8_silu_quantize_kernel<<<rows, kQThreads, smem, s>>>(gate, up, ld, k, xq, ldq, sx);
  return launch_status();
}

int q8_1_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* q8, cudaStream_t s) {
  const int64_t blocks = (int64_t)rows * (k / 32);
  const int64_t grid = (blocks + (kQThreads / 32) - 1) / (kQThreads / 32);
  q8_1_quantize_kernel<<<(unsigned)grid, kQThreads, 0, s>>>(x, ldx, rows, k, q8);
  return launch_status();
}

}  // namespace dlmh
