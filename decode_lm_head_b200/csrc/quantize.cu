// block_q8_1 row quantize (the Q6_K path).  Bytes are tiny next to the weight pass; this
// kernel aims for exact agreement with the definition.  The E4M3 pre-passes live in
// act_quant.cu.
#include "dlmh_common.cuh"
#include "gemv_launch.h"
#include "umma_common.cuh"

namespace dlmh {
namespace {

constexpr int kQThreads = 256;

// block_q8_1: one warp per 32-value block.  Layout {f16 d; f16 s; int8 qs[32]}.
__global__ void __launch_bounds__(kQThreads) q8_1_quantize_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                                  int rows, int k, uint8_t* __restrict__ q8) {
  grid_dependents_launch();  // the Q6_K GEMV may launch and set up now
  grid_dependency_wait();    // launched early (programmatic): x and q8 follow the preceding kernel
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

int q8_1_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* q8, cudaStream_t s) {
  const int64_t blocks = (int64_t)rows * (k / 32);
  const int64_t grid = (blocks + (kQThreads / 32) - 1) / (kQThreads / 32);
  return umma::launch_pdl(q8_1_quantize_kernel, dim3((unsigned)grid), dim3(kQThreads), 0, s, x, ldx, rows, k, q8);
}

}  // namespace dlmh
