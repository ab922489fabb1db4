// Activation pre-passes of the E4M3 paths, one thread-block cluster per row:
//   - W8A8 per-row dynamic quantize:   sx = amax / 448, codes = e4m3_rn_sat(h / sx)
//     with h = x (plain) or h = bf16(silu(gate) * up) (the fused FFN-down variant);
//   - W8A16 two-term split:            x' = x * 2^e (max|x'| in [2^7, 2^8)),
//                                      hi = e4m3(x'), lo = e4m3(16 (x' - hi)).
// Each needs the row maximum before it can emit a code, and decode rows are few (1..128)
// while K is long (5120..14336), so one CTA per row leaves most of the GPU idle.  Here a
// cluster of kQC CTAs shares a row: every CTA takes a contiguous 1/kQC of the row's 8-element
// groups, keeps its values in registers, reduces its maximum, and the cluster combines the
// kQC maxima through distributed shared memory.  The arithmetic is the same as a one-CTA
// pass (correctly rounded f32 steps for silu(g)*u, round-to-nearest-even codes), so the
// codes do not depend on the split.
#include <utility>

#include "dlmh_common.cuh"
#include "gemv_launch.h"

namespace dlmh {
namespace {

constexpr int kQC = 8;       // CTAs per row (a portable cluster size)
constexpr int kQT = 256;     // threads per CTA
constexpr int kQCache = 4;   // 8-element groups a thread keeps in registers

enum class Src { Plain, Silu };

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// f32 at the same shared-memory variable of CTA `rank` of this cluster.
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// h = bf16(silu(g) * u) as BF16 bits, in f32 steps: e = e^-g correctly rounded to f32 (the
// double exp, below one double ulp, rounded once), d = 1 + e, s = g / d (IEEE division),
// p = s * u, then one round-to-nearest-even to BF16.  Every step is a correctly rounded f32
// operation, so h is a function of (g, u) alone and the codes that follow are reproducible.
__device__ __forceinline__ uint32_t silu_mul_bf16_bits(float g, float u) {
  const float e = __double2float_rn(exp(-(double)g));
  const float s = __fdiv_rn(g, __fadd_rn(1.0f, e));
  return f32_to_bf16_bits(__fmul_rn(s, u));
}

// The 8 BF16 values of group `g` of a row, packed two per word (element 2i low).
template <Src S>
__device__ __forceinline__ void load_group(const uint16_t* a, const uint16_t* b, int g, uint32_t (&h)[4]) {
  const uint4 va = ldg_nc(a + 8 * g);
  const uint32_t wa[4] = {va.x, va.y, va.z, va.w};
  if constexpr (S == Src::Plain) {
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = wa[i];
  } else {
    const uint4 vb = ldg_nc(b + 8 * g);
    const uint32_t wb[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = silu_mul_bf16_bits(bf16_bits_to_f32(wa[i] & 0xffffu), bf16_bits_to_f32(wb[i] & 0xffffu));
      const uint32_t hi = silu_mul_bf16_bits(bf16_bits_to_f32(wa[i] >> 16), bf16_bits_to_f32(wb[i] >> 16));
      h[i] = lo | (hi << 16);
    }
  }
}

__device__ __forceinline__ float group_amax(const uint32_t (&h)[4], float amax) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    amax = fmaxf(amax, fabsf(bf16_bits_to_f32(h[i] & 0xffffu)));
    amax = fmaxf(amax, fabsf(bf16_bits_to_f32(h[i] >> 16)));
  }
  return amax;
}

// Row maximum over the whole cluster.  Every CTA must call it (it holds cluster barriers);
// the caller ends with cluster_sync() so no CTA exits while another reads its shared memory.
__device__ float cluster_row_max(float v, float* red, float* cta_max) {
  v = warp_max(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int i = 1; i < kQT / 32; ++i) m = fmaxf(m, red[i]);
    *cta_max = m;
  }
  cluster_sync();  // every CTA's maximum is written
  if (warp == 0) {
    float m = lane < kQC ? ld_cluster_f32(cta_max, (uint32_t)lane) : 0.f;
    m = warp_max(m);
    if (lane == 0) red[0] = m;
  }
  __syncthreads();
  return red[0];
}

// Groups [g0, g1) of this CTA's share of a row with `ngroups` groups.
__device__ __forceinline__ void cta_range(int ngroups, int& g0, int& g1) {
  const int r = (int)cluster_rank();
  g0 = (int)((int64_t)r * ngroups / kQC);
  g1 = (int)((int64_t)(r + 1) * ngroups / kQC);
}

// W8A8 quantize of row blockIdx.y: codes xq[m, :] and scale sx[m].
template <Src S>
__global__ void __launch_bounds__(kQT) w8a8_quant_cluster_kernel(const uint16_t* __restrict__ a,
                                                                 const uint16_t* __restrict__ b, int64_t ld, int k,
                                                                 uint8_t* __restrict__ xq, int64_t ldq,
                                                                 float* __restrict__ sx) {
  __shared__ float red[kQT / 32];
  __shared__ float cta_max;
  grid_dependents_launch();  // a following tensor-core GEMV may start its weight loads
  grid_dependency_wait();    // launched early (programmatic): x and the outputs follow the preceding kernel
  const int m = blockIdx.y;
  const uint16_t* ar = a + (int64_t)m * ld;
  const uint16_t* br = S == Src::Silu ? b + (int64_t)m * ld : nullptr;
  int g0, g1;
  cta_range(k / 8, g0, g1);
  uint32_t h[kQCache][4];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < kQCache; ++c) {
    const int g = g0 + threadIdx.x + c * kQT;
    if (g < g1) {
      load_group<S>(ar, br, g, h[c]);
      amax = group_amax(h[c], amax);
    }
  }
  for (int g = g0 + threadIdx.x + kQCache * kQT; g < g1; g += kQT) {  // beyond the register cache
    uint32_t t[4];
    load_group<S>(ar, br, g, t);
    amax = group_amax(t, amax);
  }
  amax = cluster_row_max(amax, red, &cta_max);
  const float s = __fdiv_rn(amax, 448.0f);
  if (cluster_rank() == 0 && threadIdx.x == 0) sx[m] = s;
  uint8_t* q = xq + (int64_t)m * ldq;
  auto emit = [&](int g, const uint32_t (&v)[4]) {
    uint32_t w[2] = {0, 0};
    if (s != 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t c2 = f32x2_to_e4m3x2(__fdiv_rn(bf16_bits_to_f32(v[i] & 0xffffu), s),
                                            __fdiv_rn(bf16_bits_to_f32(v[i] >> 16), s));
        w[i >> 1] |= c2 << (16 * (i & 1));
      }
    }
    *reinterpret_cast<uint2*>(q + 8 * g) = make_uint2(w[0], w[1]);
  };
#pragma unroll
  for (int c = 0; c < kQCache; ++c) {
    const int g = g0 + threadIdx.x + c * kQT;
    if (g < g1) emit(g, h[c]);
  }
  for (int g = g0 + threadIdx.x + kQCache * kQT; g < g1; g += kQT) {
    uint32_t t[4];
    load_group<S>(ar, br, g, t);
    emit(g, t);
  }
  cluster_sync();  // keep this CTA's shared memory alive until every CTA has read it
}

// Per-row exponent e with max|x| * 2^e in [2^7, 2^8), clamped so that 2^e and 2^-e are
// normal f32 values (rows whose maximum is below 2^-119 lose precision; zero rows give 0).
__device__ __forceinline__ int e4m3_split_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  const uint32_t b = __float_as_uint(amax);
  const int field = (int)((b >> 23) & 0xff);
  const int E = field != 0 ? field - 127 : (31 - __clz((int)(b & 0x7fffff))) - 149;  // amax in [2^E, 2^(E+1))
  return max(-126, min(126, 7 - E));
}

// W8A16 two-term split of row blockIdx.y: codes[m] = hi(x'[m]), codes[half + m] = lo(x'[m])
// and x_mul[m] = 2^-e[m]; rows m >= rows (padding up to `half`) get zero codes.
__global__ void __launch_bounds__(kQT) w8a16_split_cluster_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                                  int rows, int k, int half,
                                                                  uint8_t* __restrict__ codes,
                                                                  float* __restrict__ x_mul) {
  __shared__ float red[kQT / 32];
  __shared__ float cta_max;
  grid_dependents_launch();  // the GEMV may start its prologue and weight loads now
  grid_dependency_wait();    // launched early (programmatic): x and the codes follow the preceding kernel
  const int m = blockIdx.y;
  uint8_t* hi_row = codes + (int64_t)m * k;
  uint8_t* lo_row = codes + (int64_t)(half + m) * k;
  int g0, g1;
  cta_range(k / 8, g0, g1);
  if (m >= rows) {  // the whole cluster takes this branch: no cluster barrier is skipped
    for (int g = g0 + threadIdx.x; g < g1; g += kQT) {
      *reinterpret_cast<uint2*>(hi_row + 8 * g) = make_uint2(0, 0);
      *reinterpret_cast<uint2*>(lo_row + 8 * g) = make_uint2(0, 0);
    }
    if (cluster_rank() == 0 && threadIdx.x == 0) x_mul[m] = 0.f;
    return;
  }
  const uint16_t* xr = x + (int64_t)m * ldx;
  uint32_t h[kQCache][4];
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < kQCache; ++c) {
    const int g = g0 + threadIdx.x + c * kQT;
    if (g < g1) {
      load_group<Src::Plain>(xr, nullptr, g, h[c]);
      amax = group_amax(h[c], amax);
    }
  }
  for (int g = g0 + threadIdx.x + kQCache * kQT; g < g1; g += kQT) {
    uint32_t t[4];
    load_group<Src::Plain>(xr, nullptr, g, t);
    amax = group_amax(t, amax);
  }
  amax = cluster_row_max(amax, red, &cta_max);
  const int e = e4m3_split_exponent(amax);
  const float mul = __int_as_float((127 + e) << 23);
  if (cluster_rank() == 0 && threadIdx.x == 0) x_mul[m] = __int_as_float((127 - e) << 23);
  auto emit = [&](int g, const uint32_t (&v)[4]) {
    uint32_t hi[2] = {0, 0}, lo[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // elements 2i, 2i+1 of the group
      const float p = bf16_bits_to_f32(v[i] & 0xffffu) * mul;  // exact (power of two)
      const float q = bf16_bits_to_f32(v[i] >> 16) * mul;
      const uint32_t h2 = f32x2_to_e4m3x2(p, q);
      const uint32_t hf = e4m3x2_to_f16x2((uint16_t)h2);
      const float rp = p - f16_bits_to_f32(hf & 0xffffu);  // exact residual
      const float rq = q - f16_bits_to_f32(hf >> 16);
      const uint32_t l2 = f32x2_to_e4m3x2(rp * 16.f, rq * 16.f);
      hi[i >> 1] |= h2 << (16 * (i & 1));
      lo[i >> 1] |= l2 << (16 * (i & 1));
    }
    *reinterpret_cast<uint2*>(hi_row + 8 * g) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(lo_row + 8 * g) = make_uint2(lo[0], lo[1]);
  };
#pragma unroll
  for (int c = 0; c < kQCache; ++c) {
    const int g = g0 + threadIdx.x + c * kQT;
    if (g < g1) emit(g, h[c]);
  }
  for (int g = g0 + threadIdx.x + kQCache * kQT; g < g1; g += kQT) {
    uint32_t t[4];
    load_group<Src::Plain>(xr, nullptr, g, t);
    emit(g, t);
  }
  cluster_sync();
}

// Four pairs of values -> eight packed E2M1 codes (element 2i in the low nibble of byte i),
// round-to-nearest-even with saturation to +-6 (cvt.rn.satfinite.e2m1x2: first source in the
// high nibble).
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{ .reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3}; }"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// NVFP4 quantize of row blockIdx.y (the W4A4 activations), each decision in f32:
//   g = amax / 2688;  per 16-value block b:  s_b = e4m3_rn_sat(bmax / (6 g)),
//   S_b = e4m3(s_b) * g,  codes = e2m1_rn_sat(x / S_b)  (all zero where S_b == 0).
// One thread per block of 16 values (two 16-byte loads), a cluster of kQC CTAs per row.
__global__ void __launch_bounds__(kQT) nvfp4_quant_cluster_kernel(const uint16_t* __restrict__ x, int64_t ldx,
                                                                  int k, uint8_t* __restrict__ xq,
                                                                  uint8_t* __restrict__ xbs, float* __restrict__ xg) {
  __shared__ float red[kQT / 32];
  __shared__ float cta_max;
  grid_dependents_launch();
  grid_dependency_wait();  // launched early (programmatic): x and the codes follow the preceding kernel
  const int m = blockIdx.y;
  const uint16_t* xr = x + (int64_t)m * ldx;
  int b0, b1;
  cta_range(k / 16, b0, b1);
  constexpr int kCache = 2;  // blocks a thread keeps in registers
  uint32_t h[kCache][8];
  auto load_block = [&](int b, uint32_t (&v)[8]) {
    const uint4 lo = ldg_nc(xr + 16 * b), hi = ldg_nc(xr + 16 * b + 8);
    v[0] = lo.x, v[1] = lo.y, v[2] = lo.z, v[3] = lo.w, v[4] = hi.x, v[5] = hi.y, v[6] = hi.z, v[7] = hi.w;
  };
  auto block_max = [&](const uint32_t (&v)[8]) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a = fmaxf(a, fabsf(bf16_bits_to_f32(v[i] & 0xffffu)));
      a = fmaxf(a, fabsf(bf16_bits_to_f32(v[i] >> 16)));
    }
    return a;
  };
  float amax = 0.f;
#pragma unroll
  for (int c = 0; c < kCache; ++c) {
    const int b = b0 + threadIdx.x + c * kQT;
    if (b < b1) {
      load_block(b, h[c]);
      amax = fmaxf(amax, block_max(h[c]));
    }
  }
  for (int b = b0 + threadIdx.x + kCache * kQT; b < b1; b += kQT) {
    uint32_t t[8];
    load_block(b, t);
    amax = fmaxf(amax, block_max(t));
  }
  amax = cluster_row_max(amax, red, &cta_max);
  const float g = __fdiv_rn(amax, 2688.0f);
  const float d6 = __fmul_rn(6.0f, g);
  if (cluster_rank() == 0 && threadIdx.x == 0) xg[m] = g;
  uint8_t* qrow = xq + (int64_t)m * (k / 2);
  uint8_t* srow = xbs + (int64_t)m * (k / 16);
  auto emit = [&](int b, const uint32_t (&v)[8]) {
    const float bmax = block_max(v);
    const float sf = d6 > 0.f ? __fdiv_rn(bmax, d6) : 0.f;
    const uint32_t scode = f32x2_to_e4m3x2(sf, 0.f) & 0xffu;
    const float S = __fmul_rn(f16_bits_to_f32(e4m3x2_to_f16x2((uint16_t)scode) & 0xffffu), g);
    uint32_t w[2] = {0u, 0u};
    if (S > 0.f) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float q[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t pair = v[4 * half + i];
          q[2 * i] = __fdiv_rn(bf16_bits_to_f32(pair & 0xffffu), S);
          q[2 * i + 1] = __fdiv_rn(bf16_bits_to_f32(pair >> 16), S);
        }
        w[half] = f32x8_to_e2m1x8(q);
      }
    }
    *reinterpret_cast<uint2*>(qrow + 8 * b) = make_uint2(w[0], w[1]);
    srow[b] = (uint8_t)scode;
  };
#pragma unroll
  for (int c = 0; c < kCache; ++c) {
    const int b = b0 + threadIdx.x + c * kQT;
    if (b < b1) emit(b, h[c]);
  }
  for (int b = b0 + threadIdx.x + kCache * kQT; b < b1; b += kQT) {
    uint32_t t[8];
    load_block(b, t);
    emit(b, t);
  }
  cluster_sync();
}

template <typename... KArgs, typename... Args>
int launch_cluster(void (*kernel)(KArgs...), int rows, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(kQC, rows);
  cfg.blockDim = dim3(kQT);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  // a cluster per row; programmatic stream serialization lets the launch (and CTA set-up)
  // overlap the preceding kernel's tail: the kernels wait for it before touching memory
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kQC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    (void)cudaGetLastError();
    return DLMH_ERR_CUDA;
  }
  return DLMH_OK;
}

}  // namespace

int w8a8_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* xq, int64_t ldq, float* sx,
                         cudaStream_t s) {
  if (rows <= 0) return DLMH_OK;
  return launch_cluster(w8a8_quant_cluster_kernel<Src::Plain>, rows, s, x, static_cast<const uint16_t*>(nullptr),
                        ldx, k, xq, ldq, sx);
}

int w8a8_silu_quantize_launch(const uint16_t* gate, const uint16_t* up, int64_t ld, int rows, int k, uint8_t* xq,
                              int64_t ldq, float* sx, cudaStream_t s) {
  if (rows <= 0) return DLMH_OK;
  return launch_cluster(w8a8_quant_cluster_kernel<Src::Silu>, rows, s, gate, up, ld, k, xq, ldq, sx);
}

int nvfp4_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* xq, uint8_t* xbs, float* xg,
                          cudaStream_t s) {
  if (rows <= 0) return DLMH_OK;
  return launch_cluster(nvfp4_quant_cluster_kernel, rows, s, x, ldx, k, xq, xbs, xg);
}

int w8a16_split_launch(const uint16_t* x, int64_t ldx, int rows, int k, int half, uint8_t* codes, float* x_mul,
                       cudaStream_t s) {
  if (half <= 0) return DLMH_OK;
  return launch_cluster(w8a16_split_cluster_kernel, half, s, x, ldx, rows, k, half, codes, x_mul);
}

}  // namespace dlmh
