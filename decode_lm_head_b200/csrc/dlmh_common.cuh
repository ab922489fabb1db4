// Shared device helpers of libdlmh: PTX wrappers for loads, conversions and warp MMAs,
// and the host-side launch bookkeeping.  sm_100a only.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dlmh.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libdlmh is built for sm_100a only"
#endif

namespace dlmh {

// Streaming 128-bit load that does not allocate in L1: weights
// are read exactly once per pass.
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ldg_nc(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// 16-bit read-only load.
__device__ __forceinline__ uint32_t ldg_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(saddr));
  return r;
}

__device__ __forceinline__ void sts128(uint32_t saddr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Two E4M3 codes (low byte = element 0) -> f16x2 (exact: every E4M3 value is an f16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(v));
  return r;
}

// Programmatic dependent launch.  grid_dependents_launch(): this grid no longer holds back
// the next kernel of the stream launched with programmatic stream serialization (it may
// start its prologue now).  grid_dependency_wait(): block until the preceding kernel of the
// stream has completed and its memory is visible (returns at once without such a launch).
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Two f32 values -> two E4M3 codes (round-to-nearest-even, saturating to +-448);
// `lo` lands in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E2M1 codes in one byte (low nibble = element 0) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte_in_low8) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(r) : "r"(byte_in_low8));
  return r;
}

// Eight E2M1 codes (one 32-bit word, byte i = codes 2i, 2i+1) -> four f16x2 (exact); r[i] from
// byte i.  The word is split into its four bytes once, with no shifts or masks.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t (&r)[4]) {
  asm("{ .reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3; }"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(w));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// D += A(16x16, f16, row) * B(16x8, f16, col), f32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A(16x32, e4m3, row) * B(32x8, e4m3, col), f32 accumulate.
__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D += A(16x16, s8, row) * B(16x8, s8, col), s32 accumulate (exact).
__device__ __forceinline__ void mma_s8_16816(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// f16 bits -> f32 (exact).
__device__ __forceinline__ float f16_bits_to_f32(uint32_t bits16) {
  float r;
  asm("{ .reg .b16 h; cvt.u16.u32 h, %1; cvt.f32.f16 %0, h; }" : "=f"(r) : "r"(bits16));
  return r;
}

// f32 -> bf16 bits, round-to-nearest-even (hardware cvt).
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
  return r;
}

// f32 -> f16 bits, round-to-nearest-even.
__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
  uint16_t r;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Exponent e with max|row| * 2^e in [2^14, 2^15): the power of two that moves a BF16 row
// into f16 range without rounding (|x| >= 2^-31 * amax stays exact).  Clamped so that
// 2^e and 2^-e stay normal f32 values.
__device__ __forceinline__ int f16_row_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  int e = 14 - (int)((__float_as_uint(amax) >> 23) & 0xff) + 127;  // amax in [2^E, 2^(E+1)) -> e = 14 - E
  if ((__float_as_uint(amax) >> 23 & 0xff) == 0) e = 14 + 126;     // f32 subnormal amax
  return max(-100, min(100, e));
}

}  // namespace dlmh

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
namespace dlmh {

struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;
};

// Per-device properties, queried once per device (thread-safe after first call per device).
DeviceInfo device_info();

// cudaFuncAttributeMaxDynamicSharedMemorySize of `fn` on the current device raised to at
// least `bytes`, set once per (function, device) and remembered (thread-safe).
int ensure_dynamic_smem(const void* fn, int bytes);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? DLMH_OK : DLMH_ERR_CUDA;
}

}  // namespace dlmh
