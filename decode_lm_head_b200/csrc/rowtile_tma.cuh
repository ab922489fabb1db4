// Streamed row-tile GEMV: TMA bulk copies feed a shared-memory ring, the activation
// fragments live in registers.
//
// Same decomposition and numerics as rowtile_gemv.cuh (16-row tiles over the full K, one
// persistent 512-thread CTA per SM, 16 warps splitting K, fixed-order cross-warp reduction
// at the end of each tile), with two changes that matter on sm_100:
//   * weights arrive through `cp.async.bulk` (1-D TMA) into a ring of NS shared-memory
//     stages, each 16 rows x C KB of K (C k-blocks per warp).  One lane per row issues the
//     row's copy; a "full" mbarrier per stage counts the bytes, an "empty" mbarrier collects
//     one arrival per warp when the stage has been read.  Bulk copies land in shared memory
//     directly, so the bytes in flight are bounded by the ring (~130-160 KB), not by the L1
//     space that a large shared-memory carve-out leaves to ordinary loads.  Row copies of
//     2 KB or more run at full HBM speed; 1 KB copies do not, hence C >= 2 where K allows.
//   * warp w always handles k-blocks w, w+16, w+32, ... of each row (slot i of stage j is
//     k-block 16(jC + i) + w), so its slice of the activation rows is fixed for the whole
//     launch and is held in registers (NKB k-blocks x NT n-tiles) in MMA-fragment order.
// Every mbarrier wait is bounded: on timeout the kernel records a fault in dlmh_fault_word
// and carries on (no barrier is skipped, so nothing can hang); the host reads the word with
// dlmh_device_fault().
#pragma once

#include "rowtile_gemv.cuh"

namespace dlmh {

// Fault bits of the bounded waits (bit 0: a producer's wait for a free stage timed out;
// bit 1: a consumer's wait for a stage's bytes timed out).  Never set in a healthy run.
// This header is included by exactly one translation unit (gemv_kernels.cu).
static __device__ int dlmh_fault_word = 0;

constexpr int kSlotRowBytes = kWarps * kKBlockBytes;  // 1024: one 64-byte k-block per warp
constexpr uint32_t kWaitLimit = 1u << 22;             // try_wait rounds before a wait gives up

// A stage: 16 rows x C slots of 1 KB (+ FP4: 16 rows x C x 128 block-scale bytes).
template <class F, int C>
struct StageLayout {
  static constexpr int kRowBytes = C * kSlotRowBytes;
  static constexpr int kPitch = kRowBytes + 64;             // % 128 == 64: conflict-free fragment loads
  static constexpr int kScaleRowBytes = C * kSlotRowBytes / 8;
  static constexpr int kScalePitch = kScaleRowBytes + 16;   // % 128 == 16: rows on distinct banks
  static constexpr int kWeightBytes = kTileRows * kPitch;
  static constexpr int kScaleBytes = F::kBlockScale ? kTileRows * kScalePitch : 0;
  static constexpr int kBytes = kWeightBytes + kScaleBytes;
};

// 32-bit words of the activation fragment per lane, k-block and n-tile.
template <class F>
constexpr int x_words() {
  // W8A8: 16 codes; W4A4: 32 packed FP4 codes (4 words) + the two block scales as f16x2;
  // A16: 32 f16 values
  return F::kXBytes == 1 ? 4 : (F::kXBytes == 0 ? 5 : (F::kElemsPerKB / 4) / 2);
}

// Register-light configurations (8-row tier, at most 40 words of activation fragments per
// lane) run two tiles per reduction round when a tile is one stage, and load x in one pass.
template <int NT, int NKB, int XW>
__host__ __device__ constexpr bool register_light() {
  return NT == 1 && NKB * XW <= 40;
}
template <int NT, int NKB, int XW, int NST>
__host__ __device__ constexpr int tiles_per_round() {
  return (register_light<NT, NKB, XW>() && NST == 1) ? 2 : 1;
}

// Shared memory of the streamed kernel; the partial-sum buffer holds two rounds (parity) of
// up to two tiles for the 8-row tier.
template <class F, int NT, int C, int NS>
__host__ __device__ constexpr size_t stream_smem_bytes() {
  return (size_t)NS * StageLayout<F, C>::kBytes + 2ull * (NT == 1 ? 2 : 1) * kWarps * kTileRows * (8 * NT) * sizeof(float) +
         2 * 8 * NT * sizeof(float) + 2 * NS * sizeof(uint64_t) + 64;
}

// ---- mbarrier / bulk-copy primitives (PTX ISA: mbarrier, cp.async.bulk) ----

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait for the phase with the given parity; false if it did not complete in time.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// 1-D bulk copy global -> this CTA's shared memory, completing bytes on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void record_fault(int code) { atomicOr(&dlmh_fault_word, code); }

// ---- per-k-block MMA work with register-resident activation fragments ----

template <int NT, int XW>
__device__ __forceinline__ void kb_w8a16_reg(float (&acc)[NT][4], const uint4& ra, const uint4& rb,
                                             const uint32_t (&xr)[NT][XW]) {
  const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
  const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a0 = e4m3x2_to_f16x2((uint16_t)(wa[j] & 0xffff));
    const uint32_t a2 = e4m3x2_to_f16x2((uint16_t)(wa[j] >> 16));
    const uint32_t a1 = e4m3x2_to_f16x2((uint16_t)(wb[j] & 0xffff));
    const uint32_t a3 = e4m3x2_to_f16x2((uint16_t)(wb[j] >> 16));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a0, a1, a2, a3, xr[nt][2 * j], xr[nt][2 * j + 1]);
  }
}

template <int NT, int XW>
__device__ __forceinline__ void kb_w8a8_reg(float (&acc)[NT][4], const uint4& ra, const uint4& rb,
                                            const uint32_t (&xr)[NT][XW]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mma_e4m3_16832(acc[nt], ra.x, rb.x, ra.y, rb.y, xr[nt][0], xr[nt][1]);
    mma_e4m3_16832(acc[nt], ra.z, rb.z, ra.w, rb.w, xr[nt][2], xr[nt][3]);
  }
}

template <int NT, int XW>
__device__ __forceinline__ void kb_w4a16_reg(float (&acc)[NT][4], const uint4& ra, const uint4& rb, uint32_t s2a,
                                             uint32_t s2b, const uint32_t (&xr)[NT][XW]) {
  const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
  const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
  const uint32_t sa = e4m3x2_to_f16x2((uint16_t)s2a);
  const uint32_t sb = e4m3x2_to_f16x2((uint16_t)s2b);
  const uint32_t sa0 = __byte_perm(sa, 0, 0x1010), sa1 = __byte_perm(sa, 0, 0x3232);
  const uint32_t sb0 = __byte_perm(sb, 0, 0x1010), sb1 = __byte_perm(sb, 0, 0x3232);
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // word q: bytes 4q..4q+3 feed MMA steps 2q (bytes 4q, 4q+1) and 2q+1
    uint32_t fa[4], fb[4];
    e2m1x8_to_f16x2x4(wa[q], fa);
    e2m1x8_to_f16x2x4(wb[q], fb);
    const uint32_t ssa = (q < 2) ? sa0 : sa1;
    const uint32_t ssb = (q < 2) ? sb0 : sb1;
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // MMA step j = 2q + h: bytes 2j, 2j+1 of the lane's 16 (values 4j..4j+3)
      const int j = 2 * q + h;
      const uint32_t a0 = hmul2(fa[2 * h], ssa), a2 = hmul2(fa[2 * h + 1], ssa);
      const uint32_t a1 = hmul2(fb[2 * h], ssb), a3 = hmul2(fb[2 * h + 1], ssb);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[nt], a0, a1, a2, a3, xr[nt][2 * j], xr[nt][2 * j + 1]);
    }
  }
}

// W4A4: the activation side decoded like the weight side -- MMA step j takes bytes 2j, 2j+1
// of the lane's 16 code bytes (values 4j..4j+3 of its 32), times the block scale of values
// 0..15 (j < 4) or 16..31; every product of two such f16 values is exact in the f32 sum.
template <int NT, int XW>
__device__ __forceinline__ void kb_w4a4_reg(float (&acc)[NT][4], const uint4& ra, const uint4& rb, uint32_t s2a,
                                            uint32_t s2b, const uint32_t (&xr)[NT][XW]) {
  const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
  const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
  const uint32_t sa = e4m3x2_to_f16x2((uint16_t)s2a);
  const uint32_t sb = e4m3x2_to_f16x2((uint16_t)s2b);
  const uint32_t sa0 = __byte_perm(sa, 0, 0x1010), sa1 = __byte_perm(sa, 0, 0x3232);
  const uint32_t sb0 = __byte_perm(sb, 0, 0x1010), sb1 = __byte_perm(sb, 0, 0x3232);
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // word q feeds MMA steps 2q, 2q+1 (as in kb_w4a16_reg)
    uint32_t fa[4], fb[4];
    e2m1x8_to_f16x2x4(wa[q], fa);
    e2m1x8_to_f16x2x4(wb[q], fb);
    const uint32_t ssa = (q < 2) ? sa0 : sa1;
    const uint32_t ssb = (q < 2) ? sb0 : sb1;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t a0 = hmul2(fa[2 * h], ssa), a2 = hmul2(fa[2 * h + 1], ssa);
      const uint32_t a1 = hmul2(fb[2 * h], ssb), a3 = hmul2(fb[2 * h + 1], ssb);
      const int sh = 16 * h;  // the activation side: bytes 4q + 2h, 4q + 2h + 1 of its codes
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint32_t cw = xr[nt][q];
        const uint32_t sx = (q < 2) ? __byte_perm(xr[nt][4], 0, 0x1010) : __byte_perm(xr[nt][4], 0, 0x3232);
        const uint32_t b0 = hmul2(e2m1x2_to_f16x2((cw >> sh) & 0xff), sx);
        const uint32_t b1 = hmul2(e2m1x2_to_f16x2((cw >> (sh + 8)) & 0xff), sx);
        mma_f16_16816(acc[nt], a0, a1, a2, a3, b0, b1);
      }
    }
  }
}

// ---- the kernel ----

template <class F, int NT, int NKB, int C, int NS>
__global__ void __launch_bounds__(kThreads, 1) stream_gemv_kernel(const RowTileParams p) {
  constexpr int MT = 8 * NT;
  constexpr int XW = x_words<F>();
  constexpr int EL = F::kElemsPerKB / 4;  // activation values per lane per k-block
  constexpr int NST = (NKB + C - 1) / C;  // stages per tile
  using L = StageLayout<F, C>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(smem + (size_t)NS * L::kBytes);
  float* rowmul = red + 2 * (NT == 1 ? 2 : 1) * kWarps * kTileRows * MT;  // after two rounds of partials
  int* rowexp = reinterpret_cast<int*>(rowmul + MT);
  uint64_t* bars = reinterpret_cast<uint64_t*>(rowexp + MT + ((MT & 1) ? 1 : 0));  // full[NS], empty[NS]
  __shared__ int s_fault;

  // Programmatic dependent launch: the next kernel on the stream may start its prologue now;
  // this one touches nothing a preceding kernel may write before grid_dependency_wait().
  grid_dependents_launch();
  const int ntiles = (p.n + kTileRows - 1) / kTileRows;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  if (T0 >= T1) return;  // uniform over the CTA, before any barrier

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int kb_total = kblocks_of<F>(p.k);
  const int64_t wrb = p.w_row_bytes;
  const int64_t srb = p.k / 16;
  const int nstages = (T1 - T0) * NST;
  // Whole rows per stage: the 16-row tile (and its block scales) is one contiguous range of
  // HBM, so it lands in one bulk copy each, rows packed at their own length, instead of 16
  // (32) row copies; small copies are what limits the TMA on short rows.  The unpadded pitch
  // costs 2-way bank conflicts on the fragment loads, far below the copy time it saves.
  const bool packed = NST == 1 && wrb % 16 == 0 && (!F::kBlockScale || srb % 16 == 0);
  const uint32_t wpitch = packed ? (uint32_t)wrb : (uint32_t)L::kPitch;
  const uint32_t spitch = packed ? (uint32_t)srb : (uint32_t)L::kScalePitch;
  const uint32_t ring_u32 = smem_u32(ring);
  const uint32_t bar_u32 = smem_u32(bars);
  auto full_bar = [&](int slot) { return bar_u32 + 8u * slot; };
  auto empty_bar = [&](int slot) { return bar_u32 + 8u * (NS + slot); };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), kWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_fault = 0;
  }
  __syncthreads();

  // ---- producer (warp 0): stage s = k-slice j of tile T0 + s / NST
  auto produce = [&](int s) {
    const int tile = T0 + s / NST, j = s % NST, slot = s % NS;
    const int64_t col = (int64_t)j * L::kRowBytes;
    const int cbytes = (int)min((int64_t)L::kRowBytes, wrb - col);
    int sbytes = 0;
    int64_t scol = 0;
    if constexpr (F::kBlockScale) {
      scol = (int64_t)j * L::kScaleRowBytes;
      sbytes = (int)min((int64_t)L::kScaleRowBytes, srb - scol);
    }
    const int rows_valid = min(kTileRows, p.n - tile * kTileRows);
    if (lane == 0) {
      if (s >= NS && !mbar_wait(empty_bar(slot), ((s / NS) - 1) & 1)) {
        record_fault(1);
        s_fault = 1;
      }
      mbar_arrive_expect_tx(full_bar(slot), (uint32_t)(rows_valid * (cbytes + sbytes)));
      if (packed) {
        const int64_t row0 = (int64_t)tile * kTileRows;
        const uint32_t dst = ring_u32 + slot * L::kBytes;
        bulk_g2s(dst, p.w + row0 * wrb, (uint32_t)(rows_valid * wrb), full_bar(slot));
        if constexpr (F::kBlockScale)
          bulk_g2s(dst + L::kWeightBytes, p.w_bscale + row0 * srb, (uint32_t)(rows_valid * srb), full_bar(slot));
      }
    }
    __syncwarp();
    if (!packed && lane < rows_valid) {
      const int64_t row = (int64_t)tile * kTileRows + lane;
      const uint32_t dst = ring_u32 + slot * L::kBytes + lane * L::kPitch;
      bulk_g2s(dst, p.w + row * wrb + col, (uint32_t)cbytes, full_bar(slot));
      if constexpr (F::kBlockScale) {
        const uint32_t sdst = ring_u32 + slot * L::kBytes + L::kWeightBytes + lane * L::kScalePitch;
        bulk_g2s(sdst, p.w_bscale + row * srb + scol, (uint32_t)sbytes, full_bar(slot));
      }
    }
  };

  // The first NS stages.  After this library's own pre-pass (early_w) they are requested at
  // once; otherwise after the preceding kernel, and after this CTA's activation loads, so that
  // the few x bytes are not queued behind the ring's ~180 KB per SM.
  auto prefill = [&]() {
    if (warp == 0)
      for (int s = 0; s < NS && s < nstages; ++s) produce(s);
  };
  if (p.early_w) prefill();
  grid_dependency_wait();  // activations, outputs (and otherwise the weights) follow the preceding kernel

  // ---- activation fragments into registers (while the first stages are in flight)
  uint32_t xr[NKB][NT][XW];
  if constexpr (F::kXBytes == 2 && !register_light<NT, NKB, XW>()) {
    // Two passes over x (the wider tiers keep fewer registers live): each row's maximum from
    // its own warp, then the fragments converted as they load.
    const uint16_t* x = static_cast<const uint16_t*>(p.x);
    for (int m = warp; m < MT; m += kWarps) {  // per-row power of two into f16 range
      float amax = 0.f;
      if (m < p.rows) {
        const uint16_t* xr_ = x + (int64_t)m * p.ldx;
#pragma unroll 4
        for (int k8 = lane * 8; k8 < p.k; k8 += 32 * 8) {
          const uint4 v = ldg_nc(xr_ + k8);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(wv[i] & 0xffffu)));
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(wv[i] >> 16)));
          }
        }
      }
      amax = warp_max(amax);
      if (lane == 0) {
        const int e = f16_row_exponent(amax);
        rowexp[m] = e;
        rowmul[m] = __int_as_float((127 - e) << 23);
      }
    }
    if (!p.early_w) prefill();
    __syncthreads();
#pragma unroll
    for (int j = 0; j < NKB; ++j) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + g;
        const int k0 = (j * kWarps + warp) * F::kElemsPerKB + t * EL;
        const float mul = __int_as_float((127 + rowexp[m]) << 23);
#pragma unroll
        for (int c = 0; c < EL / 8; ++c) {  // 8 values per 16-byte load
          uint4 v = make_uint4(0, 0, 0, 0);
          if (m < p.rows && k0 + 8 * c < p.k) v = ldg_nc(x + (int64_t)m * p.ldx + k0 + 8 * c);
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const uint32_t lo = f32_to_f16_bits(bf16_bits_to_f32(wv[i] & 0xffffu) * mul);
            const uint32_t hi = f32_to_f16_bits(bf16_bits_to_f32(wv[i] >> 16) * mul);
            xr[j][nt][4 * c + i] = lo | (hi << 16);
          }
        }
      }
    }
  } else if constexpr (F::kXBytes == 2) {
    // One pass over x: the lane's fragments are loaded as raw BF16 pairs while each row's
    // maximum is reduced (lanes of a row, then warps through shared memory); the row's power
    // of two into f16 range then converts the fragments in registers.
    const uint16_t* x = static_cast<const uint16_t*>(p.x);
    float pmax[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) pmax[nt] = 0.f;
#pragma unroll
    for (int j = 0; j < NKB; ++j) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + g;
        const int k0 = (j * kWarps + warp) * F::kElemsPerKB + t * EL;
#pragma unroll
        for (int c = 0; c < EL / 8; ++c) {  // 8 values per 16-byte load
          uint4 v = make_uint4(0, 0, 0, 0);
          if (m < p.rows && k0 + 8 * c < p.k) v = ldg_nc(x + (int64_t)m * p.ldx + k0 + 8 * c);
          xr[j][nt][4 * c + 0] = v.x;
          xr[j][nt][4 * c + 1] = v.y;
          xr[j][nt][4 * c + 2] = v.z;
          xr[j][nt][4 * c + 3] = v.w;
        }
      }
    }
    if (!p.early_w) prefill();
#pragma unroll
    for (int j = 0; j < NKB; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int w = 0; w < XW; ++w) {
          pmax[nt] = fmaxf(pmax[nt], fabsf(bf16_bits_to_f32(xr[j][nt][w] & 0xffffu)));
          pmax[nt] = fmaxf(pmax[nt], fabsf(bf16_bits_to_f32(xr[j][nt][w] >> 16)));
        }
    float* wmax = red;  // [kWarps][MT], free until the first tile ends
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float v = pmax[nt];
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
      if (t == 0) wmax[warp * MT + nt * 8 + g] = v;
    }
    __syncthreads();
    if (threadIdx.x < MT) {
      float amax = 0.f;
      for (int w = 0; w < kWarps; ++w) amax = fmaxf(amax, wmax[w * MT + threadIdx.x]);
      const int e = f16_row_exponent(amax);
      rowexp[threadIdx.x] = e;
      rowmul[threadIdx.x] = __int_as_float((127 - e) << 23);
    }
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float mul = __int_as_float((127 + rowexp[nt * 8 + g]) << 23);
#pragma unroll
      for (int j = 0; j < NKB; ++j) {
#pragma unroll
        for (int w = 0; w < XW; ++w) {
          const uint32_t raw = xr[j][nt][w];
          const uint32_t lo = f32_to_f16_bits(bf16_bits_to_f32(raw & 0xffffu) * mul);
          const uint32_t hi = f32_to_f16_bits(bf16_bits_to_f32(raw >> 16) * mul);
          xr[j][nt][w] = lo | (hi << 16);
        }
      }
    }
  } else if constexpr (F::kXBytes == 0) {
    // W4A4: the lane's 32 values of each k-block as 16 packed code bytes + two block scales;
    // the row's NVFP4 global goes to the epilogue
    const uint8_t* xq = static_cast<const uint8_t*>(p.x);
    if (threadIdx.x < MT) rowmul[threadIdx.x] = threadIdx.x < p.rows ? p.x_scale[threadIdx.x] : 0.f;
#pragma unroll
    for (int j = 0; j < NKB; ++j) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + g;
        const int k0 = (j * kWarps + warp) * F::kElemsPerKB + t * EL;
        uint4 v = make_uint4(0, 0, 0, 0);
        uint32_t sc = 0;
        if (m < p.rows && k0 < p.k) {
          v = ldg_nc(xq + (int64_t)m * (p.ldx / 2) + k0 / 2);
          sc = ldg_u16(p.x_bscale + (int64_t)m * (p.k / 16) + k0 / 16);
        }
        xr[j][nt][0] = v.x;
        xr[j][nt][1] = v.y;
        xr[j][nt][2] = v.z;
        xr[j][nt][3] = v.w;
        xr[j][nt][4] = sc;
      }
    }
    if (!p.early_w) prefill();
#pragma unroll
    for (int j = 0; j < NKB; ++j)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) xr[j][nt][4] = e4m3x2_to_f16x2((uint16_t)xr[j][nt][4]);
  } else {
    const uint8_t* x = static_cast<const uint8_t*>(p.x);
    if (threadIdx.x < MT) rowmul[threadIdx.x] = threadIdx.x < p.rows ? p.x_scale[threadIdx.x] : 0.f;
#pragma unroll
    for (int j = 0; j < NKB; ++j) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + g;
        const int k0 = (j * kWarps + warp) * F::kElemsPerKB + t * EL;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < p.rows && k0 < p.k) v = ldg_nc(x + (int64_t)m * p.ldx + k0);
        xr[j][nt][0] = v.x;
        xr[j][nt][1] = v.y;
        xr[j][nt][2] = v.z;
        xr[j][nt][3] = v.w;
      }
    }
    if (!p.early_w) prefill();
  }
  __syncthreads();

  // ---- main loop: rounds of TPR tiles, one cross-warp reduction (one CTA barrier) per round.
  // Two independent tiles per round (8-row tier, one stage per tile) halve the barriers and
  // let the two tiles' MMA chains interleave; the per-output sum is the same either way.
  constexpr int TPR = tiles_per_round<NT, NKB, XW, NST>();
  constexpr int kRed = kWarps * kTileRows * MT;  // floats of one tile's partial sums
  const int red_tt = threadIdx.x / (kTileRows * MT);
  const bool reducer = red_tt < TPR;
  const int red_rr = threadIdx.x % kTileRows, red_cc = (threadIdx.x / kTileRows) % MT;
  float wscale_cur = 0.f;
  if constexpr (!F::kBlockScale) {
    const int row = (T0 + red_tt) * kTileRows + red_rr;
    if (reducer && T0 + red_tt < T1 && row < p.n) wscale_cur = p.w_scale[row];
  }
  float acc[TPR][NT][4];
#pragma unroll
  for (int tt = 0; tt < TPR; ++tt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[tt][nt][i] = 0.f;

  int s = 0, parity = 0;
  for (int tile0 = T0; tile0 < T1; tile0 += TPR) {
    const int ntl = min(TPR, T1 - tile0);
#pragma unroll
    for (int tt = 0; tt < TPR; ++tt) {
      if (tt < ntl) {
#pragma unroll
        for (int j = 0; j < NST; ++j, ++s) {
          const int slot = s % NS;
          if (!mbar_wait(full_bar(slot), (s / NS) & 1)) {
            record_fault(2);
            s_fault = 1;
          }
          const uint32_t stage = ring_u32 + slot * L::kBytes;
#pragma unroll
          for (int i = 0; i < C; ++i) {
            const int q = j * C + i;  // the warp's slot index: k-block 16 q + warp
            if (q < NKB) {
              const int kb = q * kWarps + warp;
              if (kb < kb_total) {
                const int col = kb * kKBlockBytes + 16 * t;  // lane's byte column in the row
                const uint32_t st = stage + g * wpitch + (i * kWarps + warp) * kKBlockBytes + 16 * t;
                uint4 ra = make_uint4(0, 0, 0, 0), rb = ra;
                uint32_t sa = 0, sb = 0;
                if (col < wrb) {
                  ra = lds128(st);
                  rb = lds128(st + 8 * wpitch);
                  if constexpr (F::kBlockScale) {
                    const uint32_t ss = stage + L::kWeightBytes + g * spitch + (i * kWarps + warp) * 8 + 2 * t;
                    uint16_t va, vb;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(va) : "r"(ss));
                    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(vb) : "r"(ss + 8 * spitch));
                    sa = va;
                    sb = vb;
                  }
                }
                if constexpr (F::kXBytes == 0)
                  kb_w4a4_reg<NT, XW>(acc[tt], ra, rb, sa, sb, xr[q]);
                else if constexpr (F::kBlockScale)
                  kb_w4a16_reg<NT, XW>(acc[tt], ra, rb, sa, sb, xr[q]);
                else if constexpr (F::kXBytes == 1)
                  kb_w8a8_reg<NT, XW>(acc[tt], ra, rb, xr[q]);
                else
                  kb_w8a16_reg<NT, XW>(acc[tt], ra, rb, xr[q]);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(empty_bar(slot));
          if (warp == 0 && s + NS < nstages) produce(s + NS);
        }
      }
    }

    // ---- end of round: fixed-order cross-warp reduction of each tile
    float* rb_ = red + parity * (TPR * kRed);
#pragma unroll
    for (int tt = 0; tt < TPR; ++tt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        reinterpret_cast<float4*>(rb_ + tt * kRed)[(warp * NT + nt) * 32 + lane] =
            make_float4(acc[tt][nt][0], acc[tt][nt][1], acc[tt][nt][2], acc[tt][nt][3]);
        acc[tt][nt][0] = acc[tt][nt][1] = acc[tt][nt][2] = acc[tt][nt][3] = 0.f;
      }
    __syncthreads();
    if (reducer) {
      const int rr = red_rr, cc = red_cc, tile = tile0 + red_tt;
      const int row = tile * kTileRows + rr;
      const float* rt = rb_ + red_tt * kRed;
      float wsc = 0.f;
      if constexpr (!F::kBlockScale) {
        wsc = wscale_cur;
        const int nrow = row + TPR * kTileRows;
        if (tile + TPR < T1 && nrow < p.n) wscale_cur = p.w_scale[nrow];
      }
      if (red_tt < ntl && cc < p.rows && row < p.n) {
        const int gg = rr & 7, up = rr >> 3;
        const int nt = cc >> 3, cl = cc & 7;
        const int ln = gg * 4 + (cl >> 1), comp = up * 2 + (cl & 1);
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < kWarps; ++ww) sum += rt[((ww * NT + nt) * 32 + ln) * 4 + comp];
        float y;
        if constexpr (F::kBlockScale)
          y = (sum * p.gscale) * rowmul[cc];
        else
          y = (sum * wsc) * rowmul[cc];
        p.out[(int64_t)cc * p.ldc + row] = f32_to_bf16_bits(y);
      }
    }
    parity ^= 1;
  }

  // A stage whose wait timed out may still be landing: let it finish (bounded) before the
  // CTA's shared memory is released.
  __syncthreads();
  if (s_fault && threadIdx.x == 0) {
    for (int q = max(0, nstages - NS); q < nstages; ++q) (void)mbar_wait(full_bar(q % NS), (q / NS) & 1);
  }
}

}  // namespace dlmh
