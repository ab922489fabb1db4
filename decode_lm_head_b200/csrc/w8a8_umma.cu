// W8A8 GEMV on the 5th-generation tensor cores: TMA -> shared memory -> tcgen05.mma ->
// TMEM -> registers.  One weight pass serves up to 128 activation rows.
//
//   out[m, n] = bf16( s[n] * sx[m] * sum_k e4m3(W[n, k]) * e4m3(xq[m, k]) )
//
// Swap-AB: the weight is the MMA's A operand (M = 128 weight rows per tile) and the
// quantized activation rows are its B operand (N = rows rounded up to 16, at most 128), so a
// wide batch rides along one pass over the weight.  Both operands are E4M3 bytes used as
// stored (kind::f8f6f4, f32 accumulation in tensor memory); nothing is decoded.
//
// Operand staging: both matrices are read through 3-D tensor maps over [rows][K] bytes,
// dims {128 (k within a chunk), rows, K/128 (chunk)}: one TMA load brings BM rows x KC
// chunks, i.e. KC*128 contiguous bytes of every row, and writes shared memory as
// [chunk][row][128 B] with the 128-byte swizzle, which is exactly the K-major SWIZZLE_128B
// operand layout the MMA reads (8-row groups 1024 bytes apart).
//
// Roles (192 threads, one CTA per SM, persistent over a contiguous range of 128-row tiles):
//   warp 0: producer (one thread issues the A and B tensor loads of every stage);
//   warp 1: allocates tensor memory, then one thread issues the MMAs (4 per 128-byte
//           chunk, K = 32 each) and commits each stage back to the producer and each
//           finished tile to the epilogue;
//   warps 2-5: epilogue -- tcgen05.ld the accumulator (warp w reads TMEM lanes 32*(w%4)...),
//           apply the row and activation scales, round to BF16, coalesced stores.
// Two accumulators (2 x N columns of TMEM) let the epilogue of one tile overlap the MMAs of
// the next.  Every mbarrier wait is bounded and records a fault bit instead of hanging;
// the allocating warp always frees its tensor memory before exit.
#include <cuda.h>

#include <mutex>

#include "dlmh_common.cuh"
#include "gemv_launch.h"

namespace dlmh {
namespace {

constexpr int kUmmaThreads = 192;
constexpr int kBM = 128;           // weight rows per tile (MMA M)
constexpr int kKC = 2;             // 128-byte K-chunks per stage
constexpr int kChunkBytesA = kBM * 128;
constexpr uint32_t kUWaitLimit = 1u << 22;
constexpr int kMaxUStages = 6;

static __device__ int umma_fault_word = 0;  // 1: producer, 2: MMA (stage), 4: MMA (tmem), 8: epilogue

__device__ __forceinline__ bool uwait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kUWaitLimit; ++i) {
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

__device__ __forceinline__ void ubar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void ubar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void ubar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 3-D tiled TMA load into shared memory (no multicast), completing bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);          // start address
  d |= (uint64_t)1 << 16;                          // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;                // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                          // layout: SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::f8f6f4, A = B = E4M3, D = F32, both K-major, M = 128, N.
__device__ __forceinline__ uint32_t idesc_e4m3(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ void umma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int accum) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

struct UmmaParams {
  int n, k, rows, npad;  // npad: MMA N (rows rounded up to 16)
  const float* w_scale;
  const float* x_scale;
  uint16_t* out;
  int64_t ldc;
  int ns;                // ring stages
  int stage_bytes;       // A + B bytes of one stage
};

__global__ void __launch_bounds__(kUmmaThreads, 1)
    w8a8_umma_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                     const UmmaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[kMaxUStages], bar_empty[kMaxUStages], bar_tfull[2], bar_tempty[2];
  __shared__ uint32_t s_tmem;

  const int ntiles = (p.n + kBM - 1) / kBM;
  const int T0 = (int)((int64_t)blockIdx.x * ntiles / gridDim.x);
  const int T1 = (int)((int64_t)(blockIdx.x + 1) * ntiles / gridDim.x);
  if (T0 >= T1) return;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kchunks = p.k / 128;
  const int spt = (kchunks + kKC - 1) / kKC;  // stages per tile
  const int nstages = (T1 - T0) * spt;
  const uint32_t ring_u32 = smem_u32(ring);
  const uint32_t full0 = smem_u32(bar_full), empty0 = smem_u32(bar_empty);
  const uint32_t tfull0 = smem_u32(bar_tfull), tempty0 = smem_u32(bar_tempty);
  const int a_bytes = kKC * kChunkBytesA;
  const int b_chunk = p.npad * 128;
  const uint32_t tmem_cols = p.npad <= 16 ? 32 : (p.npad <= 32 ? 64 : (p.npad <= 64 ? 128 : 256));

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ns; ++i) {
      ubar_init(full0 + 8u * i, 1);
      ubar_init(empty0 + 8u * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      ubar_init(tfull0 + 8u * i, 1);
      ubar_init(tempty0 + 8u * i, 4);  // the four epilogue warps
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_base = s_tmem;

  if (warp == 0) {
    // ---------------- producer
    if (lane == 0) {
      int slot = 0, phase = 0;
      for (int s = 0; s < nstages; ++s) {
        const int tile = T0 + s / spt, j = s % spt;
        if (s >= p.ns && !uwait(empty0 + 8u * slot, phase ^ 1)) atomicOr(&umma_fault_word, 1);
        const uint32_t st = ring_u32 + slot * p.stage_bytes;
        // the full box always lands (rows past n, rows past `rows` and a chunk past K are
        // zero-filled), so every stage completes exactly stage_bytes
        ubar_expect_tx(full0 + 8u * slot, (uint32_t)p.stage_bytes);
        // A: weight rows [tile*128, +128) x chunks [j*KC, j*KC + KC); B: all activation rows
        tma_load_3d(st, &map_w, 0, tile * kBM, j * kKC, full0 + 8u * slot);
        tma_load_3d(st + a_bytes, &map_x, 0, 0, j * kKC, full0 + 8u * slot);
        if (++slot == p.ns) {
          slot = 0;
          phase ^= 1;
        }
      }
      // no copy may still be landing when the CTA exits: wait (bounded) for the last
      // phase of every slot (already complete in a healthy run, where the MMAs consumed it)
      for (int s = nstages - 1; s >= 0 && s >= nstages - p.ns; --s)
        if (!uwait(full0 + 8u * (s % p.ns), (s / p.ns) & 1)) atomicOr(&umma_fault_word, 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3(p.npad);
      int slot = 0, phase = 0;
      for (int i = 0; T0 + i < T1; ++i) {
        const int acc = i & 1;
        if (i >= 2 && !uwait(tempty0 + 8u * acc, ((i - 2) >> 1) & 1)) atomicOr(&umma_fault_word, 4);
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t tmem_d = tmem_base + (uint32_t)acc * (tmem_cols / 2);
        for (int j = 0; j < spt; ++j) {
          if (!uwait(full0 + 8u * slot, phase)) atomicOr(&umma_fault_word, 2);
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const int nch = min(kKC, kchunks - j * kKC);
          const uint32_t st = ring_u32 + slot * p.stage_bytes;
          for (int c = 0; c < nch; ++c) {
            const uint32_t a0 = st + c * kChunkBytesA;
            const uint32_t b0 = st + a_bytes + c * b_chunk;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // K = 32 bytes per MMA
              umma_f8(tmem_d, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32), idesc,
                      (j | c | kk) != 0);
          }
          umma_commit(empty0 + 8u * slot);  // the stage is free once these MMAs have read it
          if (++slot == p.ns) {
            slot = 0;
            phase ^= 1;
          }
        }
        umma_commit(tfull0 + 8u * acc);  // the accumulator is complete
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int lane_row = q * 32 + lane;
    for (int i = 0; T0 + i < T1; ++i) {
      const int tile = T0 + i, acc = i & 1;
      if (!uwait(tfull0 + 8u * acc, (i >> 1) & 1)) atomicOr(&umma_fault_word, 8);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int row = tile * kBM + lane_row;
      const float s = row < p.n ? p.w_scale[row] : 0.f;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * (tmem_cols / 2);
      for (int c0 = 0; c0 < p.npad; c0 += 16) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(taddr + (uint32_t)c0));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (row < p.n) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int m = c0 + jj;
            if (m < p.rows) {
              const float y = (__uint_as_float(v[jj]) * s) * p.x_scale[m];
              p.out[(int64_t)m * p.ldc + row] = f32_to_bf16_bits(y);
            }
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) ubar_arrive(tempty0 + 8u * acc);
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(tmem_cols) : "memory");
  }
}

// ---- host: tensor maps through the driver entry point (no link-time libcuda dependency)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows][K] bytes (row stride ld) as {128, rows, K/128}, box {128, box_rows, KC}, 128B swizzle.
bool make_map(CUtensorMap* m, const void* base, int rows, int k, int64_t ld, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)(k / 128)};
  cuuint64_t strides[2] = {(cuuint64_t)ld, 128};
  cuuint32_t box[3] = {128, (cuuint32_t)box_rows, (cuuint32_t)kKC};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t kUmmaSmemLimit = 232448 - 2048;

}  // namespace

bool w8a8_umma_supported(int k) {
  // whole 128-byte K chunks (the tensor map's innermost box); a pure function of k so that
  // every row count of a given weight takes this kernel
  return k > 0 && k % 128 == 0;
}

int w8a8_umma_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
                   const float* x_scale, int rows, uint16_t* out, int64_t ldc, cudaStream_t s) {
  if (rows < 1 || rows > 128) return DLMH_ERR_ROWS;
  if (!w8a8_umma_supported(k)) return DLMH_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(w) & 15u) || (reinterpret_cast<uintptr_t>(xq) & 15u) || ldq % 16 != 0)
    return DLMH_ERR_ALIGN;
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  UmmaParams p{};
  p.n = n;
  p.k = k;
  p.rows = rows;
  p.npad = (rows + 15) / 16 * 16;
  p.w_scale = w_scale;
  p.x_scale = x_scale;
  p.out = out;
  p.ldc = ldc;
  p.stage_bytes = kKC * (kChunkBytesA + p.npad * 128);
  int ns = (int)(kUmmaSmemLimit / (size_t)p.stage_bytes);
  if (ns > kMaxUStages) ns = kMaxUStages;
  if (ns < 2) return DLMH_ERR_UNSUPPORTED;
  p.ns = ns;
  CUtensorMap mw, mx;
  if (!make_map(&mw, w, n, k, k, kBM) || !make_map(&mx, xq, rows, k, ldq, p.npad)) return DLMH_ERR_CUDA;
  const size_t smem = (size_t)ns * p.stage_bytes + 1024;
  if (cudaFuncSetAttribute(w8a8_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return DLMH_ERR_CUDA;
  const int ntiles = (n + kBM - 1) / kBM;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  w8a8_umma_kernel<<<grid, kUmmaThreads, smem, s>>>(mw, mx, p);
  return launch_status();
}

int umma_fault(int reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, umma_fault_word, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(umma_fault_word, &zero, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  }
  return v;
}

}  // namespace dlmh
