// Shared pieces of the tensor-core (tcgen05) kernels: bounded mbarrier waits, 3-D tensor-map
// TMA loads, shared-memory matrix descriptors, instruction descriptors, TMEM management, and
// the host-side tensor-map encoder (through the runtime's driver entry point, so the library
// needs no link-time libcuda).
//
// Operand layout used by every kernel here: a row-major [rows][K] matrix is viewed as a 3-D
// tensor {128 bytes, rows, K-chunks of 128 bytes}; one TMA box {128 B, R rows, C chunks}
// lands in shared memory as [C][R][128 B] with the 128-byte swizzle, which is the K-major
// SWIZZLE_128B operand layout of tcgen05.mma (8-row groups 1024 bytes apart).
#pragma once

#include <cuda.h>

#include <mutex>
#include <utility>

#include "dlmh_common.cuh"

namespace dlmh {
namespace umma {

constexpr int kBM = 128;                   // weight rows per tile = MMA M
constexpr uint32_t kWaitLimit = 1u << 22;  // try_wait rounds before a wait reports a fault

__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) {
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

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 3-D tiled TMA load into this CTA's shared memory (no multicast), completing on `bar`, with
// an L2 cache policy (from l2_policy_*).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(policy)
      : "memory");
}

// ---- CTA pairs (a cluster of two CTAs on one TPC sharing each MMA, cta_group::2)

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the object at this CTA's shared address `addr` in CTA `rank`
// of the cluster (the same offset there).
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or the peer's), with
// release semantics at cluster scope.
__device__ __forceinline__ void arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// Every thread of both CTAs: all shared-memory writes and arrivals before it are visible
// cluster-wide after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 3-D tiled TMA load into this CTA's shared memory (no multicast) whose completion is counted
// on an mbarrier of either CTA of the pair (`bar_cluster`, a shared::cluster address).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                                 uint32_t bar_cluster, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(bar_cluster), "l"(policy)
      : "memory");
}

// Arrive (once each) on the mbarrier at shared offset `bar` of every CTA in `cta_mask` when the
// pair MMAs issued so far by this thread have completed.
__device__ __forceinline__ void commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}

// Warp-wide in both CTAs of the pair (the same warp of each): allocate `cols` TMEM columns in
// both, at the same address, written to the same shared offset of each CTA.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar` (both addresses
// 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// L2 policies: streamed-once data (the weights) is evicted first, data every CTA re-reads
// (the activation codes) last.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart
// (start, leading offset 16 B (unused when swizzled), stride offset, version 1, layout 2).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, M = 128, F32 accumulator, both operands K-major and of format
// code 0 (E4M3 under kind::f8f6f4, F16 under kind::f16).
__device__ __forceinline__ uint32_t idesc_m128(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}
// The same for a pair MMA: M = 256 (128 rows in each CTA of the pair).
__device__ __forceinline__ uint32_t idesc_m256(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)((2 * kBM) >> 4) << 24);
}

__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Warp-wide: allocate `cols` TMEM columns (a power of two >= 32), address written to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// Warp-wide: 16 consecutive 32-bit columns of this thread's TMEM lane, then wait for them.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

// Tensor map of a row-major matrix with `row_bytes` bytes of K per row (a multiple of 128)
// and row stride `ld_bytes` (a multiple of 16), elements of `elem_bytes` bytes, viewed as
// {128 bytes, rows, row_bytes / 128}; box {128 bytes, box_rows, box_chunks}, 128-byte
// swizzle, out-of-range rows and chunks zero-filled.
inline bool make_map_k128(CUtensorMap* m, const void* base, int elem_bytes, int rows, int64_t row_bytes,
                          int64_t ld_bytes, int box_rows, int box_chunks) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const int inner = 128 / elem_bytes;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)(row_bytes / 128)};
  cuuint64_t strides[2] = {(cuuint64_t)ld_bytes, 128};
  cuuint32_t box[3] = {(cuuint32_t)inner, (cuuint32_t)box_rows, (cuuint32_t)box_chunks};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// make_map_k128 through a small cache keyed by (device, address, geometry): a tensor map
// holds only the address and the geometry, so an equal key gives an equal map (thread-safe).
inline bool cached_map_k128(CUtensorMap* m, const void* base, int elem_bytes, int rows, int64_t row_bytes,
                            int64_t ld_bytes, int box_rows, int box_chunks) {
  struct Entry {
    const void* base;
    int dev, elem_bytes, rows, box_rows, box_chunks;
    int64_t row_bytes, ld_bytes;
    CUtensorMap map;
  };
  constexpr int kEntries = 64;
  static std::mutex mu;
  static Entry cache[kEntries];
  static int used = 0, next = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const Entry& e = cache[i];
      if (e.base == base && e.dev == dev && e.elem_bytes == elem_bytes && e.rows == rows && e.row_bytes == row_bytes &&
          e.ld_bytes == ld_bytes && e.box_rows == box_rows && e.box_chunks == box_chunks) {
        *m = e.map;
        return true;
      }
    }
  }
  if (!make_map_k128(m, base, elem_bytes, rows, row_bytes, ld_bytes, box_rows, box_chunks)) return false;
  std::lock_guard<std::mutex> lock(mu);
  Entry& e = cache[next];
  e = Entry{base, dev, elem_bytes, rows, box_rows, box_chunks, row_bytes, ld_bytes, *m};
  next = (next + 1) % kEntries;
  if (used < kEntries) ++used;
  return true;
}

// Launch with programmatic stream serialization (the kernel may start while the preceding
// kernel of the stream finishes; it must call grid_dependency_wait() before touching
// anything that kernel writes), in clusters of `cluster_x` CTAs along x (grid.x a multiple
// of it; 1: no cluster).
template <typename... KArgs, typename... Args>
inline int launch_pdl_cluster(int cluster_x, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster_x > 1 ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    (void)cudaGetLastError();
    return DLMH_ERR_CUDA;
  }
  return DLMH_OK;
}

// The same without clusters.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      Args&&... args) {
  return launch_pdl_cluster(1, kernel, grid, block, smem, s, std::forward<Args>(args)...);
}

// Smallest power of two >= max(v, 32) (TMEM allocation granularity).
inline __host__ __device__ int tmem_cols_for(int v) {
  int c = 32;
  while (c < v) c <<= 1;
  return c;
}

}  // namespace umma
}  // namespace dlmh
