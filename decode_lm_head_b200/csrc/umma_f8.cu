// E4M3-weight GEMV on the 5th-generation tensor cores: TMA -> shared memory -> tcgen05.mma
// -> TMEM -> registers.  One weight pass serves up to 128 activation rows, for both
//
//   W8A8:   out[m, n] = bf16( s[n] * sx[m] * sum_k e4m3(W[n, k]) * e4m3(xq[m, k]) )
//   W8A16:  out[m, n] = bf16( s[n] * 2^-e[m] * sum_k e4m3(W[n, k]) * (hi[m, k] + lo[m, k] / 16) )
//
// where, for W8A16, x'[m, :] = x[m, :] * 2^e[m] (max|x'| in [2^7, 2^8)) is split into two
// E4M3 terms hi = e4m3(x'), lo = e4m3(16 (x' - hi)).  A BF16 value has 8 significant bits;
// rounding it to E4M3's 4 leaves a residual of at most 4 bits, so hi + lo/16 == x' exactly
// whenever |x'| >= 2^-6 (every element within 2^-13 of the row maximum); below that the
// error is at most 2^-14 in x' units.  The two terms are the B operand's first and second
// roundup8(rows) columns, so the weights stay E4M3 in the A operand.  The tensor pipe's time per
// M=128, K=32-byte instruction grows with N (about 32 clocks at N = 64, 129 at N = 256: the
// dense FP8 rate): small row counts stay far from it, while at 128 W8A16 rows (N = 256) the MMA
// is busy for about 70 % of the weight stream's time.
//
// Swap-AB: the weight is the MMA's A operand (M = 128 weight rows per tile) and the
// activation codes are its B operand (N = rows rounded up to 16; for W8A16 twice the rows
// rounded up to 8).
// Both operands are E4M3 bytes used as stored (kind::f8f6f4, f32 accumulation in TMEM).
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
#include "gemv_launch.h"
#include "umma_common.cuh"
#include "umma_sched.h"
#include "workspace_plan.h"

namespace dlmh {
namespace {

using namespace umma;

constexpr int kUmmaThreads = 192;
constexpr int kKC = kUmmaStageChunks;  // 128-byte K-chunks per schedule unit
static_assert(kBM == kUmmaTileRows, "the workspace layout assumes 128-row tiles");
constexpr int kChunkBytesA = kBM * 128;
constexpr int kMaxUStages = 8;
static_assert(kKC % 2 == 0, "a unit is one stage or two");
constexpr int kJobRing = 4;  // job descriptors in flight from the producer to the MMA and epilogue warps

static __device__ int umma_fault_word = 0;  // 1: producer, 2: MMA (stage), 4: MMA (tmem), 8: epilogue
constexpr int kWaitProbeBit = 0x40;         // set only by the bounded-wait check

__device__ __forceinline__ void umma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, int accum) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

// The pair form: M = 256, A rows [0, 128) and B rows [0, N/2) from the issuing CTA's shared
// memory, A rows [128, 256) and B rows [N/2, N) from its peer's (same offsets); D rows
// [0, 128) into the issuer's TMEM, [128, 256) into the peer's (same address).
__device__ __forceinline__ void umma_f8_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             int accum) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0; "
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p; }" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}

struct UmmaParams {
  int n, k, rows, npad;  // npad: rows rounded up to 16 (the epilogue's column loop)
  int nb;                // MMA N = B rows: npad (W8A8) or 2 * roundup8(rows) (W8A16 hi | lo)
  int split;             // 1: W8A16 two-term epilogue
  int lo_off;            // W8A16: column of row 0's lo term (roundup8(rows))
  int accw;              // TMEM columns per accumulator (a power of two >= 32)
  const float* w_scale;
  const float* x_scale;  // sx[m] (W8A8) or 2^-e[m] (W8A16)
  uint16_t* out;
  int64_t ldc;
  int ns;                // ring stages
  int cps;               // 128-byte chunks per stage: kKC, or kKC / 2 (each unit as two stages)
  int stage_bytes;       // A + B bytes of one stage
  // Stream-K schedule (umma_schedule) over P = gridDim.x / 2 parties (CTA pairs) and tile
  // pairs, a pure function of n, k and the SM count, never of the row count; partial sums are
  // laid out [slot][col][128 rows], two slots per CTA.
  int spt, wt, rem;
  float* partial;
  // Dynamic hand-out of the whole tiles from the caller workspace's queue (null: the static
  // order of the schedule).  queue[0] counts tiles claimed beyond each CTA's first, queue[1]
  // the CTAs that have finished; the last CTA to finish puts both back to 0 for the next
  // launch on the stream.  A whole tile's bits do not depend on which CTA ran it, so both
  // orders give the same outputs.
  int* queue;
  int early_w;  // 1: the preceding kernel is this library's activation pre-pass (it writes
                // neither W nor the outputs), so weight loads may start before it completes
  // A second weight matrix against the same activations (an FFN's gate and up) runs in the
  // same launch: tiles [t1, ...) read map_w2 and write out2 with w_scale2.  Without one, t1
  // is the tile count.
  int t1, n2;
  const float* w_scale2;
  uint16_t* out2;
  int64_t ldc2;
};

// Where tile `tile`'s 128 output columns go.
struct TileDst {
  int row0, n;
  const float* scale;
  uint16_t* out;
  int64_t ldc;
};

__device__ __forceinline__ TileDst tile_dst(const UmmaParams& p, int tile) {
  if (tile < p.t1) return TileDst{tile * kBM, p.n, p.w_scale, p.out, p.ldc};
  return TileDst{(tile - p.t1) * kBM, p.n2, p.w_scale2, p.out2, p.ldc2};
}


// The schedule's parties are CTA pairs and its tiles tile pairs (umma_schedule): CTAs 2j and
// 2j + 1 both run party j's jobs, CTA 2j + h on single tile 2T + h of tile pair T, so the two
// tiles of a pair always get the same K split (whichever kernel runs them, and whatever the row
// count).  Whole tiles may also be claimed one by one from the workspace queue.
//
// kPair: each pair is a cluster on one TPC and the two CTAs share every MMA (cta_group::2,
// M = 256): CTA rank h loads its tile's weight rows and rows [h N/2, (h + 1) N/2) of the
// activation box into its own ring.  Rank 0 issues the MMAs; the copies of both CTAs count on
// rank 0's full barriers, and each commit arrives on the empty (or accumulator-full) barrier of
// both CTAs.  Per SM the activation box and its shared memory are halved, so the ring holds
// more stages when N is large.  Static tile order.
template <bool kPair>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    umma_f8_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_w2,
                   const __grid_constant__ CUtensorMap map_x, const UmmaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[kMaxUStages], bar_empty[kMaxUStages], bar_tfull[2], bar_tempty[2];
  __shared__ __align__(8) uint64_t bar_jfull[kJobRing], bar_jempty[kJobRing];
  __shared__ int4 s_job[kJobRing];  // (tile, first unit, end unit, partial slot); tile < 0 ends
  __shared__ uint32_t s_tmem;

  // party b = CTAs 2b and 2b + 1; this CTA is half h of it (in a pair, its cluster rank)
  const int h = kPair ? (int)cluster_ctarank() : (int)(blockIdx.x & 1);
  const bool leader = !kPair || h == 0;  // issues the MMAs (a pair's rank 0 for both CTAs)
  const int nctas = (int)gridDim.x;
  const int P = nctas / 2;
  const int b = (int)blockIdx.x / 2;
  const Sched sc{p.spt, p.wt, p.rem, P};
  {
    int tile, u0, u1, slot;
    if (!sc.job(b, 0, tile, u0, u1, slot)) return;  // no work at all (uniform over the party)
  }
  const bool dyn = !kPair && p.queue != nullptr && p.wt > 0;
  const int nwhole = 2 * p.wt * P;  // single tiles [0, nwhole) are whole

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kchunks = p.k / 128;
  const uint32_t ring_u32 = smem_u32(ring);
  const uint32_t full0 = smem_u32(bar_full), empty0 = smem_u32(bar_empty);
  const uint32_t tfull0 = smem_u32(bar_tfull), tempty0 = smem_u32(bar_tempty);
  const int a_bytes = p.cps * kChunkBytesA;
  const int sub = kKC / p.cps;  // stages per schedule unit
  const int bn = kPair ? p.nb / 2 : p.nb;  // activation rows in this CTA's stages
  const int b_chunk = bn * 128;
  const uint32_t tmem_cols = 2u * (uint32_t)p.accw;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.ns; ++i) {
      bar_init(full0 + 8u * i, 1);
      bar_init(empty0 + 8u * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      bar_init(tfull0 + 8u * i, 1);
      bar_init(tempty0 + 8u * i, kPair ? 8 : 4);  // the four epilogue warps (of both CTAs)
    }
    for (int i = 0; i < kJobRing; ++i) {
      bar_init(smem_u32(&bar_jfull[i]), 1);
      // the MMA thread (rank 0 only) and the four epilogue warps
      bar_init(smem_u32(&bar_jempty[i]), leader ? 5 : 4);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (kPair)
      tmem_alloc_pair(smem_u32(&s_tmem), tmem_cols);
    else
      tmem_alloc(smem_u32(&s_tmem), tmem_cols);
  }
  fence_before();
  __syncwarp();
  if constexpr (kPair)
    cluster_sync();  // both CTAs' barriers exist before either signals the other's
  else
    __syncthreads();
  fence_after();
  const uint32_t tmem_base = s_tmem;
  grid_dependents_launch();  // the fixup may be scheduled; it waits for this grid to finish

  if (warp == 0) {
    // ---------------- producer: hands out the jobs and streams their stages
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first(), pol_x = l2_policy_evict_last();
      // Job sequence (single tile, first unit, end unit, partial slot): the whole tiles (the
      // first static -- tile 2b + h, or the party's tile pairs in the static order -- the rest
      // claimed from the queue or taken in order), then the party's remainder segments on this
      // CTA's half of their tile pairs, then an end marker.
      bool whole = p.wt > 0;  // still handing out whole tiles
      int wj = 0;             // whole tiles taken so far
      int rj = p.wt;          // schedule index of the next remainder segment
      auto next_job = [&](int4& jb) -> bool {
        if (whole) {
          int tile;
          if (dyn)
            tile = wj == 0 ? (int)blockIdx.x : nctas + atomicAdd(p.queue, 1);
          else
            tile = wj < p.wt ? 2 * (b * p.wt + wj) + h : -1;
          if (tile >= 0 && tile < nwhole) {
            ++wj;
            jb = make_int4(tile, 0, p.spt, -1);
            return true;
          }
          whole = false;
        }
        int tp, u0, u1, ps;
        if (sc.job(b, rj, tp, u0, u1, ps)) {
          ++rj;
          // the party's slot 2b + s is this CTA's 2 (2b + h) + s
          jb = make_int4(2 * tp + h, u0, u1, 2 * (int)blockIdx.x + (ps - 2 * b));
          return true;
        }
        return false;
      };
      int nj = 0;  // jobs published
      auto publish = [&](const int4& jb) {
        const int r = nj % kJobRing;
        if (nj >= kJobRing && !wait(smem_u32(&bar_jempty[r]), ((nj / kJobRing) - 1) & 1))
          atomicOr(&umma_fault_word, 16);
        s_job[r] = jb;
        arrive(smem_u32(&bar_jfull[r]));  // release: the descriptor is visible to the waiters
        ++nj;
      };
      // The first job is static: its first ring of weight tiles may be requested before the
      // preceding kernel has finished (early_w); activation tiles only after it.
      int4 jb;
      next_job(jb);
      publish(jb);
      // Copies count on this CTA's full barrier, or in a pair on rank 0's, whose producer
      // expects both CTAs' bytes.
      const uint32_t fullc0 = kPair ? mapa_shared(full0, 0) : full0;
      const uint32_t expect = kPair ? 2u * (uint32_t)p.stage_bytes : (uint32_t)p.stage_bytes;
      auto load = [&](uint32_t dst, const CUtensorMap* map, int c1, int c2, int slot_, uint64_t pol) {
        if constexpr (kPair)
          tma_load_3d_pair(dst, map, 0, c1, c2, fullc0 + 8u * slot_, pol);
        else
          tma_load_3d(dst, map, 0, c1, c2, full0 + 8u * slot_, pol);
      };
      // A: weight rows [tile*128, +128) x chunks [u*KC, u*KC + KC) of the tile's matrix
      // (the tile after the last of an odd tile count is read past the end: zero fill, no traffic)
      auto load_w = [&](uint32_t dst, int tt, int u, int slot_) {
        const bool first = tt < p.t1;
        const int row0 = first ? tt * kBM : (p.n2 > 0 ? (tt - p.t1) * kBM : p.t1 * kBM);
        load(dst, first ? &map_w : &map_w2, row0, u * p.cps, slot_, pol_w);
      };
      // stages v = unit * sub + i, covering chunks [v cps, (v + 1) cps)
      const int npre = p.early_w ? min(p.ns, (jb.z - jb.y) * sub) : 0;
      for (int s = 0; s < npre; ++s) {
        if (leader) expect_tx(full0 + 8u * s, expect);
        load_w(ring_u32 + s * p.stage_bytes, jb.x, jb.y * sub + s, s);
      }
      grid_dependency_wait();
      int slot = 0, phase = 0, s = 0;
      for (bool have = true; have;) {
        const int tile = jb.x;
        for (int u = jb.y * sub; u < jb.z * sub; ++u, ++s) {
          if (s >= p.ns && !wait(empty0 + 8u * slot, phase ^ 1)) atomicOr(&umma_fault_word, 1);
          const uint32_t st = ring_u32 + slot * p.stage_bytes;
          // the full boxes always land (rows past n, rows past `rows` and a chunk past K are
          // zero-filled), so every stage completes exactly stage_bytes
          if (s >= npre) {
            if (leader) expect_tx(full0 + 8u * slot, expect);
            load_w(st, tile, u, slot);
          }
          // B: the activation rows (this CTA's half of them in a pair), the same chunks
          load(st + a_bytes, &map_x, kPair ? h * bn : 0, u * p.cps, slot, pol_x);
          if (++slot == p.ns) {
            slot = 0;
            phase ^= 1;
          }
        }
        have = next_job(jb);
        publish(have ? jb : make_int4(-1, 0, 0, -1));
      }
      const int nunits = s;
      // no copy may still be landing when the CTA exits: wait (bounded) for the last
      // phase of every slot (already complete in a healthy run, where the MMAs consumed it).
      // In a pair, rank 0's barriers count both CTAs' copies and the closing cluster barrier
      // holds rank 1 until rank 0 has seen them land.
      if (leader)
        for (int t = nunits - 1; t >= 0 && t >= nunits - p.ns; --t)
          if (!wait(full0 + 8u * (t % p.ns), (t / p.ns) & 1)) atomicOr(&umma_fault_word, 1);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (rank 0 of a pair issues for both CTAs)
    if (lane == 0 && leader) {
      const uint32_t idesc = kPair ? idesc_m256(p.nb) : idesc_m128(p.nb);
      int slot = 0, phase = 0;
      for (int i = 0;; ++i) {
        const int r = i % kJobRing;
        if (!wait(smem_u32(&bar_jfull[r]), (i / kJobRing) & 1)) {
          atomicOr(&umma_fault_word, 16);
          break;
        }
        const int4 jb = s_job[r];
        arrive(smem_u32(&bar_jempty[r]));
        if (jb.x < 0) break;
        const int u0 = jb.y, u1 = jb.z;
        const int acc = i & 1;
        if (i >= 2 && !wait(tempty0 + 8u * acc, ((i - 2) >> 1) & 1)) atomicOr(&umma_fault_word, 4);
        fence_after();
        const uint32_t tmem_d = tmem_base + (uint32_t)(acc * p.accw);
        for (int u = u0 * sub; u < u1 * sub; ++u) {  // stages
          if (!wait(full0 + 8u * slot, phase)) atomicOr(&umma_fault_word, 2);
          fence_after();
          const int nch = min(p.cps, kchunks - u * p.cps);  // <= 0: a stage wholly past K
          const uint32_t st = ring_u32 + slot * p.stage_bytes;
          for (int c = 0; c < nch; ++c) {
            const uint32_t a0 = st + c * kChunkBytesA;
            const uint32_t b0 = st + a_bytes + c * b_chunk;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // K = 32 bytes per MMA
              if constexpr (kPair)
                umma_f8_pair(tmem_d, desc_sw128(a0 + kk * 32), desc_sw128(b0 + kk * 32), idesc,
                             ((u - u0 * sub) | c | kk) != 0);
              else
                umma_f8(tmem_d, desc_sw128(a0 + kk * 32), desc_sw128(b0 + kk * 32), idesc,
                        ((u - u0 * sub) | c | kk) != 0);
            }
          }
          // the stage (of both CTAs) is free once these MMAs have read it
          if constexpr (kPair)
            commit_pair(empty0 + 8u * slot, 3);
          else
            commit(empty0 + 8u * slot);
          if (++slot == p.ns) {
            slot = 0;
            phase ^= 1;
          }
        }
        // the accumulator (of both CTAs) is complete
        if constexpr (kPair)
          commit_pair(tfull0 + 8u * acc, 3);
        else
          commit(tfull0 + 8u * acc);
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int lane_row = q * 32 + lane;
    grid_dependency_wait();  // x_scale comes from the preceding kernel
    for (int i = 0;; ++i) {
      const int r = i % kJobRing;
      if (!wait(smem_u32(&bar_jfull[r]), (i / kJobRing) & 1)) {
        atomicOr(&umma_fault_word, 16);
        break;
      }
      const int4 jb = s_job[r];
      __syncwarp();
      if (lane == 0) arrive(smem_u32(&bar_jempty[r]));
      if (jb.x < 0) break;
      const int tile = jb.x, ps = jb.w;
      const int acc = i & 1;
      if (!wait(tfull0 + 8u * acc, (i >> 1) & 1)) atomicOr(&umma_fault_word, 8);
      fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.accw);
      if (ps >= 0) {
        // partial tile: raw f32 sums of the used columns, [slot][col][128 rows]
        float* dst = p.partial + (int64_t)ps * p.nb * kBM + lane_row;
        for (int half = 0; half <= p.split; ++half) {
          const int cb = half * p.lo_off;
          for (int c0 = 0; c0 < p.npad; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(taddr + (uint32_t)(cb + c0), v);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              if (c0 + jj < p.rows) dst[(int64_t)(cb + c0 + jj) * kBM] = __uint_as_float(v[jj]);
          }
        }
      } else {
        const TileDst d = tile_dst(p, tile);
        const int row = d.row0 + lane_row;
        const float s = row < d.n ? d.scale[row] : 0.f;
        for (int c0 = 0; c0 < p.npad; c0 += 16) {
          uint32_t v[16];
          tmem_ld16(taddr + (uint32_t)c0, v);
          if (p.split) {  // y = hi-term sum + lo-term sum / 16
            uint32_t u[16];
            tmem_ld16(taddr + (uint32_t)(p.lo_off + c0), u);
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              v[jj] = __float_as_uint(fmaf(__uint_as_float(u[jj]), 0.0625f, __uint_as_float(v[jj])));
          }
          if (row < d.n) {
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int m = c0 + jj;
              if (m < p.rows) {
                const float y = (__uint_as_float(v[jj]) * s) * p.x_scale[m];
                d.out[(int64_t)m * d.ldc + row] = f32_to_bf16_bits(y);
              }
            }
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair)
          arrive_cluster(mapa_shared(tempty0 + 8u * acc, 0));  // rank 0's MMA thread waits on it
        else
          arrive(tempty0 + 8u * acc);
      }
    }
  }

  fence_before();
  __syncwarp();
  if constexpr (kPair)
    cluster_sync();  // neither CTA frees TMEM or exits while the pair's MMAs or arrivals may reach it
  else
    __syncthreads();
  fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (kPair)
      tmem_dealloc_pair(tmem_base, tmem_cols);
    else
      tmem_dealloc(tmem_base, tmem_cols);
  }
  if (dyn && threadIdx.x == 0) {  // this CTA claims no more tiles; the last one resets the queue
    __threadfence();
    if (atomicAdd(p.queue + 1, 1) == nctas - 1) {
      p.queue[0] = 0;
      p.queue[1] = 0;
    }
  }
}

// Remainder tiles: CTA (t, m) finishes remainder tile t for activation row m; thread r owns
// weight row r.  All partial sums of (r, m) are loaded first, then added in K order (the
// CTAs that ran the tile's units, lowest first), so the result does not depend on which CTA
// finished first, and the loads take one round trip.
constexpr int kMaxParts = 512;  // >= the party count (the host checks)
constexpr int kFixupBatch = 16;

// With the schedule over CTA pairs and tile pairs (P parties): CTA (2 t + h, m) finishes half h
// (single tile 2 T + h) of remainder tile pair t, whose sums are in the slots of CTA 2 j + h of
// each contributing party j.
__global__ void __launch_bounds__(kBM) umma_f8_fixup_kernel(const UmmaParams p, int P) {
  __shared__ int s_slot[kMaxParts];
  __shared__ int s_nparts;
  grid_dependents_launch();  // the next call's pre-pass may launch; it waits for this grid
  const Sched sc{p.spt, p.wt, p.rem, P};
  const int h = (int)(blockIdx.x & 1);
  const int t_rem = (int)(blockIdx.x >> 1), m = blockIdx.y;
  // Contributors of this tile (independent of the main kernel's data, so computed before the
  // dependency wait): consecutive CTAs from the owner of its first unit; thread i checks
  // candidate owner + i, i.e. the list is built in parallel, in K order.
  if (threadIdx.x == 0) s_nparts = 0;
  __syncthreads();
  {
    const int64_t tu0 = (int64_t)t_rem * p.spt, tu1 = tu0 + p.spt;
    const int b0 = sc.owner(tu0);
    for (int i = threadIdx.x; i < kMaxParts && b0 + i < P; i += kBM) {
      const int bb = b0 + i;
      const int64_t a = sc.r0(bb), e = sc.r0(bb + 1);
      if (a < tu1 && e > a) {  // non-empty range starting before the tile's end (it ends after tu0)
        s_slot[i] = 2 * (2 * bb + h) + (a / p.spt == t_rem ? 0 : 1);
        atomicMax(&s_nparts, i + 1);
      } else if (a < tu1) {
        s_slot[i] = -1;  // empty range inside the run: skipped
      }
      if (a >= tu1) break;
    }
  }
  __syncthreads();
  grid_dependency_wait();  // the partial sums and scales of the preceding kernels
  const TileDst d = tile_dst(p, 2 * (p.wt * P + t_rem) + h);
  const int row = d.row0 + threadIdx.x;
  if (row >= d.n) return;
  const int np = s_nparts;
  const float* base = p.partial + threadIdx.x;
  const int64_t slot_stride = (int64_t)p.nb * kBM;
  const int64_t off_hi = (int64_t)m * kBM, off_lo = (int64_t)(p.lo_off + m) * kBM;
  float hi = 0.f, lo = 0.f;
  for (int q0 = 0; q0 < np; q0 += kFixupBatch) {
    float vh[kFixupBatch], vl[kFixupBatch];
    bool ok[kFixupBatch];
#pragma unroll
    for (int j = 0; j < kFixupBatch; ++j) {
      vh[j] = vl[j] = 0.f;
      ok[j] = q0 + j < np && s_slot[q0 + j] >= 0;
      if (ok[j]) {
        const float* src = base + s_slot[q0 + j] * slot_stride;
        vh[j] = src[off_hi];
        if (p.split) vl[j] = src[off_lo];
      }
    }
#pragma unroll
    for (int j = 0; j < kFixupBatch; ++j) {
      if (ok[j]) {
        hi += vh[j];
        lo += vl[j];
      }
    }
  }
  const float acc = p.split ? fmaf(lo, 0.0625f, hi) : hi;
  d.out[(int64_t)m * d.ldc + row] = f32_to_bf16_bits((acc * d.scale[row]) * p.x_scale[m]);
}

constexpr size_t kUmmaSmemLimit = 232448 - 2048;

// Library-owned stream-ordered pool for the W8A16 activation codes and the stream-K partial
// sums of calls without a caller workspace (one per device; memory is kept between calls so
// that steady-state calls map nothing).
std::mutex g_pool_mu;
cudaMemPool_t g_pools[64] = {};

cudaMemPool_t scratch_pool(int dev) {
  if (dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_pool_mu);
  if (!g_pools[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t keep = ~uint64_t(0);
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pools[dev] = pool;
  }
  return g_pools[dev];
}

// The optional second weight matrix of a paired launch (same k, same activations).
struct SecondWeight {
  const uint8_t* w;
  const float* w_scale;
  int n;
  uint16_t* out;
  int64_t ldc;
};

int launch_umma_f8(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* b_codes, int64_t ldb,
                   int b_rows, const float* x_scale, int rows, int split, uint16_t* out, int64_t ldc, cudaStream_t s,
                   const UmmaScratch& scratch, int early_w, const SecondWeight* second = nullptr) {
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  UmmaParams p{};
  p.n = n;
  p.k = k;
  p.rows = rows;
  p.npad = (rows + 15) / 16 * 16;
  p.lo_off = (rows + 7) / 8 * 8;
  p.nb = umma_mma_n(split != 0, rows);
  // the epilogue reads 16 columns from lo_off + c0 (c0 < npad): keep that inside the
  // accumulator when lo_off is not a multiple of 16
  p.accw = tmem_cols_for(split && (p.lo_off % 16) ? p.nb + 16 : p.nb);
  if (2 * p.accw > 512) return DLMH_ERR_UNSUPPORTED;
  p.split = split;
  p.early_w = early_w;
  const bool pair = umma_pair_mode(p.nb, di.sms);
  const int bn = pair ? p.nb / 2 : p.nb;  // activation rows in each CTA's stages
  p.w_scale = w_scale;
  p.x_scale = x_scale;
  p.out = out;
  p.ldc = ldc;
  // a stage is a whole unit (the longest run of each weight row per copy) when the ring holds
  // two of them and half units would not put more bytes in the ring, else half a unit (at
  // 32 activation rows a CTA: two 80 KB units, or five 40 KB halves)
  const size_t unit = (size_t)kKC * (kChunkBytesA + bn * 128);
  const size_t whole = kUmmaSmemLimit / unit, halves = kUmmaSmemLimit / (unit / 2);
  p.cps = whole >= 2 && halves <= 2 * whole ? kKC : kKC / 2;
  p.stage_bytes = p.cps * (kChunkBytesA + bn * 128);
  int ns = (int)(kUmmaSmemLimit / (size_t)p.stage_bytes);
  if (ns > kMaxUStages) ns = kMaxUStages;
  if (ns < 2) return DLMH_ERR_UNSUPPORTED;
  p.ns = ns;
  CUtensorMap mw, mw2, mx;
  if (!cached_map_k128(&mw, w, 1, n, k, k, kBM, p.cps) || !cached_map_k128(&mx, b_codes, 1, b_rows, k, ldb, bn, p.cps))
    return DLMH_ERR_CUDA;
  p.t1 = (n + kBM - 1) / kBM;
  if (second) {
    if (!cached_map_k128(&mw2, second->w, 1, second->n, k, k, kBM, p.cps)) return DLMH_ERR_CUDA;
    p.n2 = second->n;
    p.w_scale2 = second->w_scale;
    p.out2 = second->out;
    p.ldc2 = second->ldc;
  } else {
    mw2 = mw;
  }
  const size_t smem = (size_t)ns * p.stage_bytes + 1024;
  const void* kfn = pair ? reinterpret_cast<const void*>(umma_f8_kernel<true>)
                        : reinterpret_cast<const void*>(umma_f8_kernel<false>);
  if (ensure_dynamic_smem(kfn, (int)smem) != DLMH_OK) return DLMH_ERR_CUDA;
  // schedule: whole tiles in full waves over the SMs (or SM pairs, over tile pairs), the rest
  // split into units
  const int ntiles = p.t1 + (second ? (second->n + kBM - 1) / kBM : 0);
  p.spt = (k / 128 + kKC - 1) / kKC;
  const Sched sched = umma_schedule(ntiles, k, di.sms);
  const int P = sched.G;  // parties: CTA pairs
  if (P > kMaxParts) return DLMH_ERR_UNSUPPORTED;
  p.wt = sched.wt;
  p.rem = sched.rem;
  // whole tiles from the caller workspace's queue when there is one (both orders give the
  // same outputs); the static order otherwise, and always for pairs
  p.queue = !pair && p.wt > 0 ? scratch.queue : nullptr;
  void* ws = nullptr;
  const size_t need = (size_t)umma_partial_bytes(split != 0, ntiles, k, rows, di.sms);
  if (p.rem > 0 && scratch.caller) {
    if (!scratch.partial || scratch.partial_cap < need) return DLMH_ERR_WORKSPACE;
    p.partial = scratch.partial;
  } else if (p.rem > 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DLMH_ERR_CUDA;
    cudaMemPool_t pool = scratch_pool(dev);
    if (!pool) return DLMH_ERR_CUDA;
    if (cudaMallocFromPoolAsync(&ws, need, pool, s) != cudaSuccess)
      return DLMH_ERR_CUDA;
    p.partial = static_cast<float*>(ws);
  }
  int rc = pair ? launch_pdl_cluster(2, umma_f8_kernel<true>, dim3(2 * P), dim3(kUmmaThreads), smem, s, mw, mw2, mx, p)
                : launch_pdl(umma_f8_kernel<false>, dim3(2 * P), dim3(kUmmaThreads), smem, s, mw, mw2, mx, p);
  if (rc == DLMH_OK && p.rem > 0) {
    rc = launch_pdl(umma_f8_fixup_kernel, dim3(2 * p.rem, rows), dim3(kBM), 0, s, p, P);
  }
  if (ws && cudaFreeAsync(ws, s) != cudaSuccess && rc == DLMH_OK) rc = DLMH_ERR_CUDA;
  return rc;
}

}  // namespace

bool w8a8_umma_supported(int k) {
  // whole 128-byte K chunks (the tensor map's innermost box); a pure function of k so that
  // every row count of a given weight takes this kernel
  return k > 0 && k % 128 == 0;
}

bool w8a16_umma_supported(int k) { return k > 0 && k % 128 == 0; }

int w8a8_umma_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
                   const float* x_scale, int rows, uint16_t* out, int64_t ldc, cudaStream_t s,
                   const UmmaScratch& scratch, bool after_prepass) {
  if (rows < 1 || rows > 128) return DLMH_ERR_ROWS;
  if (!w8a8_umma_supported(k)) return DLMH_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(w) & 15u) || (reinterpret_cast<uintptr_t>(xq) & 15u) || ldq % 16 != 0)
    return DLMH_ERR_ALIGN;
  return launch_umma_f8(w, w_scale, n, k, xq, ldq, rows, x_scale, rows, 0, out, ldc, s, scratch,
                        after_prepass ? 1 : 0);
}

int w8a8_umma_pair_pass(const uint8_t* w1, const float* s1, int n1, uint16_t* out1, int64_t ldc1,
                        const uint8_t* w2, const float* s2, int n2, uint16_t* out2, int64_t ldc2, int k,
                        const uint8_t* xq, int64_t ldq, const float* x_scale, int rows, cudaStream_t s,
                        const UmmaScratch& scratch, bool after_prepass) {
  if (rows < 1 || rows > 128) return DLMH_ERR_ROWS;
  if (!w8a8_umma_supported(k)) return DLMH_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(w1) & 15u) || (reinterpret_cast<uintptr_t>(w2) & 15u) ||
      (reinterpret_cast<uintptr_t>(xq) & 15u) || ldq % 16 != 0)
    return DLMH_ERR_ALIGN;
  const SecondWeight second{w2, s2, n2, out2, ldc2};
  return launch_umma_f8(w1, s1, n1, k, xq, ldq, rows, x_scale, rows, 0, out1, ldc1, s, scratch,
                        after_prepass ? 1 : 0, &second);
}

int w8a16_umma_run(const uint8_t* w, const float* w_scale, int n, int k, const uint16_t* x, int64_t ldx, int rows,
                   uint16_t* out, int64_t ldc, cudaStream_t s, const UmmaScratch& scratch) {
  if (!w8a16_umma_supported(k)) return DLMH_ERR_SHAPE;
  if (rows <= 0) return DLMH_OK;
  if ((reinterpret_cast<uintptr_t>(w) & 15u) || (reinterpret_cast<uintptr_t>(x) & 15u) || ldx % 8 != 0)
    return DLMH_ERR_ALIGN;
  const int first = rows < 128 ? rows : 128;
  const size_t code_bytes = (size_t)2 * ((first + 7) / 8 * 8) * k;  // a multiple of 256 (k % 128 == 0)
  void* pooled = nullptr;
  uint8_t* codes = nullptr;
  if (scratch.caller) {
    if (!scratch.codes || scratch.codes_cap < (size_t)w8a16_code_bytes(first, k)) return DLMH_ERR_WORKSPACE;
    codes = scratch.codes;
  } else {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DLMH_ERR_CUDA;
    cudaMemPool_t pool = scratch_pool(dev);
    if (!pool) return DLMH_ERR_CUDA;
    if (cudaMallocFromPoolAsync(&pooled, code_bytes + 128 * sizeof(float), pool, s) != cudaSuccess)
      return DLMH_ERR_CUDA;
    codes = static_cast<uint8_t*>(pooled);
  }
  float* x_mul = reinterpret_cast<float*>(codes + code_bytes);
  int rc = DLMH_OK;
  for (int done = 0; done < rows && rc == DLMH_OK;) {
    const int m = rows - done < 128 ? rows - done : 128;
    const int half = (m + 7) / 8 * 8;  // hi rows [0, half), lo rows [half, 2 half)
    rc = w8a16_split_launch(x + (int64_t)done * ldx, ldx, m, k, half, codes, x_mul, s);
    if (rc == DLMH_OK)
      rc = launch_umma_f8(w, w_scale, n, k, codes, k, 2 * half, x_mul, m, 1, out + (int64_t)done * ldc, ldc, s,
                          scratch, 1);
    done += m;
  }
  if (pooled && cudaFreeAsync(pooled, s) != cudaSuccess && rc == DLMH_OK) rc = DLMH_ERR_CUDA;
  return rc;
}

int pool_stats(int64_t* used_current, int64_t* used_high, int reset_high) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DLMH_ERR_CUDA;
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_pool_mu);
    pool = g_pools[dev];
  }
  uint64_t cur = 0, high = 0;
  if (pool) {
    if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemCurrent, &cur) != cudaSuccess ||
        cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &high) != cudaSuccess)
      return DLMH_ERR_CUDA;
    if (reset_high) {
      uint64_t zero = 0;
      if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero) != cudaSuccess) return DLMH_ERR_CUDA;
    }
  }
  if (used_current) *used_current = (int64_t)cur;
  if (used_high) *used_high = (int64_t)high;
  return DLMH_OK;
}

namespace {

// One thread waits (bounded) on an mbarrier that nothing will ever complete.
__global__ void bounded_wait_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  bar_init(b, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (!wait(b, 0)) atomicOr(&umma_fault_word, kWaitProbeBit);
}

}  // namespace

int bounded_wait_check(cudaStream_t s) {
  int before = 0;
  if (cudaMemcpyFromSymbol(&before, umma_fault_word, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  bounded_wait_probe_kernel<<<1, 1, 0, s>>>();
  if (launch_status() != DLMH_OK || cudaStreamSynchronize(s) != cudaSuccess) return DLMH_ERR_CUDA;
  int after = 0;
  if (cudaMemcpyFromSymbol(&after, umma_fault_word, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  const int restored = before & ~kWaitProbeBit;  // leave the other bits as they were
  if (cudaMemcpyToSymbol(umma_fault_word, &restored, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  return (after & kWaitProbeBit) ? DLMH_OK : DLMH_ERR_CUDA;
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
