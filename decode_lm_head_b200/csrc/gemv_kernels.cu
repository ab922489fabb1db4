// Launchers for the row-tile GEMV kernels (FP8 W8A16, W8A8, NVFP4 W4A16).
#include <mutex>

#include "gemv_launch.h"
#include "rowtile_gemv.cuh"
#include "rowtile_tma.cuh"
#include "umma_common.cuh"

namespace dlmh {


DeviceInfo device_info() {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool have[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DeviceInfo{};
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    DeviceInfo d;
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cache[dev] = d;
    have[dev] = true;
  }
  return cache[dev];
}

int ensure_dynamic_smem(const void* fn, int bytes) {
  struct Entry {
    const void* fn;
    int dev;
    int bytes;
  };
  static std::mutex mu;
  static Entry done[256];
  static int count = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DLMH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  Entry* e = nullptr;
  for (int i = 0; i < count; ++i)
    if (done[i].fn == fn && done[i].dev == dev) e = &done[i];
  if (e && e->bytes >= bytes) return DLMH_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return DLMH_ERR_CUDA;
  if (!e && count < 256) e = &done[count++];
  if (e) *e = Entry{fn, dev, bytes};
  return DLMH_OK;
}

// The tier table is a pure function of the shape, so the host plan (dlmh_plan_chunks, no
// GPU needed) and the launches agree: it uses the sm_100 shared-memory limit per block.
constexpr size_t kSmemLimit = 232448 - 1024;

namespace {

// Depth of the register ring in k-blocks (1 KB of weight per warp each for FP8 / W8A8):
// 8 keeps ~128 KB in flight per SM.  The 32-row tier runs a shallower ring to stay within
// 128 registers per thread.
#ifndef DLMH_PREFETCH
#define DLMH_PREFETCH 8
#endif
constexpr int kPrefetch = DLMH_PREFETCH;
template <class F, int NT>
constexpr int prefetch_depth() {
  return NT >= 4 ? 4 : (F::kBlockScale ? (kPrefetch < 6 ? kPrefetch : 6) : kPrefetch);
}

template <class F, int NT>
int launch_rowtile(const RowTileParams& p, cudaStream_t stream) {
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  const size_t smem = rowtile_smem_bytes<F, NT>(p.k);
  if (smem > kSmemLimit || smem + 256 > (size_t)di.smem_optin) return DLMH_ERR_UNSUPPORTED;
  auto kern = rowtile_gemv_kernel<F, NT, prefetch_depth<F, NT>()>;
  // Setting the attribute is cheap and idempotent; do it per call so every device is covered.
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem) != DLMH_OK) return DLMH_ERR_CUDA;
  const int ntiles = (p.n + kTileRows - 1) / kTileRows;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  kern<<<grid, kThreads, smem, stream>>>(p);
  return launch_status();
}

// ---- streamed (TMA ring) kernels: which (format, n-tiles, k-blocks per warp) exist

// Largest k-blocks-per-warp instantiated for (format, n-tiles): keeps the register-resident
// activation fragments (x_words * NT * NKB registers) within the 128-register budget of a
// 512-thread CTA without spills (checked with -Xptxas -v).
template <class F, int NT>
constexpr int stream_max_nkb() {
  if constexpr (F::kXBytes == 0) return NT == 1 ? 7 : (NT == 2 ? 3 : 2);  // W4A4: 5 words per (k-block, n-tile)
  else if constexpr (F::kBlockScale) return NT == 1 ? 5 : (NT == 2 ? 2 : 0);
  else if constexpr (F::kXBytes == 1) return NT <= 2 ? 8 : 3;
  else return NT == 1 ? 7 : (NT == 2 ? 5 : 2);
}

template <class F, int NT, int C>
constexpr int stream_stages_for() {
  constexpr size_t other = stream_smem_bytes<F, NT, C, 0>();
  constexpr size_t room = kSmemLimit > other ? kSmemLimit - other : 0;
  constexpr int ns = (int)(room / (StageLayout<F, C>::kBytes + 16));
  return ns > 8 ? 8 : ns;
}

// Slots per stage: the whole tile when two tiles fit in the ring (row copies of NKB KB),
// else the largest C with at least three stages, else 2.
template <class F, int NT, int NKB>
constexpr int stream_slots() {
#ifdef DLMH_STREAM_C
  return DLMH_STREAM_C < NKB ? DLMH_STREAM_C : NKB;
#else
  if constexpr (stream_stages_for<F, NT, NKB>() >= 2) return NKB;
  else if constexpr (NKB >= 4 && stream_stages_for<F, NT, 4>() >= 3) return 4;
  else if constexpr (NKB >= 3 && stream_stages_for<F, NT, 3>() >= 3) return 3;
  else return NKB >= 2 ? 2 : 1;
#endif
}

template <class F, int NT, int NKB>
int launch_stream_nkb(const RowTileParams& p, cudaStream_t stream) {
  constexpr int C = stream_slots<F, NT, NKB>();
  constexpr int NS = stream_stages_for<F, NT, C>();
  static_assert(NS >= 2, "ring too shallow");
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  const size_t smem = stream_smem_bytes<F, NT, C, NS>();
  auto kern = stream_gemv_kernel<F, NT, NKB, C, NS>;
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem) != DLMH_OK) return DLMH_ERR_CUDA;
  const int ntiles = (p.n + kTileRows - 1) / kTileRows;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  return umma::launch_pdl(kern, dim3(grid), dim3(kThreads), smem, stream, p);
}

template <class F, int NT>
int launch_stream(int nkb, const RowTileParams& p, cudaStream_t s) {
  constexpr int kMax = stream_max_nkb<F, NT>();
  switch (nkb) {
    case 1: if constexpr (kMax >= 1) return launch_stream_nkb<F, NT, 1>(p, s); break;
    case 2: if constexpr (kMax >= 2) return launch_stream_nkb<F, NT, 2>(p, s); break;
    case 3: if constexpr (kMax >= 3) return launch_stream_nkb<F, NT, 3>(p, s); break;
    case 4: if constexpr (kMax >= 4) return launch_stream_nkb<F, NT, 4>(p, s); break;
    case 5: if constexpr (kMax >= 5) return launch_stream_nkb<F, NT, 5>(p, s); break;
    case 6: if constexpr (kMax >= 6) return launch_stream_nkb<F, NT, 6>(p, s); break;
    case 7: if constexpr (kMax >= 7) return launch_stream_nkb<F, NT, 7>(p, s); break;
    case 8: if constexpr (kMax >= 8) return launch_stream_nkb<F, NT, 8>(p, s); break;
    default: break;
  }
  return DLMH_ERR_UNSUPPORTED;
}

// k-blocks per warp of the streamed kernel at reduction length k, or 0 if it cannot run k
// (FP4 needs 16-byte-aligned block-scale rows: k % 256 == 0).
template <class F>
int stream_nkb(int k) {
  if (F::kBlockScale && k % 256 != 0) return 0;
  const int kb = kblocks_of<F>(k);
  return (kb + kWarps - 1) / kWarps;
}

template <class F>
bool stream_fits(int nt, int k) {
  const int nkb = stream_nkb<F>(k);
  if (nkb <= 0) return false;
  switch (nt) {
    case 1: return nkb <= stream_max_nkb<F, 1>();
    case 2: return nkb <= stream_max_nkb<F, 2>();
    case 4: return nkb <= stream_max_nkb<F, 4>();
    default: return false;
  }
}

template <class F>
int launch_tier(int nt, const RowTileParams& p, cudaStream_t s) {
  if (stream_fits<F>(nt, p.k)) {
    const int nkb = stream_nkb<F>(p.k);
    switch (nt) {
      case 1: return launch_stream<F, 1>(nkb, p, s);
      case 2: return launch_stream<F, 2>(nkb, p, s);
      case 4: return launch_stream<F, 4>(nkb, p, s);
      default: break;
    }
  }
  switch (nt) {
    case 1: return launch_rowtile<F, 1>(p, s);
    case 2: return launch_rowtile<F, 2>(p, s);
    case 4: return launch_rowtile<F, 4>(p, s);
    default: return DLMH_ERR_UNSUPPORTED;
  }
}

// The streamed kernel alone (W4A4 has no register-tile fallback).
template <class F>
int launch_tier_stream(int nt, const RowTileParams& p, cudaStream_t s) {
  if (!stream_fits<F>(nt, p.k)) return DLMH_ERR_UNSUPPORTED;
  const int nkb = stream_nkb<F>(p.k);
  switch (nt) {
    case 1: return launch_stream<F, 1>(nkb, p, s);
    case 2: return launch_stream<F, 2>(nkb, p, s);
    case 4: return launch_stream<F, 4>(nkb, p, s);
    default: return DLMH_ERR_UNSUPPORTED;
  }
}

template <class F>
bool tier_fits(int nt, int k) {
  if (stream_fits<F>(nt, k)) return true;
  size_t smem = 0;
  switch (nt) {
    case 1: smem = rowtile_smem_bytes<F, 1>(k); break;
    case 2: smem = rowtile_smem_bytes<F, 2>(k); break;
    case 4: smem = rowtile_smem_bytes<F, 4>(k); break;
    default: return false;
  }
  return smem <= kSmemLimit;
}

}  // namespace

// n-tiles (8 rows each) of the narrowest compiled tier covering `rows`.
int tier_ntiles(int rows) { return rows <= 8 ? 1 : (rows <= 16 ? 2 : 4); }

int w8a16_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint16_t* x, int64_t ldx, int rows,
               uint16_t* out, int64_t ldc, cudaStream_t s) {
  RowTileParams p{};
  p.w = w;
  p.w_row_bytes = k;
  p.w_scale = w_scale;
  p.n = n;
  p.k = k;
  p.x = x;
  p.ldx = ldx;
  p.rows = rows;
  p.out = out;
  p.ldc = ldc;
  return launch_tier<FmtW8A16>(tier_ntiles(rows), p, s);
}

int w8a8_gemv_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
                   const float* x_scale, int rows, uint16_t* out, int64_t ldc, cudaStream_t s) {
  RowTileParams p{};
  p.w = w;
  p.w_row_bytes = k;
  p.w_scale = w_scale;
  p.n = n;
  p.k = k;
  p.x = xq;
  p.ldx = ldq;
  p.x_scale = x_scale;
  p.rows = rows;
  p.out = out;
  p.ldc = ldc;
  return launch_tier<FmtW8A8>(tier_ntiles(rows), p, s);
}

int w4a16_pass(const uint8_t* wp, const uint8_t* wbs, float g, int n, int k, const uint16_t* x, int64_t ldx, int rows,
               uint16_t* out, int64_t ldc, cudaStream_t s) {
  RowTileParams p{};
  p.w = wp;
  p.w_row_bytes = k / 2;
  p.w_bscale = wbs;
  p.gscale = g;
  p.n = n;
  p.k = k;
  p.x = x;
  p.ldx = ldx;
  p.rows = rows;
  p.out = out;
  p.ldc = ldc;
  return launch_tier<FmtW4A16>(tier_ntiles(rows), p, s);
}

int w4a4_pass(const uint8_t* wp, const uint8_t* wbs, float g, int n, int k, const uint8_t* xq,
              const uint8_t* xbs, const float* xg, int rows, uint16_t* out, int64_t ldc, cudaStream_t s,
              bool after_prepass) {
  RowTileParams p{};
  p.w = wp;
  p.w_row_bytes = k / 2;
  p.w_bscale = wbs;
  p.gscale = g;
  p.n = n;
  p.k = k;
  p.x = xq;
  p.ldx = k;  // codes row stride: k/2 bytes
  p.x_bscale = xbs;
  p.x_scale = xg;
  p.rows = rows;
  p.out = out;
  p.ldc = ldc;
  p.early_w = after_prepass ? 1 : 0;
  return launch_tier_stream<FmtW4A4>(tier_ntiles(rows), p, s);
}

int device_fault(int reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, dlmh_fault_word, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  if (reset) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(dlmh_fault_word, &zero, sizeof(int)) != cudaSuccess) return DLMH_ERR_CUDA;
  }
  const int u = umma_fault(reset);
  if (u < 0) return u;
  const int q6 = q6k_fault(reset);
  if (q6 < 0) return q6;
  return v | (u << 8) | (q6 << 16);
}

int max_tier_rows(int op, int k) {
  auto widest = [&](auto fits) {
    if (fits(4)) return 32;
    if (fits(2)) return 16;
    if (fits(1)) return 8;
    return 0;
  };
  switch (op) {
    case DLMH_OP_W8A16: return widest([&](int nt) { return tier_fits<FmtW8A16>(nt, k); });
    case DLMH_OP_W8A8: return widest([&](int nt) { return tier_fits<FmtW8A8>(nt, k); });
    case DLMH_OP_W4A16: return widest([&](int nt) { return tier_fits<FmtW4A16>(nt, k); });
    case DLMH_OP_W4A4: return widest([&](int nt) { return stream_fits<FmtW4A4>(nt, k); });
    default: return 0;
  }
}

}  // namespace dlmh
