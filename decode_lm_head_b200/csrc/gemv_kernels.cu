// Launchers for the row-tile GEMV kernels (FP8 W8A16, W8A8, NVFP4 W4A16).
#include <mutex>

#include "gemv_launch.h"
#include "rowtile_gemv.cuh"

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

// The tier table is a pure function of the shape, so the host plan (dlmh_plan_chunks, no
// GPU needed) and the launches agree: it uses the sm_100 shared-memory limit per block.
constexpr size_t kSmemLimit = 232448 - 1024;

namespace {

constexpr int kPrefetch = 4;

template <class F, int NT>
int launch_rowtile(const RowTileParams& p, cudaStream_t stream) {
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  const size_t smem = rowtile_smem_bytes<F, NT>(p.k);
  if (smem > kSmemLimit || smem + 256 > (size_t)di.smem_optin) return DLMH_ERR_UNSUPPORTED;
  auto kern = rowtile_gemv_kernel<F, NT, kPrefetch>;
  // Setting the attribute is cheap and idempotent; do it per call so every device is covered.
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return DLMH_ERR_CUDA;
  const int ntiles = (p.n + kTileRows - 1) / kTileRows;
  const int grid = ntiles < di.sms ? ntiles : di.sms;
  kern<<<grid, kThreads, smem, stream>>>(p);
  return launch_status();
}

template <class F>
int launch_tier(int nt, const RowTileParams& p, cudaStream_t s) {
  switch (nt) {
    case 1: return launch_rowtile<F, 1>(p, s);
    case 2: return launch_rowtile<F, 2>(p, s);
    case 4: return launch_rowtile<F, 4>(p, s);
    default: return DLMH_ERR_UNSUPPORTED;
  }
}

template <class F>
bool tier_fits(int nt, int k) {
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
    default: return 0;
  }
}

}  // namespace dlmh
