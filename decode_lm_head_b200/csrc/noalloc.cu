// w8a8_proj_noalloc: the W8A8 projection with its activation scratch in a fixed
// device-global array of this library, for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc:
// - engines whose device memory is owned by a pre-reserved pool or another framework's
//   allocator, which forbids foreign allocations;
// - latency-critical decode loops, where cudaMalloc's implicit device-wide synchronization
//   is not acceptable.
// They still pass their inputs and outputs.  The 128-row quantized-activation scratch that
// w8a8_proj normally takes from the caller lives here instead, in
// g_w8a8_noalloc_scratch.  Every GPU that loads the library holds this array until the
// process exits.
//
// The array's name is a host-side stand-in in host code, not a device address.  Its
// device address is fetched once per device, with that device current, through
// cudaGetSymbolAddress.  A device's first call does that set-up.
#include <mutex>

#include "dlmh_common.cuh"
#include "gemv_launch.h"
#include "workspace_plan.h"

namespace {

constexpr size_t kCodeBytes = (size_t)DLMH_W8A8_MAX_ROWS * DLMH_NOALLOC_MAX_K;
constexpr size_t kScaleOffset = kCodeBytes;  // 256-byte aligned: kCodeBytes is a multiple of 256
constexpr size_t kScaleBytes = DLMH_W8A8_MAX_ROWS * sizeof(float);  // 512, keeps 256-byte alignment
constexpr size_t kPartialOffset = kCodeBytes + kScaleBytes;
// Partial sums of the tensor-core pass's stream-K remainder: two slots per CTA, 128 weight
// rows x up to 128 activation rows of f32 each, for up to DLMH_NOALLOC_MAX_SMS CTAs.
constexpr size_t kPartialBytes = (size_t)2 * DLMH_NOALLOC_MAX_SMS * 128 * DLMH_W8A8_MAX_ROWS * sizeof(float);
constexpr size_t kScratchBytes = kPartialOffset + kPartialBytes;
static_assert(kCodeBytes % 256 == 0, "scale block must stay aligned");
static_assert(kPartialOffset % 256 == 0, "partial area must stay aligned");

// Codes of up to 128 rows x DLMH_NOALLOC_MAX_K (row stride k), 128 float32 row scales, then
// the partial-sum area.
static __device__ __align__(256) uint8_t g_w8a8_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t* g_dev_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
int scratch_on_current_device(uint8_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DLMH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_dev_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_w8a8_noalloc_scratch) != cudaSuccess || !p) return DLMH_ERR_CUDA;
    g_dev_ptr[dev] = static_cast<uint8_t*>(p);
  }
  *out = g_dev_ptr[dev];
  return DLMH_OK;
}

}  // namespace

extern "C" int w8a8_proj_noalloc(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x,
                                 int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, void* stream) {
  if (rows < 0) return DLMH_ERR_ROWS;
  if (n <= 0 || k <= 0 || k % 16 != 0) return DLMH_ERR_SHAPE;
  if (k > DLMH_NOALLOC_MAX_K) return DLMH_ERR_UNSUPPORTED;
  if (rows == 0) return DLMH_OK;
  // The partial sums the tensor-core schedule of this shape needs on this device must fit the
  // fixed area; checked before any launch, so a refused call touches nothing.
  if (dlmh::w8a8_umma_supported(k)) {
    const int sms = dlmh::device_info().sms;
    if (sms <= 0) return DLMH_ERR_CUDA;
    const int ntiles = (n + dlmh::kUmmaTileRows - 1) / dlmh::kUmmaTileRows;
    const int widest = rows < DLMH_W8A8_MAX_ROWS ? rows : DLMH_W8A8_MAX_ROWS;
    if ((size_t)dlmh::umma_partial_bytes(false, ntiles, k, widest, sms) > kPartialBytes) return DLMH_ERR_UNSUPPORTED;
  }
  uint8_t* base = nullptr;
  const int rc = scratch_on_current_device(&base);
  if (rc != DLMH_OK) return rc;
  // Each chunk's quantize writes every code and scale the following GEMV reads, and every
  // partial sum is written before the fixup reads it, so nothing in the shared array has to
  // start at zero.  Whole tiles go in the static order (no queue to keep at zero).
  dlmh::UmmaScratch sc;
  sc.caller = true;
  sc.partial = reinterpret_cast<float*>(base + kPartialOffset);
  sc.partial_cap = kPartialBytes;
  return dlmh::w8a8_proj_fixed_scratch(w, w_scale, n, k, x, ldx, rows, out, ldc, base,
                                       reinterpret_cast<float*>(base + kScaleOffset), sc,
                                       static_cast<cudaStream_t>(stream));
}
