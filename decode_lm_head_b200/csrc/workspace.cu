// Caller-owned workspace of the tensor-core passes: sizing, the per-stream binding, and the
// scratch each call takes from it.
//
// A decode engine sizes one workspace per stream (dlmh_workspace_bytes, the largest shape its
// calls use), binds it once (dlmh_set_workspace), and from then on the FP8 calls on that
// stream take their W8A16 activation codes, stream-K partial sums and whole-tile queue from
// it: no call allocates.  Streams without a workspace keep the library pool.
#include <mutex>

#include "dlmh_common.cuh"
#include "gemv_launch.h"
#include "workspace_plan.h"

namespace dlmh {
namespace {

struct Binding {
  int dev;
  unsigned long long stream_id;
  cudaStream_t handle;
  uint8_t* ws;
  size_t bytes;
};

constexpr int kMaxBindings = 1024;
std::mutex g_mu;
Binding g_bind[kMaxBindings];
int g_nbind = 0;

// A stream's key: cudaStreamGetId (unique within the context, never reused after the stream
// is destroyed); the legacy default stream, which has no id, keys as ~0.  Not called while
// the stream is being captured (the query would invalidate the capture).
int stream_key(cudaStream_t s, int* dev, unsigned long long* id) {
  if (cudaGetDevice(dev) != cudaSuccess) return DLMH_ERR_CUDA;
  if (cudaStreamGetId(s, id) != cudaSuccess) {
    (void)cudaGetLastError();
    if (s != nullptr && s != cudaStreamLegacy) return DLMH_ERR_CUDA;
    *id = ~0ull;
  }
  return DLMH_OK;
}

int find(int dev, unsigned long long id) {
  for (int i = 0; i < g_nbind; ++i)
    if (g_bind[i].dev == dev && g_bind[i].stream_id == id) return i;
  return -1;
}

// During capture the stream's id cannot be queried: the binding is found by its handle.
int find_handle(int dev, cudaStream_t s) {
  for (int i = 0; i < g_nbind; ++i)
    if (g_bind[i].dev == dev && g_bind[i].handle == s) return i;
  return -1;
}

bool uses_tensor_cores(int op, int k) {
  if (op == DLMH_OP_W8A16) return w8a16_umma_supported(k);
  if (op == DLMH_OP_W8A8 || op == DLMH_OP_W8A8_PAIR) return w8a8_umma_supported(k);
  return false;
}

int tiles_of(int op, int n) {
  const int t = (n + kUmmaTileRows - 1) / kUmmaTileRows;
  return op == DLMH_OP_W8A8_PAIR ? 2 * t : t;
}

}  // namespace

int call_scratch(int op, int n, int k, int rows, cudaStream_t s, UmmaScratch* out) {
  *out = UmmaScratch{};
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return DLMH_ERR_CUDA;
  const bool capturing = cs != cudaStreamCaptureStatusNone;
  int dev = 0;
  unsigned long long id = 0;
  if (capturing) {
    if (cudaGetDevice(&dev) != cudaSuccess) return DLMH_ERR_CUDA;
  } else if (stream_key(s, &dev, &id) != DLMH_OK) {
    return DLMH_OK;  // no binding can exist: the pool
  }
  Binding b{};
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const int i = capturing ? find_handle(dev, s) : find(dev, id);
    if (i < 0) return DLMH_OK;
    b = g_bind[i];
  }
  const DeviceInfo di = device_info();
  if (di.sms <= 0) return DLMH_ERR_CUDA;
  const WsLayout L = ws_layout(op == DLMH_OP_W8A16, tiles_of(op, n), k, rows, di.sms);
  if ((int64_t)b.bytes < L.total) return DLMH_ERR_WORKSPACE;
  out->caller = true;
  // a captured launch takes the static tile order: a graph holds no counter, so replays of it
  // may run anywhere; both orders give the same outputs
  out->queue = capturing ? nullptr : reinterpret_cast<int*>(b.ws);
  out->codes = b.ws + L.codes_off;
  out->codes_cap = (size_t)L.codes_bytes;
  out->partial = reinterpret_cast<float*>(b.ws + L.partial_off);
  out->partial_cap = (size_t)L.partial_bytes;
  return DLMH_OK;
}

}  // namespace dlmh

extern "C" {

int64_t dlmh_workspace_bytes(int op, int n, int k, int rows, int sm_count) {
  if (op < DLMH_OP_W8A16 || op > DLMH_OP_W8A8_PAIR) return DLMH_ERR_SHAPE;
  if (n <= 0 || k <= 0 || sm_count < 0) return DLMH_ERR_SHAPE;
  if (rows < 0) return DLMH_ERR_ROWS;
  if (rows == 0 || !dlmh::uses_tensor_cores(op, k)) return 0;
  int sms = sm_count;
  if (sms == 0) {
    sms = dlmh::device_info().sms;
    if (sms <= 0) return DLMH_ERR_CUDA;
  }
  return dlmh::ws_layout(op == DLMH_OP_W8A16, dlmh::tiles_of(op, n), k, rows, sms).total;
}

int dlmh_set_workspace(void* ws, size_t bytes, void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int dev = 0;
  unsigned long long id = 0;
  if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)) return DLMH_ERR_ALIGN;
  if (ws && bytes < (size_t)dlmh::kWsQueueBytes) return DLMH_ERR_WORKSPACE;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    (void)cudaGetLastError();
    return DLMH_ERR_CUDA;
  }
  if (cs != cudaStreamCaptureStatusNone) return DLMH_ERR_UNSUPPORTED;
  if (dlmh::stream_key(s, &dev, &id) != DLMH_OK) return DLMH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(dlmh::g_mu);
  const int i = dlmh::find(dev, id);
  if (!ws) {  // unbind: the stream's calls go back to the pool
    if (i >= 0) dlmh::g_bind[i] = dlmh::g_bind[--dlmh::g_nbind];
    return DLMH_OK;
  }
  if (i < 0 && dlmh::g_nbind == dlmh::kMaxBindings) return DLMH_ERR_CAPACITY;
  // the tile queue starts at zero (every launch leaves it there), in stream order
  if (cudaMemsetAsync(ws, 0, dlmh::kWsQueueBytes, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return DLMH_ERR_CUDA;
  }
  const dlmh::Binding b{dev, id, s, static_cast<uint8_t*>(ws), bytes};
  if (i >= 0)
    dlmh::g_bind[i] = b;
  else
    dlmh::g_bind[dlmh::g_nbind++] = b;
  return DLMH_OK;
}

int dlmh_pool_stats(int64_t* used_current, int64_t* used_high, int reset_high) {
  return dlmh::pool_stats(used_current, used_high, reset_high);
}

}  // extern "C"
