// The C ABI of libdlmh: argument checks, row chunking and tier choice, then launches.
// Host code only; every check runs before any launch, so a rejected call touches nothing.
#include <stdint.h>

#include "dlmh_common.cuh"
#include "gemv_launch.h"

using dlmh::aligned16;

namespace {

constexpr int kMaxK = 1 << 20;

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

int check_rows(int rows, int cap) {
  if (rows < 0) return DLMH_ERR_ROWS;
  if (cap > 0 && rows > cap) return DLMH_ERR_ROWS;
  return DLMH_OK;
}

int check_nk(int n, int k, int kmult) {
  if (n <= 0 || k <= 0 || k > kMaxK || k % kmult != 0) return DLMH_ERR_SHAPE;
  return DLMH_OK;
}

// x-like BF16 input: 16-byte aligned base, ld a multiple of 8 elements, ld >= k.
int check_bf16_in(const void* x, int64_t ld, int k) {
  if (!x) return DLMH_ERR_NULL;
  if (ld < k) return DLMH_ERR_LD;
  if (!aligned16(x) || ld % 8 != 0) return DLMH_ERR_ALIGN;
  return DLMH_OK;
}

int check_out(const void* out, int64_t ldc, int n) {
  if (!out) return DLMH_ERR_NULL;
  if (ldc < n) return DLMH_ERR_LD;
  if ((reinterpret_cast<uintptr_t>(out) & 1u) != 0) return DLMH_ERR_ALIGN;
  return DLMH_OK;
}

#define DLMH_TRY(expr)            \
  do {                            \
    const int rc_ = (expr);       \
    if (rc_ != DLMH_OK) return rc_; \
  } while (0)

// Rows per weight pass of each op at reduction length k (0 = not servable).
int pass_rows(int op, int k) {
  switch (op) {
    case DLMH_OP_W8A16: {
      if (dlmh::w8a16_umma_supported(k)) return 128;
      const int t = dlmh::max_tier_rows(DLMH_OP_W8A16, k);
      return t >= DLMH_W8A16_CHUNK_ROWS ? DLMH_W8A16_CHUNK_ROWS : 0;
    }
    case DLMH_OP_W8A8:
      return dlmh::w8a8_umma_supported(k) ? DLMH_W8A8_MAX_ROWS : dlmh::max_tier_rows(DLMH_OP_W8A8, k);
    case DLMH_OP_W4A16: return dlmh::max_tier_rows(DLMH_OP_W4A16, k);
    case DLMH_OP_W4A4: return k % 256 == 0 ? dlmh::max_tier_rows(DLMH_OP_W4A4, k) : 0;
    case DLMH_OP_Q6K: return DLMH_Q6K_MAX_ROWS;
    default: return 0;
  }
}


}  // namespace

extern "C" {

int dlmh_version(void) { return 100; }

int dlmh_device_fault(int reset) { return dlmh::device_fault(reset); }

int dlmh_check_bounded_wait(void* stream) { return dlmh::bounded_wait_check(as_stream(stream)); }

const char* dlmh_error_string(int code) {
  switch (code) {
    case DLMH_OK: return "ok";
    case DLMH_ERR_NULL: return "a required pointer is NULL";
    case DLMH_ERR_SHAPE: return "invalid shape (n, k or the format's k multiple)";
    case DLMH_ERR_ALIGN: return "a pointer or leading dimension breaks the required alignment";
    case DLMH_ERR_ROWS: return "rows is negative or above the entry point's cap";
    case DLMH_ERR_LD: return "a leading dimension is smaller than the row it holds";
    case DLMH_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case DLMH_ERR_UNSUPPORTED: return "shape beyond this build's on-chip limits";
    case DLMH_ERR_CAPACITY: return "output array or table too small";
    case DLMH_ERR_WORKSPACE: return "the stream's workspace is smaller than the call needs (dlmh_workspace_bytes)";
    default: return "unknown status";
  }
}

int dlmh_plan_chunks(int op, int rows, int k, int* offsets, int* counts, int* tiers, int cap) {
  if (op < DLMH_OP_W8A16 || op > DLMH_OP_W8A8_PAIR) return DLMH_ERR_SHAPE;
  if (k <= 0) return DLMH_ERR_SHAPE;
  DLMH_TRY(check_rows(rows, 0));
  if (op == DLMH_OP_W8A8_PAIR) op = DLMH_OP_W8A8;  // the pair runs w8a8_proj's passes
  const int width = pass_rows(op, k);
  if (width <= 0) return DLMH_ERR_UNSUPPORTED;
  int nchunks = 0;
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    if (nchunks < cap) {
      if (!offsets || !counts || !tiers) return DLMH_ERR_NULL;
      offsets[nchunks] = done;
      counts[nchunks] = m;
      if (op == DLMH_OP_Q6K)
        tiers[nchunks] = dlmh::q6k_wide_rows(m);
      else if ((op == DLMH_OP_W8A8 && dlmh::w8a8_umma_supported(k)) ||
               (op == DLMH_OP_W8A16 && dlmh::w8a16_umma_supported(k)))
        tiers[nchunks] = (m + 15) / 16 * 16;  // tensor-core tier: MMA N = rows rounded up to 16
      else
        tiers[nchunks] = dlmh::tier_width(m);
    }
    ++nchunks;
    done += m;
  }
  if (cap > 0 && nchunks > cap) return DLMH_ERR_CAPACITY;
  return nchunks;
}

int lm_head_fp8_w8a16(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x, int64_t ldx, int rows,
                      dlmh_bf16* out, int64_t ldc, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 16));
  if (rows == 0) return DLMH_OK;
  if (!w || !w_scale) return DLMH_ERR_NULL;
  if (!aligned16(w)) return DLMH_ERR_ALIGN;
  DLMH_TRY(check_bf16_in(x, ldx, k));
  DLMH_TRY(check_out(out, ldc, n));
  if (dlmh::w8a16_umma_supported(k)) {
    dlmh::UmmaScratch sc;
    DLMH_TRY(dlmh::call_scratch(DLMH_OP_W8A16, n, k, rows, as_stream(stream), &sc));
    return dlmh::w8a16_umma_run(w, w_scale, n, k, x, ldx, rows, out, ldc, as_stream(stream), sc);
  }
  const int width = pass_rows(DLMH_OP_W8A16, k);
  if (width <= 0) return DLMH_ERR_UNSUPPORTED;
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    DLMH_TRY(dlmh::w8a16_pass(w, w_scale, n, k, x + (int64_t)done * ldx, ldx, m, out + (int64_t)done * ldc, ldc,
                              as_stream(stream)));
    done += m;
  }
  return DLMH_OK;
}

static int check_quant_out(const uint8_t* xq, int64_t ldq, const float* xs, int k) {
  if (!xq || !xs) return DLMH_ERR_NULL;
  if (ldq < k) return DLMH_ERR_LD;
  if (!aligned16(xq) || ldq % 16 != 0) return DLMH_ERR_ALIGN;
  return DLMH_OK;
}

int w8a8_quantize_rows(const dlmh_bf16* x, int64_t ldx, int rows, int k, uint8_t* xq, int64_t ldq, float* x_scale,
                       void* stream) {
  DLMH_TRY(check_rows(rows, DLMH_W8A8_MAX_ROWS));
  if (k <= 0 || k > kMaxK || k % 16) return DLMH_ERR_SHAPE;
  if (rows == 0) return DLMH_OK;
  DLMH_TRY(check_bf16_in(x, ldx, k));
  DLMH_TRY(check_quant_out(xq, ldq, x_scale, k));
  return dlmh::w8a8_quantize_launch(x, ldx, rows, k, xq, ldq, x_scale, as_stream(stream));
}

int w8a8_silu_quantize_rows(const dlmh_bf16* gate, const dlmh_bf16* up, int64_t ld, int rows, int k, uint8_t* xq,
                            int64_t ldq, float* x_scale, void* stream) {
  DLMH_TRY(check_rows(rows, DLMH_W8A8_MAX_ROWS));
  if (k <= 0 || k > kMaxK || k % 16) return DLMH_ERR_SHAPE;
  if (rows == 0) return DLMH_OK;
  DLMH_TRY(check_bf16_in(gate, ld, k));
  DLMH_TRY(check_bf16_in(up, ld, k));
  DLMH_TRY(check_quant_out(xq, ldq, x_scale, k));
  return dlmh::w8a8_silu_quantize_launch(gate, up, ld, rows, k, xq, ldq, x_scale, as_stream(stream));
}

// `fixed`: the tensor-core scratch chosen by the caller of this helper (null: the stream's
// workspace or the pool, resolved after the argument checks).
static int w8a8_gemv_impl(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
                          const float* x_scale, int rows, dlmh_bf16* out, int64_t ldc, void* stream,
                          const dlmh::UmmaScratch* fixed, bool after_prepass = false) {
  DLMH_TRY(check_rows(rows, DLMH_W8A8_MAX_ROWS));
  DLMH_TRY(check_nk(n, k, 16));
  if (rows == 0) return DLMH_OK;
  if (!w || !w_scale) return DLMH_ERR_NULL;
  if (!aligned16(w)) return DLMH_ERR_ALIGN;
  if (!xq || !x_scale) return DLMH_ERR_NULL;
  if (ldq < k) return DLMH_ERR_LD;
  if (!aligned16(xq) || ldq % 16 != 0) return DLMH_ERR_ALIGN;
  DLMH_TRY(check_out(out, ldc, n));
  const int width = pass_rows(DLMH_OP_W8A8, k);
  if (width <= 0) return DLMH_ERR_UNSUPPORTED;
  dlmh::UmmaScratch sc;
  if (fixed)
    sc = *fixed;
  else if (dlmh::w8a8_umma_supported(k))
    DLMH_TRY(dlmh::call_scratch(DLMH_OP_W8A8, n, k, rows, as_stream(stream), &sc));
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    if (dlmh::w8a8_umma_supported(k))
      DLMH_TRY(dlmh::w8a8_umma_pass(w, w_scale, n, k, xq + (int64_t)done * ldq, ldq, x_scale + done, m,
                                    out + (int64_t)done * ldc, ldc, as_stream(stream), sc,
                                    after_prepass && done == 0));
    else
      DLMH_TRY(dlmh::w8a8_gemv_pass(w, w_scale, n, k, xq + (int64_t)done * ldq, ldq, x_scale + done, m,
                                    out + (int64_t)done * ldc, ldc, as_stream(stream)));
    done += m;
  }
  return DLMH_OK;
}

int w8a8_gemv(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
              const float* x_scale, int rows, dlmh_bf16* out, int64_t ldc, void* stream) {
  return w8a8_gemv_impl(w, w_scale, n, k, xq, ldq, x_scale, rows, out, ldc, stream, nullptr);
}

static int w8a8_proj_impl(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x,
                          const dlmh_bf16* up, int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, uint8_t* xq,
                          float* xs, void* stream, const dlmh::UmmaScratch* fixed = nullptr) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 16));
  if (rows == 0) return DLMH_OK;
  if (!w || !w_scale) return DLMH_ERR_NULL;
  if (!aligned16(w)) return DLMH_ERR_ALIGN;
  DLMH_TRY(check_bf16_in(x, ldx, k));
  if (up) DLMH_TRY(check_bf16_in(up, ldx, k));
  DLMH_TRY(check_out(out, ldc, n));
  if (!xq || !xs) return DLMH_ERR_NULL;
  if (!aligned16(xq) || k % 16 != 0) return DLMH_ERR_ALIGN;
  if (pass_rows(DLMH_OP_W8A8, k) <= 0) return DLMH_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  dlmh::UmmaScratch sc;  // resolved before the first launch
  if (fixed)
    sc = *fixed;
  else if (dlmh::w8a8_umma_supported(k))
    DLMH_TRY(dlmh::call_scratch(DLMH_OP_W8A8, n, k, rows, s, &sc));
  for (int done = 0; done < rows;) {
    const int m = rows - done < DLMH_W8A8_MAX_ROWS ? rows - done : DLMH_W8A8_MAX_ROWS;
    const dlmh_bf16* xc = x + (int64_t)done * ldx;
    if (up)
      DLMH_TRY(dlmh::w8a8_silu_quantize_launch(xc, up + (int64_t)done * ldx, ldx, m, k, xq, k, xs, s));
    else
      DLMH_TRY(dlmh::w8a8_quantize_launch(xc, ldx, m, k, xq, k, xs, s));
    DLMH_TRY(w8a8_gemv_impl(w, w_scale, n, k, xq, k, xs, m, out + (int64_t)done * ldc, ldc, stream, &sc, true));
    done += m;
  }
  return DLMH_OK;
}

int w8a8_proj(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x, int64_t ldx, int rows,
              dlmh_bf16* out, int64_t ldc, uint8_t* xq_scratch, float* xscale_scratch, void* stream) {
  return w8a8_proj_impl(w, w_scale, n, k, x, nullptr, ldx, rows, out, ldc, xq_scratch, xscale_scratch, stream);
}

int w8a8_silu_proj(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* gate, const dlmh_bf16* up,
                   int64_t ld, int rows, dlmh_bf16* out, int64_t ldc, uint8_t* xq_scratch, float* xscale_scratch,
                   void* stream) {
  if (!up && rows != 0) return DLMH_ERR_NULL;
  if (!up) return w8a8_proj_impl(w, w_scale, n, k, gate, nullptr, ld, rows, out, ldc, xq_scratch, xscale_scratch,
                                 stream);
  return w8a8_proj_impl(w, w_scale, n, k, gate, up, ld, rows, out, ldc, xq_scratch, xscale_scratch, stream);
}

int w8a8_gate_up_proj(const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up, const float* s_up, int n,
                      int k, const dlmh_bf16* x, int64_t ldx, int rows, dlmh_bf16* gate_out, dlmh_bf16* up_out,
                      int64_t ldc, uint8_t* xq_scratch, float* xscale_scratch, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 16));
  if (rows == 0) return DLMH_OK;
  if (!w_gate || !s_gate || !w_up || !s_up) return DLMH_ERR_NULL;
  if (!aligned16(w_gate) || !aligned16(w_up)) return DLMH_ERR_ALIGN;
  DLMH_TRY(check_bf16_in(x, ldx, k));
  DLMH_TRY(check_out(gate_out, ldc, n));
  DLMH_TRY(check_out(up_out, ldc, n));
  if (!xq_scratch || !xscale_scratch) return DLMH_ERR_NULL;
  if (!aligned16(xq_scratch) || k % 16 != 0) return DLMH_ERR_ALIGN;
  if (pass_rows(DLMH_OP_W8A8, k) <= 0) return DLMH_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  dlmh::UmmaScratch sc;  // resolved before the first launch
  if (dlmh::w8a8_umma_supported(k)) DLMH_TRY(dlmh::call_scratch(DLMH_OP_W8A8_PAIR, n, k, rows, s, &sc));
  for (int done = 0; done < rows;) {
    const int m = rows - done < DLMH_W8A8_MAX_ROWS ? rows - done : DLMH_W8A8_MAX_ROWS;
    DLMH_TRY(dlmh::w8a8_quantize_launch(x + (int64_t)done * ldx, ldx, m, k, xq_scratch, k, xscale_scratch, s));
    dlmh_bf16* g = gate_out + (int64_t)done * ldc;
    dlmh_bf16* u = up_out + (int64_t)done * ldc;
    if (dlmh::w8a8_umma_supported(k)) {
      DLMH_TRY(dlmh::w8a8_umma_pair_pass(w_gate, s_gate, n, g, ldc, w_up, s_up, n, u, ldc, k, xq_scratch, k,
                                         xscale_scratch, m, s, sc, true));
    } else {
      DLMH_TRY(w8a8_gemv_impl(w_gate, s_gate, n, k, xq_scratch, k, xscale_scratch, m, g, ldc, stream, &sc));
      DLMH_TRY(w8a8_gemv_impl(w_up, s_up, n, k, xq_scratch, k, xscale_scratch, m, u, ldc, stream, &sc));
    }
    done += m;
  }
  return DLMH_OK;
}

int w4a16_gemv(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int n, int k,
               const dlmh_bf16* x, int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 128));
  if (rows == 0) return DLMH_OK;
  if (!w_packed || !w_block_scale) return DLMH_ERR_NULL;
  if (!aligned16(w_packed) || !aligned16(w_block_scale)) return DLMH_ERR_ALIGN;
  DLMH_TRY(check_bf16_in(x, ldx, k));
  DLMH_TRY(check_out(out, ldc, n));
  const int width = pass_rows(DLMH_OP_W4A16, k);
  if (width <= 0) return DLMH_ERR_UNSUPPORTED;
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    DLMH_TRY(dlmh::w4a16_pass(w_packed, w_block_scale, global_scale, n, k, x + (int64_t)done * ldx, ldx, m,
                              out + (int64_t)done * ldc, ldc, as_stream(stream)));
    done += m;
  }
  return DLMH_OK;
}

int nvfp4_quantize_rows(const dlmh_bf16* x, int64_t ldx, int rows, int k, uint8_t* xq, uint8_t* x_block_scale,
                        float* x_global, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  if (k <= 0 || k > kMaxK || k % 16) return DLMH_ERR_SHAPE;
  if (rows == 0) return DLMH_OK;
  DLMH_TRY(check_bf16_in(x, ldx, k));
  if (!xq || !x_block_scale || !x_global) return DLMH_ERR_NULL;
  if (!aligned16(xq) || (reinterpret_cast<uintptr_t>(x_global) & 3u)) return DLMH_ERR_ALIGN;
  return dlmh::nvfp4_quantize_launch(x, ldx, rows, k, xq, x_block_scale, x_global, as_stream(stream));
}

// NVFP4 weight and output checks shared by the W4A4 entry points (after the shape checks).
static int check_w4a4_weight_out(const uint8_t* w_packed, const uint8_t* w_block_scale, int n, dlmh_bf16* out,
                                 int64_t ldc) {
  if (!w_packed || !w_block_scale) return DLMH_ERR_NULL;
  if (!aligned16(w_packed) || !aligned16(w_block_scale)) return DLMH_ERR_ALIGN;
  return check_out(out, ldc, n);
}

int w4a4_gemv(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int n, int k,
              const uint8_t* xq, const uint8_t* x_block_scale, const float* x_global, int rows, dlmh_bf16* out,
              int64_t ldc, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 256));
  if (rows == 0) return DLMH_OK;
  DLMH_TRY(check_w4a4_weight_out(w_packed, w_block_scale, n, out, ldc));
  if (!xq || !x_block_scale || !x_global) return DLMH_ERR_NULL;
  if (!aligned16(xq) || (reinterpret_cast<uintptr_t>(x_block_scale) & 1u) ||
      (reinterpret_cast<uintptr_t>(x_global) & 3u))
    return DLMH_ERR_ALIGN;
  const int width = pass_rows(DLMH_OP_W4A4, k);
  if (width <= 0) return DLMH_ERR_UNSUPPORTED;
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    DLMH_TRY(dlmh::w4a4_pass(w_packed, w_block_scale, global_scale, n, k, xq + (int64_t)done * (k / 2),
                             x_block_scale + (int64_t)done * (k / 16), x_global + done, m, out + (int64_t)done * ldc,
                             ldc, as_stream(stream)));
    done += m;
  }
  return DLMH_OK;
}

int w4a4_proj(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int n, int k,
              const dlmh_bf16* x, int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, uint8_t* xq_scratch,
              uint8_t* xs_scratch, float* xg_scratch, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 256));
  if (rows == 0) return DLMH_OK;
  DLMH_TRY(check_w4a4_weight_out(w_packed, w_block_scale, n, out, ldc));
  DLMH_TRY(check_bf16_in(x, ldx, k));
  if (!xq_scratch || !xs_scratch || !xg_scratch) return DLMH_ERR_NULL;
  if (!aligned16(xq_scratch) || (reinterpret_cast<uintptr_t>(xs_scratch) & 1u) ||
      (reinterpret_cast<uintptr_t>(xg_scratch) & 3u))
    return DLMH_ERR_ALIGN;
  const int width = pass_rows(DLMH_OP_W4A4, k);
  if (width <= 0) return DLMH_ERR_UNSUPPORTED;
  cudaStream_t s = as_stream(stream);
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    DLMH_TRY(dlmh::nvfp4_quantize_launch(x + (int64_t)done * ldx, ldx, m, k, xq_scratch, xs_scratch, xg_scratch, s));
    DLMH_TRY(dlmh::w4a4_pass(w_packed, w_block_scale, global_scale, n, k, xq_scratch, xs_scratch, xg_scratch, m,
                             out + (int64_t)done * ldc, ldc, s, true));
    done += m;
  }
  return DLMH_OK;
}

int q8_1_quantize_rows(const dlmh_bf16* x, int64_t ldx, int rows, int k, void* q8_out, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  if (k <= 0 || k > kMaxK || k % 32) return DLMH_ERR_SHAPE;
  if (rows == 0) return DLMH_OK;
  if (!x || !q8_out) return DLMH_ERR_NULL;
  if (ldx < k) return DLMH_ERR_LD;
  if ((reinterpret_cast<uintptr_t>(x) & 1u) || (reinterpret_cast<uintptr_t>(q8_out) & 3u)) return DLMH_ERR_ALIGN;
  return dlmh::q8_1_quantize_launch(x, ldx, rows, k, static_cast<uint8_t*>(q8_out), as_stream(stream));
}

int q6k_mmvq(const void* blocks, int n, int k, const void* q8, int rows, dlmh_bf16* out, int64_t ldc, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 256));
  if (rows == 0) return DLMH_OK;
  if (!blocks || !q8) return DLMH_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(blocks) & 1u) || (reinterpret_cast<uintptr_t>(q8) & 3u)) return DLMH_ERR_ALIGN;
  DLMH_TRY(check_out(out, ldc, n));
  const int64_t q8_row = (int64_t)(k / 32) * DLMH_Q8_1_BLOCK_BYTES;
  const int width = aligned16(q8) && aligned16(blocks) ? DLMH_Q6K_MAX_ROWS : DLMH_Q6K_CHUNK_ROWS;
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    DLMH_TRY(dlmh::q6k_mmvq_launch(static_cast<const uint8_t*>(blocks), n, k,
                                   static_cast<const uint8_t*>(q8) + done * q8_row, m, out + (int64_t)done * ldc, ldc,
                                   as_stream(stream)));
    done += m;
  }
  return DLMH_OK;
}

int q6k_lm_head(const void* blocks, int n, int k, const dlmh_bf16* x, int64_t ldx, int rows, dlmh_bf16* out,
                int64_t ldc, void* q8_scratch, void* stream) {
  DLMH_TRY(check_rows(rows, 0));
  DLMH_TRY(check_nk(n, k, 256));
  if (rows == 0) return DLMH_OK;
  if (!blocks || !x || !q8_scratch) return DLMH_ERR_NULL;
  if (ldx < k) return DLMH_ERR_LD;
  if ((reinterpret_cast<uintptr_t>(blocks) & 1u) || (reinterpret_cast<uintptr_t>(q8_scratch) & 3u) ||
      (reinterpret_cast<uintptr_t>(x) & 1u))
    return DLMH_ERR_ALIGN;
  DLMH_TRY(check_out(out, ldc, n));
  cudaStream_t s = as_stream(stream);
  const int width = aligned16(q8_scratch) && aligned16(blocks) ? DLMH_Q6K_MAX_ROWS : DLMH_Q6K_CHUNK_ROWS;
  for (int done = 0; done < rows;) {
    const int m = rows - done < width ? rows - done : width;
    DLMH_TRY(dlmh::q8_1_quantize_launch(x + (int64_t)done * ldx, ldx, m, k, static_cast<uint8_t*>(q8_scratch), s));
    DLMH_TRY(dlmh::q6k_mmvq_launch(static_cast<const uint8_t*>(blocks), n, k,
                                   static_cast<const uint8_t*>(q8_scratch), m, out + (int64_t)done * ldc, ldc, s, true));
    done += m;
  }
  return DLMH_OK;
}

}  // extern "C"

extern "C" {

int nvfp4_dequant_bf16(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int is_reciprocal,
                       int n, int k, dlmh_bf16* out, int64_t ldo, void* stream) {
  DLMH_TRY(check_nk(n, k, 16));
  if (!w_packed || !w_block_scale) return DLMH_ERR_NULL;
  if (!aligned16(w_packed) || !aligned16(w_block_scale)) return DLMH_ERR_ALIGN;
  if (!out) return DLMH_ERR_NULL;
  if (ldo < k) return DLMH_ERR_LD;
  if (!aligned16(out) || ldo % 8 != 0) return DLMH_ERR_ALIGN;
  // fold the stored global into one float32 multiplier, as the loader does
  const float g = is_reciprocal ? (global_scale != 0.f ? 1.0f / global_scale : 0.f) : global_scale;
  return dlmh::nvfp4_dequant_launch(w_packed, w_block_scale, g, n, k, out, ldo, as_stream(stream));
}

int e8m0_fp4_dequant_bf16(const uint8_t* w_packed, const uint8_t* scales, int64_t num_scales, int n, int k,
                          dlmh_bf16* out, int64_t ldo, void* stream) {
  DLMH_TRY(check_nk(n, k, 16));
  if (!w_packed || !scales) return DLMH_ERR_NULL;
  const int64_t total = (int64_t)n * k;
  if (num_scales <= 0 || total % num_scales != 0) return DLMH_ERR_SHAPE;
  if (!aligned16(w_packed)) return DLMH_ERR_ALIGN;
  if (!out) return DLMH_ERR_NULL;
  if (ldo < k) return DLMH_ERR_LD;
  if (!aligned16(out) || ldo % 8 != 0) return DLMH_ERR_ALIGN;
  return dlmh::e8m0_dequant_launch(w_packed, scales, total / num_scales, n, k, out, ldo, as_stream(stream));
}

}  // extern "C"

namespace dlmh {

int w8a8_proj_fixed_scratch(const uint8_t* w, const float* w_scale, int n, int k, const uint16_t* x, int64_t ldx,
                            int rows, uint16_t* out, int64_t ldc, uint8_t* xq, float* xs, const UmmaScratch& scratch,
                            cudaStream_t stream) {
  return w8a8_proj_impl(w, w_scale, n, k, x, nullptr, ldx, rows, out, ldc, xq, xs, stream, &scratch);
}

}  // namespace dlmh
