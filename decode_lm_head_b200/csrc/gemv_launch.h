// Internal launch entry points of libdlmh (host side).  Every function launches
// asynchronously on `s` and returns a dlmh_status.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dlmh {

// Internal scratch of one tensor-core call.  caller == false: the library's stream-ordered
// pool serves the W8A16 codes and the stream-K partial sums, and whole tiles go in the static
// order.  caller == true: the pointers below serve the call and nothing is allocated
// (DLMH_ERR_WORKSPACE when a needed area is missing or too small); `queue` (two ints, zero
// between launches) hands out the whole tiles, or null keeps the static order.
struct UmmaScratch {
  bool caller = false;
  int* queue = nullptr;
  uint8_t* codes = nullptr;  // W8A16: two-term codes, then 128 float32 row multipliers
  size_t codes_cap = 0;
  float* partial = nullptr;
  size_t partial_cap = 0;
};

// Widest row count one weight pass of `op` (a dlmh_op) serves at reduction length k, or 0
// when even the 8-row tier does not fit on chip.  Pure function of (op, k).
int max_tier_rows(int op, int k);
// Fault bits recorded by bounded device waits since the last reset (0 in a healthy run);
// reads synchronously.
// NVFP4 W4A4 pass (streamed kernel, k % 256 == 0): NVFP4 weights against NVFP4 activation rows
// xq [rows][k/2], xbs [rows][k/16], xg [rows] as written by nvfp4_quantize_launch.
// after_prepass: the preceding kernel on `s` is nvfp4_quantize_launch (weight loads may overlap it).
int w4a4_pass(const uint8_t* wp, const uint8_t* wbs, float g, int n, int k, const uint8_t* xq,
              const uint8_t* xbs, const float* xg, int rows, uint16_t* out, int64_t ldc, cudaStream_t s,
              bool after_prepass = false);
// Per-row NVFP4 quantize of BF16 rows (one 8-CTA cluster per row): codes [rows][k/2] (row
// stride k/2), block scales [rows][k/16], globals [rows].  k % 16 == 0.
int nvfp4_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* xq, uint8_t* xbs, float* xg,
                          cudaStream_t s);
int device_fault(int reset);
// Width (8, 16 or 32) of the narrowest compiled tier that covers `rows` (1..32).
inline int tier_width(int rows) { return rows <= 8 ? 8 : (rows <= 16 ? 16 : 32); }

int w8a16_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint16_t* x, int64_t ldx, int rows,
               uint16_t* out, int64_t ldc, cudaStream_t s);
int w8a8_gemv_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
                   const float* x_scale, int rows, uint16_t* out, int64_t ldc, cudaStream_t s);
// Tensor-core W8A8 pass (tcgen05, TMA-fed): one weight pass for 1..128 rows.  Taken for every
// row count whenever w8a8_umma_supported(k) holds (a pure function of k).
bool w8a8_umma_supported(int k);
// The stream-K remainder's partial sums and the tile order come from `scratch` (above).
// after_prepass: the preceding kernel on `s` is this library's activation quantize (weight
// loads may then overlap its tail).
int w8a8_umma_pass(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
                   const float* x_scale, int rows, uint16_t* out, int64_t ldc, cudaStream_t s,
                   const UmmaScratch& scratch, bool after_prepass = false);
// Two weight matrices (same k) against the same activation codes in ONE tensor-core launch
// (an FFN's gate and up): the tiles of both share one stream-K schedule over the SMs, a pure
// function of (n1, n2, k, #SMs).
int w8a8_umma_pair_pass(const uint8_t* w1, const float* s1, int n1, uint16_t* out1, int64_t ldc1,
                        const uint8_t* w2, const float* s2, int n2, uint16_t* out2, int64_t ldc2, int k,
                        const uint8_t* xq, int64_t ldq, const float* x_scale, int rows, cudaStream_t s,
                        const UmmaScratch& scratch, bool after_prepass);
// w8a8_proj with caller-fixed scratch for everything, including the partial sums: never
// allocates (the allocation-free entry point).
int w8a8_proj_fixed_scratch(const uint8_t* w, const float* w_scale, int n, int k, const uint16_t* x, int64_t ldx,
                            int rows, uint16_t* out, int64_t ldc, uint8_t* xq, float* xs, const UmmaScratch& scratch,
                            cudaStream_t stream);
// Used and peak bytes of the library pool of the current device (0 before its first use);
// reset_high != 0 sets the peak back to the current use.
int pool_stats(int64_t* used_current, int64_t* used_high, int reset_high);
// The scratch of a call of `op` (a dlmh_op) with this shape on stream `s`: the stream's bound
// caller workspace (DLMH_ERR_WORKSPACE when it is smaller than the call needs) or the pool.
int call_scratch(int op, int n, int k, int rows, cudaStream_t s, UmmaScratch* out);
// Fault bits of the tensor-core kernel's bounded waits (read synchronously).
int umma_fault(int reset);
// Runs one bounded mbarrier wait that can never complete; DLMH_OK if it gave up and recorded
// its fault bit (then cleared again), synchronizes `s`.
int bounded_wait_check(cudaStream_t s);

// Tensor-core W8A16 (the same kernel; activations split into two exact E4M3 terms): one
// weight pass per 128 rows, taken for every row count whenever w8a16_umma_supported(k)
// holds.  Runs its own row loop; the activation codes live in `scratch` (the caller's
// workspace, or the library's stream-ordered pool).
bool w8a16_umma_supported(int k);
int w8a16_umma_run(const uint8_t* w, const float* w_scale, int n, int k, const uint16_t* x, int64_t ldx, int rows,
                   uint16_t* out, int64_t ldc, cudaStream_t s, const UmmaScratch& scratch);

int w4a16_pass(const uint8_t* wp, const uint8_t* wbs, float g, int n, int k, const uint16_t* x, int64_t ldx, int rows,
               uint16_t* out, int64_t ldc, cudaStream_t s);

int w8a8_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* xq, int64_t ldq, float* sx,
                         cudaStream_t s);
int w8a8_silu_quantize_launch(const uint16_t* gate, const uint16_t* up, int64_t ld, int rows, int k, uint8_t* xq,
                              int64_t ldq, float* sx, cudaStream_t s);
// W8A16 two-term split (act_quant.cu): rows [0, half) of `codes` get hi(x'), rows
// [half, 2 half) lo(x'), padding rows zeros; x_mul[m] = 2^-e[m].
int w8a16_split_launch(const uint16_t* x, int64_t ldx, int rows, int k, int half, uint8_t* codes, float* x_mul,
                       cudaStream_t s);
int q8_1_quantize_launch(const uint16_t* x, int64_t ldx, int rows, int k, uint8_t* q8, cudaStream_t s);
// Load-time FP4 dequant to BF16 (dequant.cu); k % 16 == 0, out 16-byte aligned, ldo % 8 == 0.
int nvfp4_dequant_launch(const uint8_t* packed, const uint8_t* bscale, float g, int n, int k, uint16_t* out,
                         int64_t ldo, cudaStream_t s);
int e8m0_dequant_launch(const uint8_t* packed, const uint8_t* scales, int64_t block, int n, int k, uint16_t* out,
                        int64_t ldo, cudaStream_t s);

// Fault bits of the streamed Q6_K kernel's bounded waits (read synchronously).
int q6k_fault(int reset);
// Q6_K GEMV of 1..64 q8_1 rows in one weight pass: the 8-row kernels up to 8 rows, the wide
// kernel (tiers 16 / 32 / 64, q8 16-byte aligned, else DLMH_ERR_ALIGN) above; same bits.
int q6k_wide_rows(int rows);
// after_prepass: the preceding kernel on `s` is q8_1_quantize_launch (weight copies may start
// before it completes).
int q6k_mmvq_launch(const uint8_t* blocks, int n, int k, const uint8_t* q8, int rows, uint16_t* out, int64_t ldc,
                    cudaStream_t s, bool after_prepass = false);

}  // namespace dlmh
