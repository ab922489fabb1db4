/*
 * dlmh.h -- C ABI of the B200 (sm_100a) decode LM-head / projection GEMV library.
 *
 * One library, libdlmh.so, turns M = 1..128 BF16 decode rows into BF16 logits or
 * projection outputs against a quantized weight, reading the weight as few times as
 * possible (one pass per row chunk).  Formats:
 *   - FP8 E4M3 weights with one float32 scale per output row, run W8A16
 *     ("metrale_model_engine/model/lm_head_fp8_rows.rs", module doc and lm_head_fp8_run);
 *   - the same weights run W8A8 after a per-row dynamic E4M3 activation quantize, also
 *     from bf16(silu(gate) * up) for an FFN down projection
 *     ("metrale_model_layers/layers/w8a8_layer.rs", W8a8Ctx::proj and W8a8Ctx::silu_proj);
 *   - NVFP4 W4A16: E2M1 codes two per byte, one E4M3 scale per 16 K-elements, one folded
 *     float32 global ("metrale_model_layers/layers/w4a16_gemv_tiers.rs";
 *     "metrale_model_layers/weight_map/fp8_lut.rs", dequant_nvfp4_to_bf16);
 *   - Q6_K 210-byte super-blocks against block_q8_1-quantized rows
 *     ("metrale_model_engine/model/lm_head_q6k.rs", lm_head_q6k_run).
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *   - Every pointer argument named w*, x*, gate, up, out*, xq*, *scale*, q8*, blocks or
 *     *scratch is a DEVICE pointer on the current CUDA device.  The caller owns all of
 *     them; the library keeps no pointer after return.
 *   - Internal scratch of the tensor-core passes (k % 128 == 0) of lm_head_fp8_w8a16 and of
 *     the W8A8 GEMVs (W8A16 activation codes, stream-K partial sums, a whole-tile queue):
 *       * with a caller workspace bound to the stream (dlmh_set_workspace, sized with
 *         dlmh_workspace_bytes) it comes from that workspace and NO call allocates anything;
 *         the CTAs then take the whole weight tiles from the workspace's atomic queue;
 *       * without one, the codes and partial sums come from a library-owned memory pool of
 *         the current device (cudaMallocFromPoolAsync / cudaFreeAsync on `stream`; the pool
 *         keeps its memory, so steady-state calls map nothing and never synchronize) and the
 *         whole tiles go in a static order.
 *     Both tile orders give the same outputs.  A launch being captured into a CUDA graph
 *     takes the static order (a graph holds no counter).  w8a8_proj_noalloc uses neither the
 *     pool nor a workspace.
 *   - BF16 values are passed as raw 16-bit patterns (dlmh_bf16).
 *   - Matrices are row-major.  Leading dimensions (ld*) count ELEMENTS of the pointed-to
 *     type, so row r of x starts at x + r * ldx.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Every launch is asynchronous on that stream; no call synchronizes.
 *   - rows == 0 is valid: after the shape checks (n, k) the call returns DLMH_OK without
 *     looking at any pointer and launches nothing.
 *   - Return value: DLMH_OK (0) or a negative dlmh_status.  On any argument error the
 *     call returns before launching anything, so outputs are left untouched.
 *     DLMH_ERR_CUDA reports a failed launch (cudaGetLastError after the launch).
 *   - Output rows are independent of how many rows share a call: the same input row
 *     gives the same output bits at any `rows` (row invariance, w8a8_layer.rs module
 *     doc; lm_head_fp8_rows.rs, the W8A8 branch of lm_head_fp8_run).
 *   - Alignment: weight, scale-block and x pointers must be 16-byte aligned, and ldx
 *     (and ld of gate/up) must be a multiple of 8 elements, else DLMH_ERR_ALIGN.
 *
 * Thread safety: entry points are reentrant.  Calls that share a scratch buffer must be
 * ordered on one stream (w8a8_layer.rs module doc: quantize -> GEMV pairs of one
 * scratch never interleave).
 */
#ifndef DLMH_H_
#define DLMH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols (the library is built with hidden visibility by default). */
#if defined(__GNUC__)
#define DLMH_API __attribute__((visibility("default")))
#else
#define DLMH_API
#endif

typedef uint16_t dlmh_bf16; /* raw BF16 bit pattern */

typedef enum dlmh_status {
  DLMH_OK = 0,
  DLMH_ERR_NULL = -1,        /* a required pointer is NULL */
  DLMH_ERR_SHAPE = -2,       /* n <= 0, k <= 0, k not a multiple of the format's block */
  DLMH_ERR_ALIGN = -3,       /* a pointer or leading dimension breaks 16-byte alignment */
  DLMH_ERR_ROWS = -4,        /* rows < 0, or rows above the entry point's cap */
  DLMH_ERR_LD = -5,          /* a leading dimension is smaller than the row it holds */
  DLMH_ERR_CUDA = -6,        /* a CUDA runtime call or launch failed */
  DLMH_ERR_UNSUPPORTED = -7, /* the shape is valid but beyond this build's limits (k too large) */
  DLMH_ERR_CAPACITY = -8,    /* an output array passed to a host helper (or a table) is too small */
  DLMH_ERR_WORKSPACE = -9    /* the stream's bound workspace is smaller than the call needs */
} dlmh_status;

/* Largest row count of one W8A8 quantize / GEMV call (ops::W8A8_MAX_ROWS in
 * lm_head_fp8_rows.rs and w8a8_layer.rs: one weight pass per 128 rows). */
#define DLMH_W8A8_MAX_ROWS 128
/* Rows per weight pass of the FP8 W8A16 head (16-row chunks above 16 rows,
 * lm_head_fp8_rows.rs module doc). */
#define DLMH_W8A16_CHUNK_ROWS 16
/* Widest NVFP4 W4A16 weight pass (w4a16_gemv_tiers.rs, kernel_within: one kernel launch
 * serves at most 32 rows).  w4a16_gemv runs more rows as several such passes. */
#define DLMH_W4A16_MAX_ROWS 32
/* Widest W4A4 pass (w4a4_proj::W4A4_MAX_M in w4a16_gemv_tiers.rs). */
#define DLMH_W4A4_MAX_ROWS 32
/* Rows of the pages' Q6_K launch (MAX_M / KQ_MAX_M in lm_head_q6k.rs): the narrowest tier. */
#define DLMH_Q6K_CHUNK_ROWS 8
/* Rows per Q6_K weight pass here (tiers 8 / 16 / 32 / 64; the pages run 8-row launches). */
#define DLMH_Q6K_MAX_ROWS 64
/* Bytes of one block_q8_1 (32 values) and one Q6_K super-block (256 values). */
#define DLMH_Q8_1_BLOCK_BYTES 36
#define DLMH_Q6K_BLOCK_BYTES 210

/* ---------------------------------------------------------------------------------------
 * FP8 E4M3 W8A16 GEMV (the FP8 LM head)
 *   out[m, n] = bf16( s[n] * sum_k e4m3(w[n, k]) * x[m, k] )   for m < rows, n < n
 * lm_head_fp8_rows.rs, module doc and lm_head_fp8_run (the W8A16 branch).
 *   w       [n, k] E4M3 bytes, row stride k bytes, 16-byte aligned.
 *   w_scale [n] float32, one per output row.
 *   x       [rows, ldx] BF16, ldx >= k, ldx % 8 == 0, 16-byte aligned.
 *   out     [rows, ldc] BF16, ldc >= n.
 *   k % 16 == 0.  Any rows >= 0.
 *   k % 128 == 0 (the tensor-core path, every FP8 head): one weight pass per 128 rows (the
 *   last pass ragged).  Each x row is scaled by a power of two 2^e with max|x| 2^e in
 *   [2^7, 2^8) and split into two E4M3 terms hi = e4m3(x'), lo = e4m3(16 (x' - hi)); then
 *   out = bf16(s[n] 2^-e (sum_k w hi + (sum_k w lo) / 16)) with f32 sums.  hi + lo/16 equals
 *   x' exactly for every element with |x| >= 2^-13 max|x| of its row (every BF16 value has
 *   8 significant bits, E4M3 4); smaller elements keep an error below 2^-21 max|x|.
 *   Scratch: 2 * roundup8(min(rows, 128)) * k bytes + 512 B, plus the stream-K partial
 *   sums (at most 2 * #SMs * 128 * 256 * 4 bytes), from the stream's workspace or the
 *   library pool (see above; dlmh_workspace_bytes(DLMH_OP_W8A16, ...)).
 *   Other k: one weight pass per 16 rows; E4M3 weights decoded exactly to f16 and each x row
 *   scaled by a power of two into f16 (exact for every |x| >= 2^-31 max|x|), products
 *   summed in f32.  k above the shared-memory limit of a 16-row chunk (k > 6144) returns
 *   DLMH_ERR_UNSUPPORTED.
 *   Either way the row scale and the power of two are applied to the f32 sum, then rounded
 *   to BF16 (round-to-nearest-even).
 * ------------------------------------------------------------------------------------- */
DLMH_API int lm_head_fp8_w8a16(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x,
                      int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, void* stream);

/* ---------------------------------------------------------------------------------------
 * W8A8 per-row dynamic E4M3 activation quantize
 *   per row m:  amax = max_k |x[m, k]|,  sx[m] = amax / 448  (float32 IEEE division),
 *               xq[m, k] = e4m3_rn_sat( x[m, k] / sx[m] )    (float32 IEEE division,
 *               round-to-nearest-even, magnitudes above 448 saturate to 448);
 *               a row with sx == 0 gets all-zero codes.
 * w8a8_layer.rs, W8a8Ctx::proj (the quantized rows live in the shared W8A8 scratch).
 *   x       [rows, ldx] BF16;  xq [rows, ldq] E4M3 bytes (ldq >= k, ldq % 16 == 0,
 *   16-byte aligned);  x_scale [rows] float32.  k % 16 == 0.  rows <= 128.
 * ------------------------------------------------------------------------------------- */
DLMH_API int w8a8_quantize_rows(const dlmh_bf16* x, int64_t ldx, int rows, int k, uint8_t* xq, int64_t ldq,
                       float* x_scale, void* stream);

/* Fused SiLU quantize: h[m, k] = bf16( silu(gate[m, k]) * up[m, k] ), silu(g) = g / (1 + e^-g),
 * in correctly rounded f32 steps (e = rn32(e^-g), d = rn32(1 + e), s = rn32(g / d),
 * p = rn32(s * up)) and one round-to-nearest-even to BF16, then quantized per row exactly as
 * w8a8_quantize_rows; h is never written to memory.  w8a8_layer.rs, W8a8Ctx::silu_proj
 * (ops::w8a8_act_quant_silu).  gate and up [rows, ld] BF16; rows <= 128. */
DLMH_API int w8a8_silu_quantize_rows(const dlmh_bf16* gate, const dlmh_bf16* up, int64_t ld, int rows, int k,
                            uint8_t* xq, int64_t ldq, float* x_scale, void* stream);

/* ---------------------------------------------------------------------------------------
 * W8A8 GEMV on already-quantized rows
 *   out[m, n] = bf16( s[n] * sx[m] * sum_k e4m3(w[n, k]) * e4m3(xq[m, k]) )
 * lm_head_fp8_rows.rs (W8A8 branch), w8a8_layer.rs (ops::w8a8_gemv).
 *   rows <= 128; one weight pass per call when k % 128 == 0 (tensor cores; stream-K partial
 *   sums in the stream's workspace or pool scratch, see above), else passes of up to 32 rows (k bounded by the
 *   shared-memory activation tile, DLMH_ERR_UNSUPPORTED beyond).  xq [rows, ldq] as written
 *   by the quantize entry points; x_scale [rows].  k % 16 == 0.
 * ------------------------------------------------------------------------------------- */
DLMH_API int w8a8_gemv(const uint8_t* w, const float* w_scale, int n, int k, const uint8_t* xq, int64_t ldq,
              const float* x_scale, int rows, dlmh_bf16* out, int64_t ldc, void* stream);

/* W8A8 projection of BF16 rows: quantize into the caller's scratch, then GEMV, on one
 * stream, in 128-row chunks (lm_head_fp8_rows.rs, W8A8 branch of lm_head_fp8_run).
 *   xq_scratch      device buffer of at least 128 * k bytes, 16-byte aligned (row stride k).
 *   xscale_scratch  device buffer of at least 128 float32.
 * After the call the scratch holds the last chunk's codes and scales. */
DLMH_API int w8a8_proj(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x, int64_t ldx,
              int rows, dlmh_bf16* out, int64_t ldc, uint8_t* xq_scratch, float* xscale_scratch,
              void* stream);

/* The down projection of a SiLU FFN: w8a8_silu_quantize_rows then w8a8_gemv per 128-row
 * chunk (w8a8_layer.rs, W8a8Ctx::silu_proj).  Scratch as for w8a8_proj. */
DLMH_API int w8a8_silu_proj(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* gate,
                   const dlmh_bf16* up, int64_t ld, int rows, dlmh_bf16* out, int64_t ldc,
                   uint8_t* xq_scratch, float* xscale_scratch, void* stream);

/* Gate and up projections of a SiLU FFN on ONE quantized copy of x (w8a8_layer.rs, W8a8Ffn:
 * gate and up read the same input).  Per 128-row chunk: w8a8_quantize_rows once, then
 *   gate_out[m, n] = bf16( s_gate[n] * sx[m] * sum_k e4m3(w_gate[n, k]) * xq[m, k] )
 *   up_out[m, n]   = bf16( s_up[n]   * sx[m] * sum_k e4m3(w_up[n, k])   * xq[m, k] )
 * in one launch over the tiles of both weights when k % 128 == 0 (two register-kernel GEMVs
 * on the same codes otherwise).  Same numerics as w8a8_proj of each weight; a row's bits do
 * not depend on `rows`, and they may differ in the last place from a lone w8a8_proj of the
 * same weight (the two weights share one split-K schedule).
 *   w_gate, w_up   [n, k] E4M3 bytes (16-byte aligned), s_gate, s_up [n] float32.
 *   x              [rows, ldx] BF16, any rows >= 0 (chunks of 128).
 *   gate_out, up_out  [rows, ldc] BF16 (ldc >= n); they feed w8a8_silu_proj with ld = ldc.
 *   xq_scratch, xscale_scratch  as for w8a8_proj.
 * Errors as w8a8_proj (DLMH_ERR_NULL for a NULL weight, scale or output of either). */
DLMH_API int w8a8_gate_up_proj(const uint8_t* w_gate, const float* s_gate, const uint8_t* w_up,
                               const float* s_up, int n, int k, const dlmh_bf16* x, int64_t ldx, int rows,
                               dlmh_bf16* gate_out, dlmh_bf16* up_out, int64_t ldc, uint8_t* xq_scratch,
                               float* xscale_scratch, void* stream);

/* ---------------------------------------------------------------------------------------
 * W8A8 projection that allocates nothing, not even caller scratch
 *   Same operation, rows and results as w8a8_proj.  The quantized-activation scratch is a
 *   fixed device array inside this library instead of a caller buffer.  The pages have no
 *   counterpart: this entry point is this library's own addition.
 *
 *   Who it is for: callers that cannot call cudaMalloc.  Examples are engines whose device
 *   memory belongs to a pre-reserved pool or to another framework's allocator, and decode
 *   loops that cannot afford cudaMalloc's implicit device synchronization.  They still pass
 *   w, w_scale, x and out.
 *
 *   Limits: k <= DLMH_NOALLOC_MAX_K (16384), else DLMH_ERR_UNSUPPORTED; a device with more
 *   than DLMH_NOALLOC_MAX_SMS (160) SMs gets DLMH_ERR_UNSUPPORTED for shapes whose
 *   tensor-core pass needs stream-K partial sums.  Both are checked before any launch.  Every GPU that loads the library holds
 *   the array until the process exits: 2 MiB of codes, 512 B of scales and 20 MiB of
 *   partial sums (22 MiB + 512 B).
 *
 *   Set-up: a device's first call looks the array's device address up
 *   (cudaGetSymbolAddress, with that device current) and keeps it for the life of the
 *   process.  Make that first call before any stream capture.  The kept address does not
 *   survive cudaDeviceReset (the module, and the array with it, is loaded again): do not
 *   call this entry point after resetting a device it was used on.
 *
 *   Sharing: all calls on a device share the one array, and it keeps the last call's codes
 *   and scales.  Each call overwrites, before reading, every byte it uses, so nothing needs
 *   clearing.  Calls that overlap on the GPU (concurrent streams, or several host threads)
 *   race on the array: order them on one stream.
 *   No cudaMalloc, cudaFree or allocating library routine is called.
 * ------------------------------------------------------------------------------------- */
#define DLMH_NOALLOC_MAX_K 16384
#define DLMH_NOALLOC_MAX_SMS 160
DLMH_API int w8a8_proj_noalloc(const uint8_t* w, const float* w_scale, int n, int k, const dlmh_bf16* x,
                               int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, void* stream);

/* ---------------------------------------------------------------------------------------
 * NVFP4 W4A16 GEMV
 *   out[m, n] = bf16( g * sum_b e4m3(S[n, b]) * sum_{k in b} e2m1(W[n, k]) * x[m, k] )
 * w4a16_gemv_tiers.rs (the W4A16 tiers; more than 32 rows refused);
 * fp8_lut.rs, dequant_nvfp4_to_bf16 (layout and the folded global g).
 *   w_packed      [n, k/2] bytes, element 2i in the low nibble of byte i.
 *   w_block_scale [n, k/16] E4M3 bytes, one per 16 consecutive k of a row.
 *   global_scale  the folded float32 multiplier g.
 *   k % 128 == 0, k <= 8192.  Any rows >= 0: weight passes of at most DLMH_W4A16_MAX_ROWS
 *   (the pages' kernel_within limit of one launch; fewer when the activation tile of a wider
 *   tier does not fit on chip, see dlmh_plan_chunks), each through the narrowest tier of
 *   8 / 16 / 32 rows that covers it; a row's bits do not depend on `rows`.
 * ------------------------------------------------------------------------------------- */
DLMH_API int w4a16_gemv(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int n, int k,
               const dlmh_bf16* x, int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, void* stream);

/* ---------------------------------------------------------------------------------------
 * NVFP4 W4A4: FP4 activations for the wider row edge (w4a16_gemv_tiers.rs,
 * W4a16BatchmTiers: a weight that declares FP4 activations runs its narrow projections
 * W4A4, up to W4A4_MAX_M = 32 rows; NVFP4 layout of fp8_lut.rs).
 *
 * nvfp4_quantize_rows: per row m, every decision in float32 (the pages do not print the
 * activation quantize; this is the plain NVFP4 recipe):
 *   g[m] = amax_k |x[m, k]| / 2688                       (IEEE division; 2688 = 6 * 448)
 *   per 16-value block b:  s[m, b] = e4m3_rn_sat( amax_b / (6 g[m]) )   (6 g: one f32 product)
 *                          S = e4m3(s[m, b]) * g[m]      (one f32 product)
 *                          code = e2m1_rn_sat( x / S )   (IEEE division; ties to even,
 *                          magnitudes above 6 give 6, a negative zero keeps its sign);
 *                          all codes 0 where S == 0.
 *   x      [rows, ldx] BF16, 16-byte aligned, ldx % 8 == 0.  k % 16 == 0.
 *   xq     [rows][k/2] packed codes (row stride k/2, element 2i in the low nibble of byte i),
 *          16-byte aligned.  x_block_scale [rows][k/16] E4M3.  x_global [rows] float32.
 *
 * w4a4_gemv: out[m, n] = bf16( g_w * g[m] * sum_b e4m3(S[n, b]) e4m3(s[m, b])
 *                                           * sum_{k in b} e2m1(W[n, k]) e2m1(X[m, k]) )
 *   Both operands are decoded exactly to f16 (E2M1 x E4M3 has at most 6 significant bits)
 *   and multiplied on the tensor cores with f32 accumulation; one BF16 rounding.
 *   w_packed [n, k/2] and w_block_scale [n, k/16] as for w4a16_gemv (16-byte aligned);
 *   xq / x_block_scale / x_global as written by nvfp4_quantize_rows (x_block_scale 2-byte
 *   aligned).  k % 256 == 0.  Any rows: weight passes of up to DLMH_W4A4_MAX_ROWS (fewer when
 *   k is long: dlmh_plan_chunks(DLMH_OP_W4A4, ...)); DLMH_ERR_UNSUPPORTED when no pass fits k.
 *
 * w4a4_proj: per pass, nvfp4_quantize_rows into the scratch, then w4a4_gemv.  xq_scratch
 *   holds min(rows, 32) * k/2 bytes (16-byte aligned), xs_scratch min(rows, 32) * k/16,
 *   xg_scratch min(rows, 32) floats.
 * ------------------------------------------------------------------------------------- */
DLMH_API int nvfp4_quantize_rows(const dlmh_bf16* x, int64_t ldx, int rows, int k, uint8_t* xq,
                                 uint8_t* x_block_scale, float* x_global, void* stream);
DLMH_API int w4a4_gemv(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int n, int k,
                       const uint8_t* xq, const uint8_t* x_block_scale, const float* x_global, int rows,
                       dlmh_bf16* out, int64_t ldc, void* stream);
DLMH_API int w4a4_proj(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale, int n, int k,
                       const dlmh_bf16* x, int64_t ldx, int rows, dlmh_bf16* out, int64_t ldc, uint8_t* xq_scratch,
                       uint8_t* xs_scratch, float* xg_scratch, void* stream);

/* ---------------------------------------------------------------------------------------
 * block_q8_1 row quantize (lm_head_q6k.rs, lm_head_q6k_run: kquant_q8_1_rows_bf16)
 *   Block layout (36 bytes per 32 values): { f16 d; f16 s; int8 qs[32] }.
 *   d = amax / 127 (f32 division), qs = round-half-away( x / d ) (f32 division; 0 when
 *   d == 0), stored d = f16(d), s = f16( d * (float)sum(qs) ).
 *   q8_out: [rows][k/32] blocks, row stride k/32 * 36 bytes, 4-byte aligned.  k % 32 == 0.
 * ------------------------------------------------------------------------------------- */
DLMH_API int q8_1_quantize_rows(const dlmh_bf16* x, int64_t ldx, int rows, int k, void* q8_out, void* stream);

/* ---------------------------------------------------------------------------------------
 * Q6_K x block_q8_1 GEMV
 *   out[m, n] = bf16( sum_sb sum_j d(sb) * sc_j(sb) * d8(m, blk(j)) * sum_{i in j} (q_i - 32) * qs_i )
 * lm_head_q6k.rs, lm_head_q6k_run (kquant_mmvq_q6_k_w).  Super-block byte map: ql[128] at 0,
 * qh[64] at 128, int8 scales[16] at 192, f16 d at 208; element 128h + 32t + l takes its low
 * 4 bits from ql[64h + 32(t&1) + l] (low nibble for t < 2, high for t >= 2) and its top
 * 2 bits from bits 2t..2t+1 of qh[32h + l]; element i uses scales[i/16].
 *   blocks [n][k/256] super-blocks, row stride k/256 * 210 bytes (the raw store layout).
 *   q8     [rows][k/32] block_q8_1 as written by q8_1_quantize_rows.
 *   k % 256 == 0 (set_lm_head_q6k requires hidden % 256 == 0).  Any rows: one weight pass per
 *   64 rows, through the narrowest tier of 8 / 16 / 32 / 64 that covers them (above 8 rows the
 *   q8_1 rows must start 16-byte aligned, else the pass falls back to 8-row launches); the
 *   16-row tier runs as two 8-row passes when k <= 8192 (faster than one 16-row pass).  Every
 *   tier adds the same products in the same order, so a row's bits do not depend on `rows`.
 * ------------------------------------------------------------------------------------- */
DLMH_API int q6k_mmvq(const void* blocks, int n, int k, const void* q8, int rows, dlmh_bf16* out, int64_t ldc,
             void* stream);

/* The Q6_K head for BF16 rows (lm_head_q6k.rs, lm_head_q6k_run): for each chunk of up to
 * DLMH_Q6K_MAX_ROWS rows, q8_1_quantize_rows into q8_scratch, then q6k_mmvq.  q8_scratch holds
 * at least min(rows, 64) * k/32 * 36 bytes (16-byte aligned for one pass per 64 rows; a
 * 4-byte aligned scratch runs 8-row passes). */
DLMH_API int q6k_lm_head(const void* blocks, int n, int k, const dlmh_bf16* x, int64_t ldx, int rows,
                dlmh_bf16* out, int64_t ldc, void* q8_scratch, void* stream);

/* ---------------------------------------------------------------------------------------
 * Load-time FP4 dequant to BF16 (the step before the path)
 *
 * NVFP4:  out[n, k] = bf16( e2m1(w[n, k]) * e4m3(s[n, k/16]) * g )
 *   fp8_lut.rs, dequant_nvfp4_to_bf16.  The stored global is folded into one float32
 *   multiplier: is_reciprocal != 0 (compressed-tensors weight_global_scale) gives
 *   g = 1 / global_scale, or 0 when global_scale == 0; is_reciprocal == 0 (ModelOpt
 *   weight_scale_2) gives g = global_scale.  Float32 arithmetic: e2m1 * e4m3 is exact, its
 *   product with g is rounded once to float32, then to BF16 (round-to-nearest-even).
 *   w_packed [n, k/2] E2M1 pairs (element 2i in the low nibble), w_block_scale [n, k/16]
 *   E4M3, both 16-byte aligned; out [n, ldo] BF16, ldo >= k, ldo % 8 == 0, 16-byte aligned.
 *   k % 16 == 0.  Errors as for the GEMV entry points.
 * ------------------------------------------------------------------------------------- */
DLMH_API int nvfp4_dequant_bf16(const uint8_t* w_packed, const uint8_t* w_block_scale, float global_scale,
                                int is_reciprocal, int n, int k, dlmh_bf16* out, int64_t ldo, void* stream);

/* E8M0-scaled FP4:  out[f] = bf16( e2m1(w[f]) * 2^(e[f / block] - 127) ), f the flat (row-major)
 * index, block = n * k / num_scales (DLMH_ERR_SHAPE unless it divides exactly); E8M0 codes 0
 * and 255 decode to 0; no global scale.  fp8_lut.rs, dequant_nvfp4_e8m0_to_bf16 (there a
 * host-side loop; here the same values on the GPU).  The float32 product is exact unless it
 * leaves the float32 range (then +-inf).  w_packed [n * k / 2] 16-byte aligned, scales
 * [num_scales] bytes; out as above; k % 16 == 0. */
DLMH_API int e8m0_fp4_dequant_bf16(const uint8_t* w_packed, const uint8_t* scales, int64_t num_scales, int n, int k,
                                   dlmh_bf16* out, int64_t ldo, void* stream);

/* ---------------------------------------------------------------------------------------
 * Host helpers (no device work; callable without a GPU)
 * ------------------------------------------------------------------------------------- */

/* Operation ids for dlmh_plan_chunks. */
typedef enum dlmh_op {
  DLMH_OP_W8A16 = 0, /* lm_head_fp8_w8a16 */
  DLMH_OP_W8A8 = 1,  /* w8a8_proj / w8a8_silu_proj */
  DLMH_OP_W4A16 = 2, /* w4a16_gemv */
  DLMH_OP_Q6K = 3,   /* q6k_mmvq / q6k_lm_head */
  DLMH_OP_W4A4 = 4,  /* w4a4_gemv / w4a4_proj */
  DLMH_OP_W8A8_PAIR = 5 /* w8a8_gate_up_proj (n = rows of EACH weight) */
} dlmh_op;

/* The weight passes an entry point runs for `rows` at reduction length k: pass i covers rows
 * [offsets[i], offsets[i] + counts[i]) and runs the kernel tier of width tiers[i] (the
 * narrowest compiled tier that covers counts[i], w4a16_gemv_tiers.rs select_tier).
 * For W8A16 and W8A8 with k % 128 == 0 the tensor-core tier serves 128 rows per pass and
 * its width is counts[i] rounded up to 16 (the MMA's N, doubled inside for W8A16).
 * The pass width is a pure function of (op, k) (which kernel serves k, and which activation
 * tile fits on chip), so this needs no GPU.  Returns the number of passes (0 for rows == 0), DLMH_ERR_ROWS for
 * rows < 0, DLMH_ERR_SHAPE for an unknown op or k <= 0,
 * DLMH_ERR_UNSUPPORTED when no tier fits k, DLMH_ERR_CAPACITY when more than `cap`
 * passes are needed.  Arrays may be NULL when cap == 0 (count only). */
DLMH_API int dlmh_plan_chunks(int op, int rows, int k, int* offsets, int* counts, int* tiers, int cap);

/* ---------------------------------------------------------------------------------------
 * Caller-owned workspace (w8a8_layer.rs, W8a8Ctx::new: the scratch is allocated once per
 * model, outside the launch path, and shared by every projection of a stream)
 *
 * dlmh_workspace_bytes: bytes of workspace a call of `op` (a dlmh_op) with weight rows n,
 *   reduction length k and `rows` activation rows needs; a workspace of that size serves
 *   every call of that op and shape with at most `rows` rows.  0 when the call runs no
 *   tensor-core pass (k % 128 != 0, W4A16, W4A4, Q6_K) or rows == 0.  The stream-K schedule
 *   depends on the SM count: sm_count > 0 sizes for that many SMs (host-only, no GPU
 *   needed), 0 for the current device.  Errors: DLMH_ERR_SHAPE (unknown op, n <= 0,
 *   k <= 0, sm_count < 0), DLMH_ERR_ROWS (rows < 0), DLMH_ERR_CUDA (no current device).
 *   Layout (256-byte aligned regions): a 256-byte tile queue, the W8A16 two-term codes
 *   2 * roundup8(min(rows, 128)) * k bytes + 512, the stream-K partial sums
 *   2 * (2 P) * N_mma * 128 * 4 bytes when the schedule has a remainder (P = sm_count / 2
 *   parties of two CTAs over pairs of 128-row tiles; a remainder when the tile pairs are
 *   fewer than P or not a multiple of it).
 *
 * dlmh_set_workspace: binds the device buffer ws (256-byte aligned, `bytes` long, owned by the
 *   caller, kept bound until replaced) to `stream` on the current device.  From then on every
 *   FP8 call on that stream takes its internal scratch from ws and allocates nothing; a call
 *   whose shape needs more than `bytes` returns DLMH_ERR_WORKSPACE before launching anything.
 *   The call zeroes the first 256 bytes (the tile queue) with cudaMemsetAsync on `stream`;
 *   every launch leaves them at zero.  ws == NULL unbinds (calls go back to the pool).  Calls
 *   that use one workspace must not overlap on the GPU: bind one per stream.  The library
 *   never frees ws; unbind before freeing it, and before destroying the stream (a call being
 *   captured into a CUDA graph finds its stream's workspace by the stream handle, which a
 *   new stream may reuse; eager calls use the stream's id).  Bind outside stream capture
 *   (DLMH_ERR_UNSUPPORTED while the stream is capturing).  Errors: DLMH_ERR_ALIGN,
 *   DLMH_ERR_WORKSPACE (bytes < 256), DLMH_ERR_CAPACITY (1024 streams bound),
 *   DLMH_ERR_CUDA.  (No counterpart in the pages' argument lists: their scratch is a field
 *   of the context; here the stream carries it, so the entry points keep the pages' lists.)
 *
 * dlmh_pool_stats: bytes of the library pool of the current device in use now and at the
 *   peak since the last reset (both 0 before the pool's first use); reset_high != 0 sets the
 *   peak back to the current use.  A diagnostic: a stream with a workspace never raises them.
 * ------------------------------------------------------------------------------------- */
DLMH_API int64_t dlmh_workspace_bytes(int op, int n, int k, int rows, int sm_count);
DLMH_API int dlmh_set_workspace(void* ws, size_t bytes, void* stream);
DLMH_API int dlmh_pool_stats(int64_t* used_current, int64_t* used_high, int reset_high);

/* Fault bits recorded on the current device by the kernels' bounded waits (a wait for a
 * shared-memory stage that did not complete in time; the kernel then finishes without
 * hanging and its output is not valid).  0 in a healthy run.  Synchronizes the device;
 * reset != 0 clears the bits.  Returns DLMH_ERR_CUDA if the device cannot be read.
 * (Library diagnostic, no counterpart on the pages.) */
DLMH_API int dlmh_device_fault(int reset);

/* Failure-detection check (library diagnostic, no counterpart on the pages): runs one bounded
 * mbarrier wait on a barrier that nothing completes, the same wait every TMA / tensor-core
 * kernel here uses instead of an unbounded spin, and returns DLMH_OK when it gave up (after
 * 2^22 polls, well under a second) and recorded its fault bit; the bit is cleared again and the
 * other bits are left as they were.  Synchronizes `stream`; DLMH_ERR_CUDA otherwise. */
DLMH_API int dlmh_check_bounded_wait(void* stream);

/* Static description of a status code (never NULL). */
DLMH_API const char* dlmh_error_string(int code);

/* Library version: major * 10000 + minor * 100 + patch. */
DLMH_API int dlmh_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DLMH_H_ */
