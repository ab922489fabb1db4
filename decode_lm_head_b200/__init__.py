"""B200-native decode LM-head / projection GEMV (FP8 W8A16, W8A8, NVFP4 W4A16, Q6_K).

The compute path is libdlmh.so (hand-written sm_100a CUDA behind a C ABI, declared in
include/dlmh.h); this package is its thin ctypes binding plus the seeded synthetic input
generators used by the tests and the benchmark.
"""

from ._lib import (  # noqa: F401
    DlmhError,
    OP_Q6K,
    OP_W4A4,
    OP_W4A16,
    OP_W8A8,
    OP_W8A8_PAIR,
    OP_W8A16,
    check_bounded_wait,
    device_fault,
    e8m0_fp4_dequant_bf16,
    error_string,
    lib,
    lm_head_fp8_w8a16,
    nvfp4_dequant_bf16,
    nvfp4_quantize_rows,
    plan_chunks,
    pool_stats,
    q6k_lm_head,
    q6k_mmvq,
    q8_1_quantize_rows,
    set_workspace,
    version,
    w4a16_gemv,
    w4a4_gemv,
    w4a4_proj,
    w8a8_gate_up_proj,
    w8a8_gemv,
    w8a8_proj,
    w8a8_proj_noalloc,
    w8a8_quantize_rows,
    w8a8_silu_proj,
    w8a8_silu_quantize_rows,
    workspace_bytes,
)
