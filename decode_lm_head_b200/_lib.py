"""ctypes binding of libdlmh.so: argument marshalling only.

Every function here takes torch CUDA tensors, checks that they are on the GPU with the
layout the C ABI wants, and passes raw pointers, sizes, leading dimensions and the current
CUDA stream to the library.  There is no fallback: without the built library, or with CPU
tensors, every call raises.
"""

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# DLMH_LIBRARY may point at another build of the same library (for example a tuning build).
LIB_PATH = os.environ.get("DLMH_LIBRARY") or os.path.join(_HERE, "libdlmh.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "dlmh.h")

# op ids of dlmh_plan_chunks (dlmh_op in dlmh.h)
OP_W8A16, OP_W8A8, OP_W4A16, OP_Q6K, OP_W4A4, OP_W8A8_PAIR = 0, 1, 2, 3, 4, 5
W4A4_MAX_ROWS = 32

W8A8_MAX_ROWS = 128
W8A16_CHUNK_ROWS = 16
W4A16_MAX_ROWS = 32
Q6K_CHUNK_ROWS = 8
Q6K_MAX_ROWS = 64
Q8_1_BLOCK_BYTES = 36
Q6K_BLOCK_BYTES = 210


class DlmhError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {error_string(code)} (status {code})")


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_F = ctypes.c_float

_SIGNATURES = {
    "lm_head_fp8_w8a16": [_P, _P, _I, _I, _P, _L, _I, _P, _L, _P],
    "w8a8_quantize_rows": [_P, _L, _I, _I, _P, _L, _P, _P],
    "w8a8_silu_quantize_rows": [_P, _P, _L, _I, _I, _P, _L, _P, _P],
    "w8a8_gemv": [_P, _P, _I, _I, _P, _L, _P, _I, _P, _L, _P],
    "w8a8_proj": [_P, _P, _I, _I, _P, _L, _I, _P, _L, _P, _P, _P],
    "w8a8_silu_proj": [_P, _P, _I, _I, _P, _P, _L, _I, _P, _L, _P, _P, _P],
    "w8a8_gate_up_proj": [_P, _P, _P, _P, _I, _I, _P, _L, _I, _P, _P, _L, _P, _P, _P],
    "w8a8_proj_noalloc": [_P, _P, _I, _I, _P, _L, _I, _P, _L, _P],
    "w4a16_gemv": [_P, _P, _F, _I, _I, _P, _L, _I, _P, _L, _P],
    "nvfp4_quantize_rows": [_P, _L, _I, _I, _P, _P, _P, _P],
    "w4a4_gemv": [_P, _P, _F, _I, _I, _P, _P, _P, _I, _P, _L, _P],
    "w4a4_proj": [_P, _P, _F, _I, _I, _P, _L, _I, _P, _L, _P, _P, _P, _P],
    "q8_1_quantize_rows": [_P, _L, _I, _I, _P, _P],
    "q6k_mmvq": [_P, _I, _I, _P, _I, _P, _L, _P],
    "q6k_lm_head": [_P, _I, _I, _P, _L, _I, _P, _L, _P, _P],
    "nvfp4_dequant_bf16": [_P, _P, _F, _I, _I, _I, _P, _L, _P],
    "e8m0_fp4_dequant_bf16": [_P, _P, _L, _I, _I, _P, _L, _P],
    "dlmh_plan_chunks": [_I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I), _I],
    "dlmh_set_workspace": [_P, ctypes.c_size_t, _P],
    "dlmh_pool_stats": [ctypes.POINTER(_L), ctypes.POINTER(_L), _I],
    "dlmh_device_fault": [_I],
    "dlmh_check_bounded_wait": [_P],
    "dlmh_version": [],
}


def lib():
    """Load libdlmh.so (built in-tree by ``python -m decode_lm_head_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m decode_lm_head_b200.build`")
        h = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGNATURES.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = _I
        h.dlmh_error_string.argtypes = [_I]
        h.dlmh_error_string.restype = ctypes.c_char_p
        h.dlmh_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
        h.dlmh_workspace_bytes.restype = _L
        _lib = h
    return _lib


def header_functions():
    """Names of the functions declared in include/dlmh.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_0-9]+)\s*\(", text, flags=re.M)))


def error_string(code):
    return lib().dlmh_error_string(int(code)).decode()


def version():
    return lib().dlmh_version()


def device_fault(reset=False):
    """Fault bits of the kernels' bounded waits on the current device (0 when healthy)."""
    rc = lib().dlmh_device_fault(1 if reset else 0)
    if rc < 0:
        raise DlmhError(rc, "dlmh_device_fault")
    return rc


def check_bounded_wait(stream=None):
    """Run the library's bounded-wait check on the current device (see dlmh.h)."""
    _check(lib().dlmh_check_bounded_wait(_stream(stream)), "dlmh_check_bounded_wait")


def workspace_bytes(op, n, k, rows, sm_count=0):
    """Bytes of caller workspace a call of `op` (n weight rows, reduction k, up to `rows` rows)
    needs; sm_count 0 sizes for the current device (see dlmh.h)."""
    rc = lib().dlmh_workspace_bytes(op, n, k, rows, sm_count)
    if rc < 0:
        raise DlmhError(rc, "dlmh_workspace_bytes")
    return rc


def set_workspace(ws, stream=None):
    """Bind the CUDA uint8 tensor `ws` (256-byte aligned) as the workspace of `stream` (the
    current stream if None); ws=None unbinds.  The caller keeps `ws` alive while bound."""
    if ws is None:
        _check(lib().dlmh_set_workspace(None, 0, _stream(stream)), "dlmh_set_workspace")
        return
    _cuda(ws, torch.uint8, "ws", 1)
    _check(lib().dlmh_set_workspace(_ptr(ws), ws.numel(), _stream(stream, ws.device)), "dlmh_set_workspace")


def pool_stats(reset_high=False):
    """(bytes in use, peak bytes) of the library pool on the current device."""
    cur, high = _L(0), _L(0)
    _check(lib().dlmh_pool_stats(ctypes.byref(cur), ctypes.byref(high), 1 if reset_high else 0), "dlmh_pool_stats")
    return cur.value, high.value


def _check(rc, what):
    if rc != 0:
        raise DlmhError(rc, what)


_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device=None):
    """The cudaStream_t to launch on, as an int (the current stream of `device` if None)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_current_stream is not None:
        index = device.index if device is not None and device.index is not None else torch.cuda.current_device()
        return _raw_current_stream(index)
    return torch.cuda.current_stream().cuda_stream


def _cuda(t, dtype, name, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libdlmh has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    if ndim >= 1 and t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name} must be contiguous in its last dim")
    return t


def _ld(t):
    return t.stride(0) if t.shape[0] > 1 else max(t.shape[1], t.stride(0))


def _ptr(t):
    return t.data_ptr()


def plan_chunks(op, rows, k):
    """Host-only: list of (offset, count, tier) passes for op/rows/k (no GPU needed)."""
    n = lib().dlmh_plan_chunks(op, rows, k, None, None, None, 0)
    if n < 0:
        raise DlmhError(n, "dlmh_plan_chunks")
    if n == 0:
        return []
    arr = (_I * n)
    o, c, t = arr(), arr(), arr()
    rc = lib().dlmh_plan_chunks(op, rows, k, o, c, t, n)
    if rc != n:
        raise DlmhError(rc, "dlmh_plan_chunks")
    return list(zip(o, c, t))


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------


def lm_head_fp8_w8a16(w, w_scale, x, out=None, stream=None):
    """FP8 E4M3 W8A16 GEMV: out[m, n] = bf16(s[n] * sum_k e4m3(w[n,k]) x[m,k])."""
    _cuda(w, torch.uint8, "w", 2)
    _cuda(w_scale, torch.float32, "w_scale", 1)
    _cuda(x, torch.bfloat16, "x", 2)
    n, k = w.shape
    rows = x.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    _cuda(out, torch.bfloat16, "out", 2)
    _check(lib().lm_head_fp8_w8a16(_ptr(w), _ptr(w_scale), n, k, _ptr(x), _ld(x), rows, _ptr(out), _ld(out),
                                   _stream(stream, x.device)), "lm_head_fp8_w8a16")
    return out


def w8a8_quantize_rows(x, xq=None, x_scale=None, stream=None):
    _cuda(x, torch.bfloat16, "x", 2)
    rows, k = x.shape
    if xq is None:
        xq = torch.empty(rows, k, dtype=torch.uint8, device=x.device)
    if x_scale is None:
        x_scale = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib().w8a8_quantize_rows(_ptr(x), _ld(x), rows, k, _ptr(xq), _ld(xq), _ptr(x_scale),
                                    _stream(stream, x.device)), "w8a8_quantize_rows")
    return xq, x_scale


def w8a8_silu_quantize_rows(gate, up, xq=None, x_scale=None, stream=None):
    _cuda(gate, torch.bfloat16, "gate", 2)
    _cuda(up, torch.bfloat16, "up", 2)
    if gate.shape != up.shape or _ld(gate) != _ld(up):
        raise ValueError("gate and up must have the same shape and row stride")
    rows, k = gate.shape
    if xq is None:
        xq = torch.empty(rows, k, dtype=torch.uint8, device=gate.device)
    if x_scale is None:
        x_scale = torch.empty(rows, dtype=torch.float32, device=gate.device)
    _check(lib().w8a8_silu_quantize_rows(_ptr(gate), _ptr(up), _ld(gate), rows, k, _ptr(xq), _ld(xq),
                                         _ptr(x_scale), _stream(stream, gate.device)), "w8a8_silu_quantize_rows")
    return xq, x_scale


def w8a8_gemv(w, w_scale, xq, x_scale, out=None, stream=None):
    _cuda(w, torch.uint8, "w", 2)
    _cuda(w_scale, torch.float32, "w_scale", 1)
    _cuda(xq, torch.uint8, "xq", 2)
    _cuda(x_scale, torch.float32, "x_scale", 1)
    n, k = w.shape
    rows = xq.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=w.device)
    _check(lib().w8a8_gemv(_ptr(w), _ptr(w_scale), n, k, _ptr(xq), _ld(xq), _ptr(x_scale), rows, _ptr(out),
                           _ld(out), _stream(stream, xq.device)), "w8a8_gemv")
    return out


def _w8a8_scratch(k, device, xq_scratch, xscale_scratch):
    if xq_scratch is None:
        xq_scratch = torch.empty(W8A8_MAX_ROWS * k, dtype=torch.uint8, device=device)
    if xscale_scratch is None:
        xscale_scratch = torch.empty(W8A8_MAX_ROWS, dtype=torch.float32, device=device)
    return xq_scratch, xscale_scratch


def w8a8_proj(w, w_scale, x, out=None, xq_scratch=None, xscale_scratch=None, stream=None):
    _cuda(w, torch.uint8, "w", 2)
    _cuda(w_scale, torch.float32, "w_scale", 1)
    _cuda(x, torch.bfloat16, "x", 2)
    n, k = w.shape
    rows = x.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    xq_scratch, xscale_scratch = _w8a8_scratch(k, x.device, xq_scratch, xscale_scratch)
    _check(lib().w8a8_proj(_ptr(w), _ptr(w_scale), n, k, _ptr(x), _ld(x), rows, _ptr(out), _ld(out),
                           _ptr(xq_scratch), _ptr(xscale_scratch), _stream(stream, x.device)), "w8a8_proj")
    return out


def w8a8_proj_noalloc(w, w_scale, x, out=None, stream=None):
    """w8a8_proj with the library's own fixed device scratch (no caller scratch, no allocation
    inside the library)."""
    _cuda(w, torch.uint8, "w", 2)
    _cuda(w_scale, torch.float32, "w_scale", 1)
    _cuda(x, torch.bfloat16, "x", 2)
    n, k = w.shape
    rows = x.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    _check(lib().w8a8_proj_noalloc(_ptr(w), _ptr(w_scale), n, k, _ptr(x), _ld(x), rows, _ptr(out), _ld(out),
                                   _stream(stream, x.device)), "w8a8_proj_noalloc")
    return out


def w8a8_silu_proj(w, w_scale, gate, up, out=None, xq_scratch=None, xscale_scratch=None, stream=None):
    _cuda(w, torch.uint8, "w", 2)
    _cuda(w_scale, torch.float32, "w_scale", 1)
    _cuda(gate, torch.bfloat16, "gate", 2)
    _cuda(up, torch.bfloat16, "up", 2)
    if gate.shape != up.shape or _ld(gate) != _ld(up):
        raise ValueError("gate and up must have the same shape and row stride")
    n, k = w.shape
    rows = gate.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=gate.device)
    xq_scratch, xscale_scratch = _w8a8_scratch(k, gate.device, xq_scratch, xscale_scratch)
    _check(lib().w8a8_silu_proj(_ptr(w), _ptr(w_scale), n, k, _ptr(gate), _ptr(up), _ld(gate), rows, _ptr(out),
                                _ld(out), _ptr(xq_scratch), _ptr(xscale_scratch), _stream(stream, gate.device)),
           "w8a8_silu_proj")
    return out


def w8a8_gate_up_proj(w_gate, s_gate, w_up, s_up, x, gate_out=None, up_out=None, xq_scratch=None,
                      xscale_scratch=None, stream=None):
    """(gate, up) = the two W8A8 projections of x on one quantized copy of it."""
    for t, name in ((w_gate, "w_gate"), (w_up, "w_up")):
        _cuda(t, torch.uint8, name, 2)
    for t, name in ((s_gate, "s_gate"), (s_up, "s_up")):
        _cuda(t, torch.float32, name, 1)
    _cuda(x, torch.bfloat16, "x", 2)
    if w_gate.shape != w_up.shape:
        raise ValueError("w_gate and w_up must have the same shape")
    n, k = w_gate.shape
    rows = x.shape[0]
    if gate_out is None:
        gate_out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    if up_out is None:
        up_out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    if _ld(gate_out) != _ld(up_out):
        raise ValueError("gate_out and up_out must have the same row stride")
    xq_scratch, xscale_scratch = _w8a8_scratch(k, x.device, xq_scratch, xscale_scratch)
    _check(lib().w8a8_gate_up_proj(_ptr(w_gate), _ptr(s_gate), _ptr(w_up), _ptr(s_up), n, k, _ptr(x), _ld(x), rows,
                                   _ptr(gate_out), _ptr(up_out), _ld(gate_out), _ptr(xq_scratch),
                                   _ptr(xscale_scratch), _stream(stream, x.device)),
           "w8a8_gate_up_proj")
    return gate_out, up_out


def w4a16_gemv(w_packed, w_block_scale, global_scale, x, out=None, stream=None):
    _cuda(w_packed, torch.uint8, "w_packed", 2)
    _cuda(w_block_scale, torch.uint8, "w_block_scale", 2)
    _cuda(x, torch.bfloat16, "x", 2)
    n, k2 = w_packed.shape
    k = 2 * k2
    if tuple(w_block_scale.shape) != (n, k // 16):
        raise ValueError("w_block_scale must be [n, k/16]")
    rows = x.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    _check(lib().w4a16_gemv(_ptr(w_packed), _ptr(w_block_scale), float(global_scale), n, k, _ptr(x), _ld(x), rows,
                            _ptr(out), _ld(out), _stream(stream, x.device)), "w4a16_gemv")
    return out


def nvfp4_quantize_rows(x, xq=None, x_block_scale=None, x_global=None, stream=None):
    """(codes [rows, k/2] uint8, block scales [rows, k/16] uint8, globals [rows] f32)."""
    _cuda(x, torch.bfloat16, "x", 2)
    rows, k = x.shape
    if xq is None:
        xq = torch.empty(rows, k // 2, dtype=torch.uint8, device=x.device)
    if x_block_scale is None:
        x_block_scale = torch.empty(rows, k // 16, dtype=torch.uint8, device=x.device)
    if x_global is None:
        x_global = torch.empty(rows, dtype=torch.float32, device=x.device)
    _check(lib().nvfp4_quantize_rows(_ptr(x), _ld(x), rows, k, _ptr(xq), _ptr(x_block_scale), _ptr(x_global),
                                     _stream(stream, x.device)), "nvfp4_quantize_rows")
    return xq, x_block_scale, x_global


def _w4a4_weight(w_packed, w_block_scale):
    _cuda(w_packed, torch.uint8, "w_packed", 2)
    _cuda(w_block_scale, torch.uint8, "w_block_scale", 2)
    n, k2 = w_packed.shape
    k = 2 * k2
    if tuple(w_block_scale.shape) != (n, k // 16):
        raise ValueError("w_block_scale must be [n, k/16]")
    return n, k


def w4a4_gemv(w_packed, w_block_scale, global_scale, xq, x_block_scale, x_global, out=None, stream=None):
    n, k = _w4a4_weight(w_packed, w_block_scale)
    _cuda(xq, torch.uint8, "xq", 2)
    rows = xq.shape[0]
    if tuple(xq.shape) != (rows, k // 2) or tuple(x_block_scale.shape) != (rows, k // 16) or \
            tuple(x_global.shape) != (rows,) or not xq.is_contiguous() or not x_block_scale.is_contiguous():
        raise ValueError("xq [rows, k/2], x_block_scale [rows, k/16] (contiguous), x_global [rows]")
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=xq.device)
    _check(lib().w4a4_gemv(_ptr(w_packed), _ptr(w_block_scale), float(global_scale), n, k, _ptr(xq),
                           _ptr(x_block_scale), _ptr(x_global), rows, _ptr(out), _ld(out),
                           _stream(stream, xq.device)), "w4a4_gemv")
    return out


def w4a4_proj(w_packed, w_block_scale, global_scale, x, out=None, xq_scratch=None, xs_scratch=None,
              xg_scratch=None, stream=None):
    n, k = _w4a4_weight(w_packed, w_block_scale)
    _cuda(x, torch.bfloat16, "x", 2)
    rows = x.shape[0]
    r = max(1, min(rows, W4A4_MAX_ROWS))
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    if xq_scratch is None:
        xq_scratch = torch.empty(r * k // 2, dtype=torch.uint8, device=x.device)
    if xs_scratch is None:
        xs_scratch = torch.empty(r * k // 16, dtype=torch.uint8, device=x.device)
    if xg_scratch is None:
        xg_scratch = torch.empty(r, dtype=torch.float32, device=x.device)
    _check(lib().w4a4_proj(_ptr(w_packed), _ptr(w_block_scale), float(global_scale), n, k, _ptr(x), _ld(x), rows,
                           _ptr(out), _ld(out), _ptr(xq_scratch), _ptr(xs_scratch), _ptr(xg_scratch),
                           _stream(stream, x.device)), "w4a4_proj")
    return out


def q8_1_quantize_rows(x, q8=None, stream=None):
    _cuda(x, torch.bfloat16, "x", 2)
    rows, k = x.shape
    if q8 is None:
        q8 = torch.empty(rows, k // 32, Q8_1_BLOCK_BYTES, dtype=torch.uint8, device=x.device)
    _check(lib().q8_1_quantize_rows(_ptr(x), _ld(x), rows, k, _ptr(q8), _stream(stream, x.device)),
           "q8_1_quantize_rows")
    return q8


def q6k_mmvq(blocks, q8, out=None, stream=None):
    _cuda(blocks, torch.uint8, "blocks", 3)
    _cuda(q8, torch.uint8, "q8", 3)
    if not blocks.is_contiguous() or not q8.is_contiguous():
        raise ValueError("blocks and q8 must be contiguous")
    n, nsb, _ = blocks.shape
    k = nsb * 256
    rows = q8.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=blocks.device)
    _check(lib().q6k_mmvq(_ptr(blocks), n, k, _ptr(q8), rows, _ptr(out), _ld(out), _stream(stream, q8.device)),
           "q6k_mmvq")
    return out


def q6k_lm_head(blocks, x, out=None, q8_scratch=None, stream=None):
    _cuda(blocks, torch.uint8, "blocks", 3)
    _cuda(x, torch.bfloat16, "x", 2)
    if not blocks.is_contiguous():
        raise ValueError("blocks must be contiguous")
    n, nsb, _ = blocks.shape
    k = nsb * 256
    rows = x.shape[0]
    if out is None:
        out = torch.empty(rows, n, dtype=torch.bfloat16, device=x.device)
    if q8_scratch is None:
        q8_scratch = torch.empty(min(rows, Q6K_MAX_ROWS) * (k // 32) * Q8_1_BLOCK_BYTES, dtype=torch.uint8,
                                 device=x.device)
    _check(lib().q6k_lm_head(_ptr(blocks), n, k, _ptr(x), _ld(x), rows, _ptr(out), _ld(out), _ptr(q8_scratch),
                             _stream(stream, x.device)), "q6k_lm_head")
    return out


# ---------------------------------------------------------------------------
# load-time FP4 dequant
# ---------------------------------------------------------------------------


def nvfp4_dequant_bf16(w_packed, w_block_scale, global_scale, is_reciprocal, out=None, stream=None):
    """NVFP4 [n, k/2] codes + [n, k/16] E4M3 block scales -> BF16 [n, k] (see dlmh.h)."""
    _cuda(w_packed, torch.uint8, "w_packed", 2)
    _cuda(w_block_scale, torch.uint8, "w_block_scale", 2)
    n, k2 = w_packed.shape
    k = 2 * k2
    if tuple(w_block_scale.shape) != (n, k // 16):
        raise ValueError("w_block_scale must be [n, k/16]")
    if out is None:
        out = torch.empty(n, k, dtype=torch.bfloat16, device=w_packed.device)
    _check(lib().nvfp4_dequant_bf16(_ptr(w_packed), _ptr(w_block_scale), float(global_scale),
                                    1 if is_reciprocal else 0, n, k, _ptr(out), _ld(out),
                                    _stream(stream, w_packed.device)), "nvfp4_dequant_bf16")
    return out


def e8m0_fp4_dequant_bf16(w_packed, scales, n, k, out=None, stream=None):
    """E2M1 pairs (n*k/2 bytes) + E8M0 group scales -> BF16 [n, k] (see dlmh.h)."""
    if not isinstance(w_packed, torch.Tensor) or not w_packed.is_cuda or w_packed.dtype != torch.uint8:
        raise TypeError("w_packed must be a CUDA uint8 tensor")
    if not isinstance(scales, torch.Tensor) or not scales.is_cuda or scales.dtype != torch.uint8:
        raise TypeError("scales must be a CUDA uint8 tensor")
    if not w_packed.is_contiguous() or not scales.is_contiguous() or w_packed.numel() * 2 != n * k:
        raise ValueError("w_packed must be n*k/2 contiguous bytes and scales contiguous")
    if out is None:
        out = torch.empty(n, k, dtype=torch.bfloat16, device=w_packed.device)
    _check(lib().e8m0_fp4_dequant_bf16(_ptr(w_packed), _ptr(scales), scales.numel(), n, k, _ptr(out), _ld(out),
                                       _stream(stream, w_packed.device)), "e8m0_fp4_dequant_bf16")
    return out
