"""Seeded synthetic inputs shaped like the decode LM-head / projection workloads.

This module holds no arithmetic of the GEMV method: it only draws random numbers with
torch's generators and casts them to storage formats with torch's own conversions
(float32 -> float8_e4m3fn / bfloat16 / float16, round-to-nearest-even).  Both the GPU
path and the CPU oracle consume what it returns.

Recipes (one torch.Generator per tensor, seeded with seed * 1000 + tensor id):
  * FP8 weight: E4M3 codes of clamp(N(0,1) * 64, -448, 448); row scales U[1e-3, 4e-3].
  * BF16 activations: bf16(N(0,1) * std).
  * NVFP4: packed bytes uniform 0..255 (uniform E2M1 codes); E4M3 block scales of
    U[0.5, 4]; global float32(1) / float32(448).
  * Q6_K: ql / qh bytes uniform 0..255 (uniform 6-bit codes), int8 sub-scales uniform in
    -32..31, f16 d of U[1e-4, 1e-3]; shape [n, k/256, 210].
Generation runs on `device` in row chunks so a 1.27 GB head never needs a 5 GB temporary.
"""

import numpy as np
import torch

_CHUNK = 8192


def _gen(seed, tensor_id, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000 + int(tensor_id))
    return g


def fp8_weight(n, k, seed, device="cpu", tensor_id=1):
    """E4M3 codes [n, k] (uint8) of clamp(N(0,1)*64, +-448)."""
    out = torch.empty(n, k, dtype=torch.uint8, device=device)
    g = _gen(seed, tensor_id, device)
    for r in range(0, n, _CHUNK):
        e = min(n, r + _CHUNK)
        v = torch.randn(e - r, k, generator=g, device=device, dtype=torch.float32)
        v.mul_(64.0).clamp_(-448.0, 448.0)
        out[r:e] = v.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def row_scales(n, seed, device="cpu", tensor_id=2, lo=1e-3, hi=4e-3):
    """float32 [n] uniform in [lo, hi)."""
    g = _gen(seed, tensor_id, device)
    return torch.rand(n, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def bf16_rows(m, k, seed, device="cpu", tensor_id=3, std=1.0):
    """bf16 [m, k] of N(0,1) * std."""
    g = _gen(seed, tensor_id, device)
    return (torch.randn(m, k, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def nvfp4_weight(n, k, seed, device="cpu"):
    """(packed uint8 [n, k/2], block scales uint8 [n, k/16], global float) for the NVFP4 recipe."""
    g = _gen(seed, 11, device)
    packed = torch.randint(0, 256, (n, k // 2), generator=g, device=device, dtype=torch.int32).to(torch.uint8)
    g2 = _gen(seed, 12, device)
    s = torch.rand(n, k // 16, generator=g2, device=device, dtype=torch.float32) * 3.5 + 0.5
    scales = s.to(torch.float8_e4m3fn).view(torch.uint8)
    glob = float(np.float32(1.0) / np.float32(448.0))
    return packed, scales, glob


def q6k_blocks(n, k, seed, device="cpu"):
    """Q6_K super-blocks uint8 [n, k/256, 210] for the Q6_K recipe."""
    nsb = k // 256
    out = torch.empty(n, nsb, 210, dtype=torch.uint8, device=device)
    g = _gen(seed, 21, device)
    for r in range(0, n, _CHUNK):
        e = min(n, r + _CHUNK)
        rows = e - r
        out[r:e, :, 0:192] = torch.randint(0, 256, (rows, nsb, 192), generator=g, device=device,
                                           dtype=torch.int32).to(torch.uint8)
        sc = torch.randint(-32, 32, (rows, nsb, 16), generator=g, device=device, dtype=torch.int32).to(torch.int8)
        out[r:e, :, 192:208] = sc.view(torch.uint8)
        d = (torch.rand(rows, nsb, generator=g, device=device, dtype=torch.float32) * 9e-4 + 1e-4).to(torch.float16)
        out[r:e, :, 208:210] = d.view(torch.uint8).reshape(rows, nsb, 2)
    return out


def to_numpy_bits(t):
    """Tensor -> numpy with raw bit patterns (bf16 / f16 as uint16, uint8 as is)."""
    t = t.detach().cpu().contiguous()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
