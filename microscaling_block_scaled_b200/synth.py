"""Seeded synthetic FP32 inputs for the MX GEMM workloads.

This module only draws random numbers; it holds none of the method's
arithmetic (no quantisation, no scaling rule, no product).  Both the CUDA
path and the CPU oracle consume the FP32 tensors it returns, so the two sides
quantise identical bytes.

Recipes (one per workload family):

* ``normal``: A [M][K] then B [N][K], each element N(0, 1) in FP32.
* ``heavy``: as ``normal``, then per 32-element K-block an exponent
  u ~ U(-20, 20) drawn for A's blocks and then for B's blocks, each block
  multiplied by 2^u; then a Bernoulli(1/64) draw per block (A's, then B's)
  sets whole blocks to exact zero.

All draws come from one ``torch.Generator`` seeded with ``seed`` on the
requested device, in the order listed.  CPU and CUDA generators give
different streams for the same seed; every consumer states which one it uses.
"""
from __future__ import annotations

import torch


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def operands(M: int, N: int, K: int, seed: int, kind: str = "normal",
             device: str | torch.device = "cpu"):
    """Return FP32 (A [M][K], B [N][K]) drawn by recipe ``kind``."""
    if K % 32 != 0:
        raise ValueError("K must be a multiple of 32")
    g = _gen(device, seed)
    A = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    B = torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
    if kind == "normal":
        return A, B
    if kind != "heavy":
        raise ValueError("unknown recipe %r" % kind)
    ua = torch.rand(M, K // 32, generator=g, device=device, dtype=torch.float32) * 40.0 - 20.0
    ub = torch.rand(N, K // 32, generator=g, device=device, dtype=torch.float32) * 40.0 - 20.0
    za = torch.rand(M, K // 32, generator=g, device=device, dtype=torch.float32) < (1.0 / 64.0)
    zb = torch.rand(N, K // 32, generator=g, device=device, dtype=torch.float32) < (1.0 / 64.0)
    A = (A.view(M, K // 32, 32) * torch.exp2(ua).unsqueeze(-1))
    B = (B.view(N, K // 32, 32) * torch.exp2(ub).unsqueeze(-1))
    A = A.masked_fill(za.unsqueeze(-1), 0.0).reshape(M, K)
    B = B.masked_fill(zb.unsqueeze(-1), 0.0).reshape(N, K)
    return A.contiguous(), B.contiguous()


# The workloads, by name: (format, M, N, K, seed, recipe).
WORKLOADS = {
    "mxfp8_32x256x512": ("mxfp8", 32, 256, 512, 0, "normal"),
    "mxfp4_32x14336x4096": ("mxfp4", 32, 14336, 4096, 1, "normal"),
    "mxfp8_64x4096x4096": ("mxfp8", 64, 4096, 4096, 2, "normal"),
    "mxfp4_64x4096x4096": ("mxfp4", 64, 4096, 4096, 2, "normal"),
    "mxfp8_2048x28672x8192": ("mxfp8", 2048, 28672, 8192, 3, "normal"),
    "mxfp4_2048x28672x8192": ("mxfp4", 2048, 28672, 8192, 3, "normal"),
    "mxfp8_8192x8192x8192": ("mxfp8", 8192, 8192, 8192, 3, "normal"),
    "mxfp4_8192x8192x8192": ("mxfp4", 8192, 8192, 8192, 3, "normal"),
    "mxfp8_4096x4096x14336": ("mxfp8", 4096, 4096, 14336, 3, "normal"),
    "mxfp4_4096x4096x14336": ("mxfp4", 4096, 4096, 14336, 3, "normal"),
}

# Workloads of the extensions beyond the MX product, by name: op and sizes.
#  bf16:      dense BF16 GEMM (A, B drawn N(0,1) in FP32 then rounded to BF16)
#  grouped:   grouped GEMM, `groups` rows of A per group (uneven, one empty)
#  fused:     MX GEMM with bias + activation + residual in the epilogue
#  quantized: MX GEMM whose epilogue writes the next layer's MX operand
EXTRA_WORKLOADS = {
    "bf16_64x4096x4096": dict(op="bf16", fmt="bf16", M=64, N=4096, K=4096, seed=2),
    "mxfp8_grouped_8x4096x4096_uneven": dict(op="grouped", fmt="mxfp8", groups=(1024, 0, 512, 768, 256, 1280, 128, 128),
                                             N=4096, K=4096, seed=5),
    "mxfp4_32x14336x4096_bias_gelu_residual": dict(op="fused", fmt="mxfp4", M=32, N=14336, K=4096, seed=1, act=3),
    "mxfp4_32x14336x4096_to_mxfp8": dict(op="quantized", fmt="mxfp4", M=32, N=14336, K=4096, seed=1, out_fmt=0),
}

SWEEP_M = (16, 32, 64, 128, 256, 1024, 4096, 8192)
SWEEP_NK = ((4096, 4096), (14336, 4096), (4096, 14336), (8192, 8192), (28672, 8192))
SWEEP_SEED = 4
