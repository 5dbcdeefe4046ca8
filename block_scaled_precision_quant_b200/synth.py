"""Seeded synthetic inputs shaped like the pages' workloads.

This module only draws random numbers: it holds none of the quantization or
GEMM arithmetic, and both the CUDA path's tests/benchmark and the CPU oracle
are fed from it.  Every array is produced on the host from a
``torch.Generator('cpu')`` seeded explicitly, so a (shape, seed) pair always
gives the same bytes.

Distributions (all integers drawn inclusive):
  activations   bf16 N(0, 1), optionally times 2^U{lo..hi} per 32-group
  bias          bf16 N(0, 0.02)
  residual      bf16 N(0, 1)
  MXFP4 weight  uniform bytes (both nibbles cover all 16 E2M1 codes, -0
                included) [N, K/2]; E8M0 scales U{118..126} [N, K/32]
  FP8 weight    uniform over the 254 finite E4M3 bytes [N, K]; E8M0 block
                scales U{120..128} [ceil(N/32), ceil(K/32)]
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def activations(M: int, K: int, seed: int = 0, std: float = 1.0,
                group_pow2: tuple[int, int] | None = None) -> np.ndarray:
    """bf16 bit patterns [M, K] of N(0, std^2) samples; with ``group_pow2``
    = (lo, hi) each 32-element group is multiplied by 2^U{lo..hi}."""
    g = _gen(seed)
    x = torch.randn((M, K), generator=g, dtype=torch.float32) * std
    if group_pow2 is not None and K:
        lo, hi = group_pow2
        e = torch.randint(lo, hi + 1, (M, K // 32), generator=g, dtype=torch.int32)
        x = x * torch.pow(2.0, e.to(torch.float32)).repeat_interleave(32, dim=1)
    return _bf16_bits(x)


def bias(N: int, seed: int = 0, std: float = 0.02) -> np.ndarray:
    g = _gen(seed)
    return _bf16_bits(torch.randn((N,), generator=g, dtype=torch.float32) * std)


def residual(M: int, N: int, seed: int = 0) -> np.ndarray:
    g = _gen(seed)
    return _bf16_bits(torch.randn((M, N), generator=g, dtype=torch.float32))


def mxfp4_weight(N: int, K: int, seed: int = 0, scale_lo: int = 118, scale_hi: int = 126):
    """(packed uint8 [N, K/2], E8M0 scales uint8 [N, K/32])."""
    g = _gen(seed)
    packed = torch.randint(0, 256, (N, K // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    sf = torch.randint(scale_lo, scale_hi + 1, (N, K // 32), generator=g,
                       dtype=torch.int32).to(torch.uint8)
    return packed.numpy().copy(), sf.numpy().copy()


def fp8_weight_blk32(N: int, K: int, seed: int = 0, scale_lo: int = 120, scale_hi: int = 128):
    """(E4M3 codes uint8 [N, K] without 0x7F/0xFF, block scales uint8
    [ceil(N/32), ceil(K/32)])."""
    g = _gen(seed)
    finite = torch.tensor([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=torch.uint8)
    idx = torch.randint(0, finite.numel(), (N, K), generator=g, dtype=torch.int64)
    codes = finite[idx]
    sf = torch.randint(scale_lo, scale_hi + 1, ((N + 31) // 32, (K + 31) // 32), generator=g,
                       dtype=torch.int32).to(torch.uint8)
    return codes.numpy().copy(), sf.numpy().copy()


def uniform_bytes(shape, seed: int = 0, lo: int = 0, hi: int = 255) -> np.ndarray:
    g = _gen(seed)
    return torch.randint(lo, hi + 1, tuple(shape), generator=g,
                         dtype=torch.int32).to(torch.uint8).numpy().copy()
