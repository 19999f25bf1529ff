"""Seeded synthetic inputs for the five MX workloads.

This module holds only random-number generation: no quantisation, scale or codec
arithmetic.  Both the CUDA path's tests/benchmark and the CPU oracle read the same
bytes produced here.  Every generator draws fp32 values with ``numpy.random.default_rng``
and rounds them to bf16 (round-to-nearest-even, by torch's dtype conversion); the result
is returned as uint16 bf16 bit patterns, row-major.

Workloads (shapes and distributions of the MX pages' use cases):
  mx8_rowwise   1024 x 1024, N(0,1) * 2^u per row with u ~ U[-8, 8], 1% of entries x100
  weight_fp4    4096 x 4096, N(0, 0.02), 0.1% of entries replaced by N(0, 1)
  activations   16384 x 4096, N(0,1) * per-column 2^v with v ~ U[-4, 4]
  gradients     16384 x 14336, N(0, 1e-3) with 5% exact zeros
  gemm operands N(0, 1) activations / N(0, 1) or N(0, 0.02) weights
"""
from __future__ import annotations

import numpy as np
import torch


def to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (RNE, torch conversion) -> uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits_to_float(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal(rows: int, cols: int, sigma: float = 1.0, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(sigma))


def mx8_rowwise(rows: int = 1024, cols: int = 1024, seed: int = 0) -> np.ndarray:
    """N(0,1) times a per-row 2^u, u ~ U[-8, 8]; 1% of entries multiplied by 100."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    u = rng.uniform(-8.0, 8.0, size=(rows, 1)).astype(np.float32)
    x *= np.exp2(u)
    outlier = rng.random((rows, cols)) < 0.01
    x[outlier] *= np.float32(100.0)
    return to_bf16_bits(x)


def weight_fp4(rows: int = 4096, cols: int = 4096, seed: int = 0) -> np.ndarray:
    """N(0, 0.02) with 0.1% of entries replaced by N(0, 1) draws."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(0.02)
    mask = rng.random((rows, cols)) < 0.001
    x[mask] = rng.standard_normal(int(mask.sum()), dtype=np.float32)
    return to_bf16_bits(x)


def activations(rows: int = 16384, cols: int = 4096, seed: int = 0) -> np.ndarray:
    """N(0,1) times a per-channel (column) scale 2^v, v ~ U[-4, 4] (log-uniform)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    v = rng.uniform(-4.0, 4.0, size=(1, cols)).astype(np.float32)
    x *= np.exp2(v)
    return to_bf16_bits(x)


def gradients(rows: int = 16384, cols: int = 14336, seed: int = 1) -> np.ndarray:
    """N(0, 1e-3) with 5% exact zeros."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(1e-3)
    x[rng.random((rows, cols)) < 0.05] = 0.0
    return to_bf16_bits(x)


def special_values_block() -> np.ndarray:
    """Hand-picked edge values (zeros, subnormals, extremes, Inf, NaN) as bf16 bits."""
    vals = [0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x0080, 0x7F7F, 0xFF7F,
            0x3F80, 0xBF80, 0x4300, 0x43E0, 0x43E8, 0x43F0, 0x4760, 0x4770]
    return np.array(vals, dtype=np.uint16)


def nvfp4_quotient_grid(amax_bits: int, cols: int = 256, seed: int = 0) -> np.ndarray:
    """Sixteen-element blocks that sweep the NVFP4 scale and element space for a tensor
    whose largest magnitude is the bf16 pattern ``amax_bits`` (positive, finite).

    Block maxima run over every bf16 magnitude pattern from ``amax_bits - 19*128`` (19
    binades down, floored at the smallest subnormal) up to ``amax_bits``; the other 15
    entries of the blocks led by maximum p take, in turn, every magnitude pattern from
    ``p - 5*128`` up to p (five binades), with random signs; the last block of each
    maximum is padded with signed zeros.  Rows of ``cols`` entries (a multiple of 16),
    zero blocks fill the last row.  Pattern arithmetic only: no scale or codec math.
    """
    assert 0 < amax_bits < 0x7F80 and cols % 16 == 0
    rng = np.random.default_rng(seed)
    blocks = []
    for p in range(max(1, amax_bits - 19 * 128), amax_bits + 1):
        xs = np.arange(max(0, p - 5 * 128), p + 1, dtype=np.uint16)
        pad = (-xs.size) % 15
        xs = np.concatenate([xs, np.zeros(pad, dtype=np.uint16)]).reshape(-1, 15)
        lead = np.full((xs.shape[0], 1), p, dtype=np.uint16)
        blk = np.concatenate([lead, xs], axis=1)
        blk |= (rng.integers(0, 2, blk.shape, dtype=np.uint16) << 15).astype(np.uint16)
        blocks.append(blk)
    b = np.concatenate(blocks, axis=0).reshape(-1)
    b = np.concatenate([b, np.zeros((-b.size) % cols, dtype=np.uint16)])
    return b.reshape(-1, cols)
