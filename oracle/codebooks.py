"""The evenly spaced int4 comparison codebook, float64 oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "What is QLoRA ..." (mantramindai.in), "Follow-up questions to
expect": plain int4 spaces its 16 levels evenly and so spends levels on rare
large values, while NF4 follows the bell-shaped weights and errs less for the
same 4 bits. To measure that claim on equal terms the comparison codec keeps
everything of the NF4 format (blocks of 64, absmax scaling, the same 8-bit
double quantisation, packing, ties to the lower index) and changes only the
levels: (k - 8) / 7 for k = 0..15 rounded to float32, so code 8 is zero,
codes 1 and 15 are -1 and +1, and code 0 (-8/7) is never chosen.
"""

from __future__ import annotations

import numpy as np

from . import nf4

INT4_ZERO_CODE = 8


def int4_levels() -> np.ndarray:
    return (np.arange(16, dtype=np.float64) - 8.0).__truediv__(7.0).astype(np.float32)


def quantize_int4(W: np.ndarray):
    """The NF4 format's encoding with the int4 levels: (packed codes, scale8, scale2)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % nf4.BLOCK != 0:
        raise ValueError("W must be [N, K] with K % 64 == 0")
    if not np.all(np.isfinite(W)):
        raise nf4.NonFiniteInput("non-finite weight")
    c1 = nf4.block_absmax(W)
    codes = nf4.encode_blocks(W, c1, int4_levels()).reshape(-1, nf4.BLOCK)
    codes[c1 == 0] = INT4_ZERO_CODE   # an all-zero block takes the zero level's code
    scale8, scale2 = nf4.double_quantize(c1)
    return nf4.pack_codes(codes.reshape(-1)), scale8, scale2


def dequantize_int4_bits(packed, scale8, scale2, rows: int, cols: int) -> np.ndarray:
    """bf16 bit patterns of RN_bf16(RN32(level * s)) with the int4 levels."""
    levels = int4_levels().astype(np.float64)
    codes = nf4.unpack_codes(packed).reshape(-1, nf4.BLOCK)
    s = nf4.block_scales(scale8, scale2).astype(np.float64)
    prod = (levels[codes] * s[:, None]).astype(np.float32)
    return nf4.bf16_round_bits(prod.reshape(-1)).reshape(rows, cols)
