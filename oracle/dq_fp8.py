"""NF4 with an 8-bit-float, mean-centred second level: float64 oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page title, section):
  * "QLoRA and Fine-Tuning on One Consumer GPU" (multigrid.ai), "NF4 and
    double quantisation": double quantisation quantises the per-block absmax
    constants themselves and saves about 0.37 bits per parameter; the page
    attributes the method to the QLoRA paper (arXiv 2305.14314).
  * "What is QLoRA ..." (mantramindai.in), "The three QLoRA ideas": the
    constants are quantised to 8 bits in blocks of 256.

The pages fix "8 bits, blocks of 256" and the saving, not the 8-bit format.
The library's main format reads it as unsigned linear absmax codes (nf4.py).
This module is the comparison format the cited paper describes: the block
constants of a group are centred on their mean (they are all positive, so
centring lets a symmetric format use both signs) and stored as 8-bit floats.
Readings:
  * 8-bit float = E4M3 (4 exponent bits, bias 7, 3 mantissa bits, no
    infinities, largest finite 448); encoding rounds to nearest, ties to an
    even mantissa, and saturates to +-448.
  * mean mu_g = RN32(RN64(S / n)) with S the float64 sum of the group's
    constants taken in block order (s <- RN64(s + c1_b)), n the blocks in the
    group.
  * centred constant cen_b = RN32(c1_b - mu_g); a_g = max_b |cen_b|;
    stored scale d_g = RN32(a_g / 448); code q_b = E4M3(RN32(cen_b / d_g))
    (q_b = +0 when d_g = 0).
  * decoded constant s_b = RN32(RN32(e4m3(q_b) * d_g) + mu_g), used as the
    block scale: w' = RN_bf16(RN32(level[code] * s_b)).
  * storage per group: d_g and mu_g (two float32), so 4 + 8/64 + 64/16384 =
    4.12890625 bits per weight.
Every RN32 of an operation on float32 values is computed as float64 and then
rounded to float32, which equals the correctly rounded float32 result for +,
-, * and / (53 >= 2 * 24 + 2).
"""

from __future__ import annotations

import numpy as np

from . import nf4

E4M3_MAX = 448.0
BITS_PER_WEIGHT = 4.0 + 8.0 / nf4.BLOCK + 64.0 / (nf4.BLOCK * nf4.GROUP)


def e4m3_value(code: int) -> float:
    """Value of an E4M3 code (NaN for 0x7F / 0xFF)."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_table() -> np.ndarray:
    """float64 values of all 256 codes."""
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


_POS = e4m3_table()[:127]          # codes 0x00 .. 0x7E: +0 .. 448, increasing


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of each float32 value (ties to the even code,
    magnitudes above 448 saturate to 448, the sign bit follows x's sign)."""
    x = np.asarray(x, dtype=np.float32)
    mag = np.abs(x.astype(np.float64))
    hi = np.clip(np.searchsorted(_POS, mag, side="left"), 0, 126)   # first value >= mag
    lo = np.clip(hi - 1, 0, 126)
    d_lo = mag - _POS[lo]
    d_hi = _POS[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= E4M3_MAX, 126, code)
    sign = np.signbit(x).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return e4m3_table()[np.asarray(codes, dtype=np.uint8)]


def group_mean(c1g: np.ndarray) -> np.float32:
    """mu = RN32(RN64(S / n)), S the block-order float64 sum."""
    s = np.add.accumulate(np.asarray(c1g, dtype=np.float32).astype(np.float64))[-1]
    return np.float32(s / float(c1g.size))


def double_quantize_fp8(c1: np.ndarray):
    """Second level of the comparison format. Returns (scale8 uint8 [nb]
    E4M3 codes, scale2 float32 [ng, 2] rows (d_g, mu_g))."""
    c1 = np.asarray(c1, dtype=np.float32)
    nb = c1.size
    ng = -(-nb // nf4.GROUP)
    q = np.zeros(nb, dtype=np.uint8)
    s2 = np.zeros((ng, 2), dtype=np.float32)
    for g in range(ng):
        sl = slice(g * nf4.GROUP, min(nb, (g + 1) * nf4.GROUP))
        vals = c1[sl]
        mu = group_mean(vals)
        cen = (vals.astype(np.float64) - np.float64(mu)).astype(np.float32)
        a = np.float32(np.max(np.abs(cen)))
        d = np.float32(np.float64(a) / E4M3_MAX)
        if d > 0:
            t = (cen.astype(np.float64) / np.float64(d)).astype(np.float32)
            q[sl] = e4m3_encode(t)
        s2[g] = (d, mu)
    return q, s2


def block_scales_fp8(scale8: np.ndarray, scale2: np.ndarray) -> np.ndarray:
    """s_b = RN32(RN32(e4m3(q_b) * d_g) + mu_g) as float32."""
    q = e4m3_decode(scale8)
    s2 = np.asarray(scale2, dtype=np.float32).reshape(-1, 2).astype(np.float64)
    g = np.arange(q.size) // nf4.GROUP
    prod = (q * s2[g, 0]).astype(np.float32).astype(np.float64)    # exact product, one rounding
    return (prod + s2[g, 1]).astype(np.float32)


def quantize_fp8dq(W: np.ndarray):
    """NF4 codes as in nf4.quantize, second level in the comparison format.
    Returns (packed codes, scale8 E4M3 codes [nb], scale2 float32 [ng, 2])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % nf4.BLOCK != 0:
        raise ValueError("W must be [N, K] with K % 64 == 0")
    if not np.all(np.isfinite(W)):
        raise nf4.NonFiniteInput("non-finite weight")
    c1 = nf4.block_absmax(W)
    codes = nf4.encode_blocks(W, c1, nf4.nf4_levels())
    scale8, scale2 = double_quantize_fp8(c1)
    return nf4.pack_codes(codes), scale8, scale2


def dequantize_fp8dq_bits(packed, scale8, scale2, rows: int, cols: int) -> np.ndarray:
    """bf16 bit patterns of RN_bf16(RN32(level * s_b)) with the decoded s_b."""
    levels = nf4.nf4_levels().astype(np.float64)
    codes = nf4.unpack_codes(packed).reshape(-1, nf4.BLOCK)
    s = block_scales_fp8(scale8, scale2).astype(np.float64)
    prod = (levels[codes] * s[:, None]).astype(np.float32)
    return nf4.bf16_round_bits(prod.reshape(-1)).reshape(rows, cols)
