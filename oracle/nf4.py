"""NF4 codec oracle: codebook, blockwise absmax quantisation, double
quantisation of the block constants, dequantisation to bf16.

TEST INFRASTRUCTURE ONLY (see the package docstring). Plain numpy float64.

Sources (page title, section):
  * "QLoRA, in depth" (aicassindra.com), "The mechanism in brief": NF4 has 16
    levels at quantiles of a normal distribution; W is split into blocks of 64
    values with one scale each; double quantisation stores those scales in
    8 bits with a second-level 32-bit scale for every 256 blocks; on every
    forward W is dequantised to the compute dtype, usually bf16.
  * "What is QLoRA ..." (mantramindai.in), "The three QLoRA ideas": blocks of
    64 with an fp32 scale each; the scales are themselves quantised to 8 bits
    in blocks of 256.
  * "QLoRA and Fine-Tuning on One Consumer GPU" (multigrid.ai), "NF4 and
    double quantisation": blockwise quantisation stores one absmax constant
    per block; NF4 levels sit at normal quantiles; 0.5 byte per parameter.

Readings where the pages are silent:
  * codebook: 8 positive and 7 negative quantiles plus an exact zero, from the
    construction of the paper the multigrid.ai page cites (arXiv 2305.14314),
    restated here as mathematics; offset NF4_OFFSET (parity unpinned: the
    pages do not fix this constant).
  * blocks are 64 consecutive elements of the row-major flattening of W[N, K]
    with K % 64 == 0.
  * normalised value n = RN32(w / c1); code = nearest level, ties to the lower
    index; an all-zero block gets c1 = 0 and every code 7.
  * packing: byte j = (code[2j] << 4) | code[2j + 1].
  * second level: unsigned linear absmax over each group of 256 block
    constants: q8 = round-half-even(255 c1 / c2), stored d = RN32(c2 / 255).
  * dequant: s = RN32(q8 * d); w' = RN_bf16(RN32(level[code] * s)).
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 64          # weights per first-level block
GROUP = 256         # first-level blocks per second-level group
# Offset of the outermost quantile: 1 - (1/32 + 1/30) / 2 = 929/960.
# The pages say only "16 levels placed at quantiles of a normal distribution";
# this constant is the paper's choice and is NOT fixed by the pages.
NF4_OFFSET = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
ZERO_CODE = 7


# ---------------------------------------------------------------------------
# Codebook
# ---------------------------------------------------------------------------

def normal_cdf(x: float) -> float:
    """Standard normal CDF, Phi(x) = erfc(-x / sqrt 2) / 2."""
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def normal_quantile(p: float) -> float:
    """Phi^{-1}(p) for 0.5 <= p < 1 by bisection on Phi, to full fp64
    resolution (the interval is halved until it stops shrinking)."""
    if not (0.5 <= p < 1.0):
        raise ValueError("p must lie in [0.5, 1)")
    lo, hi = 0.0, 10.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            break
        if normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    # choose the endpoint whose CDF is closer to p
    return lo if abs(normal_cdf(lo) - p) <= abs(normal_cdf(hi) - p) else hi


def nf4_levels_f64() -> np.ndarray:
    """The 16 NF4 levels in float64, ascending.

    Positive side: Phi^{-1} at 8 probabilities equally spaced from 1/2
    (exclusive) to the offset o (inclusive); negative side: minus Phi^{-1} at
    7 such probabilities; plus an exact zero; everything divided by
    Phi^{-1}(o) so that the extremes are exactly -1 and +1 (the block's absmax
    element must map to a +-1 level, "QLoRA, in depth", "The mechanism in
    brief": scales are block absmax values).
    """
    o = NF4_OFFSET
    top = normal_quantile(o)
    pos = [normal_quantile(0.5 + (o - 0.5) * j / 8.0) / top for j in range(1, 9)]
    neg = [-normal_quantile(0.5 + (o - 0.5) * j / 7.0) / top for j in range(1, 8)]
    pos[-1] = 1.0    # j = 8 is the offset itself: exactly Phi^{-1}(o) / Phi^{-1}(o)
    neg[-1] = -1.0
    levels = sorted(neg) + [0.0] + pos
    return np.array(levels, dtype=np.float64)


def nf4_levels() -> np.ndarray:
    """The NF4 levels rounded to float32 (the values the codec works with)."""
    return nf4_levels_f64().astype(np.float32)


# ---------------------------------------------------------------------------
# bf16 rounding by definition
# ---------------------------------------------------------------------------

def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even) and
    return the bf16 bit patterns as uint16.

    Written from the definition: the two bf16 neighbours of x are the value
    with the low 16 bits of the float32 pattern cleared (towards zero) and the
    next bf16 away from zero; pick the nearer, and on a tie the one whose last
    kept bit is 0. Distances are exact in float64. NaN/inf are not expected
    here (the codec rejects non-finite input).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    low = bits & 0xFFFF0000                     # truncated towards zero
    high = low + 0x10000                        # next bf16 away from zero
    lo_val = low.astype(np.uint32).view(np.float32).astype(np.float64)
    # high may step into the exponent: still the next representable magnitude
    hi_val = high.astype(np.uint32).view(np.float32).astype(np.float64)
    xv = x.astype(np.float64)
    d_lo = np.abs(xv - lo_val)
    d_hi = np.abs(hi_val - xv)
    lo_even = ((low >> 16) & 1) == 0
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~lo_even)
    out = np.where(take_hi, high, low) >> 16
    return out.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Quantisation
# ---------------------------------------------------------------------------

class NonFiniteInput(ValueError):
    """The weight matrix holds a NaN or an infinity."""


def block_absmax(W: np.ndarray) -> np.ndarray:
    """c1_b = max |w| over each block of 64 consecutive row-major elements."""
    flat = np.ascontiguousarray(W, dtype=np.float32).reshape(-1, BLOCK)
    return np.max(np.abs(flat), axis=1)


def encode_blocks(W: np.ndarray, c1: np.ndarray, levels: np.ndarray,
                  chunk: int = 1 << 14) -> np.ndarray:
    """Codes (uint8, one per weight, row-major) by nearest level.

    n = RN32(w / c1) (float64 division of two float32 values, then rounding to
    float32, is the correctly rounded float32 quotient); code = argmin over i
    of |n - level_i| with distances in float64 and ties going to the lower
    index (numpy's argmin returns the first minimum). Blocks with c1 == 0 get
    the zero code.
    """
    flat = np.ascontiguousarray(W, dtype=np.float32).reshape(-1, BLOCK)
    lv = levels.astype(np.float64)
    codes = np.empty(flat.shape, dtype=np.uint8)
    for s in range(0, flat.shape[0], chunk):
        w = flat[s:s + chunk].astype(np.float64)
        c = c1[s:s + chunk].astype(np.float64)
        nz = c > 0
        n = np.zeros_like(w)
        n[nz] = (w[nz] / c[nz, None]).astype(np.float32).astype(np.float64)
        dist = np.abs(n[:, :, None] - lv[None, None, :])
        code = np.argmin(dist, axis=2).astype(np.uint8)
        code[~nz] = ZERO_CODE
        codes[s:s + chunk] = code
    return codes.reshape(-1)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte, first element in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return ((c[:, 0] << 4) | c[:, 1]).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0x0F
    return out


def round_half_even_ratio(num: np.ndarray, den: np.ndarray) -> np.ndarray:
    """round-half-even(num / den) for non-negative float64 num, den > 0 whose
    products with small integers are exact in float64 (num = 255 * c1 with c1
    a float32; den = c2 a float32). Exact: the floor is corrected with exact
    products, the remainder is compared exactly with den / 2."""
    q = np.floor(num / den)
    q = np.where(q * den > num, q - 1, q)
    q = np.where((q + 1) * den <= num, q + 1, q)
    rem2 = 2.0 * (num - q * den)
    up = (rem2 > den) | ((rem2 == den) & (np.mod(q, 2) == 1))
    return np.where(up, q + 1, q)


def double_quantize(c1: np.ndarray):
    """Second-level quantisation of the block constants.

    Groups of 256 consecutive blocks (the last group may be short); per group
    c2 = max c1; q8_b = round-half-even(255 c1_b / c2) (0 when c2 == 0);
    stored second-level scale d = RN32(c2 / 255).
    Returns (scale8 uint8 [nb], scale2 float32 [ng]).
    """
    c1 = np.asarray(c1, dtype=np.float32)
    nb = c1.size
    ng = -(-nb // GROUP)
    pad = np.zeros(ng * GROUP, dtype=np.float32)
    pad[:nb] = c1
    c2 = pad.reshape(ng, GROUP).max(axis=1)                       # float32, exact
    c2_per_block = np.repeat(c2, GROUP)[:nb].astype(np.float64)
    num = 255.0 * c1.astype(np.float64)                           # exact
    q8 = np.zeros(nb, dtype=np.float64)
    nz = c2_per_block > 0
    q8[nz] = round_half_even_ratio(num[nz], c2_per_block[nz])
    d = (c2.astype(np.float64) / 255.0).astype(np.float32)
    return q8.astype(np.uint8), d


def quantize(W: np.ndarray):
    """Full NF4 + double-quant encoding of a float32 matrix W[N, K], K % 64 == 0.

    Returns (codes_packed uint8 [N*K/2], scale8 uint8 [N*K/64],
    scale2 float32 [ceil(N*K/64/256)]). Raises NonFiniteInput on NaN/inf.
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % BLOCK != 0:
        raise ValueError("W must be [N, K] with K % 64 == 0")
    if not np.all(np.isfinite(W)):
        raise NonFiniteInput("non-finite weight")
    levels = nf4_levels()
    c1 = block_absmax(W)
    codes = encode_blocks(W, c1, levels)
    scale8, scale2 = double_quantize(c1)
    return pack_codes(codes), scale8, scale2


# ---------------------------------------------------------------------------
# Dequantisation
# ---------------------------------------------------------------------------

def block_scales(scale8: np.ndarray, scale2: np.ndarray) -> np.ndarray:
    """s_b = RN32(q8_b * d_g) as float32 (the product is exact in float64)."""
    q8 = np.asarray(scale8, dtype=np.uint8).astype(np.float64)
    g = np.arange(q8.size) // GROUP
    d = np.asarray(scale2, dtype=np.float32).astype(np.float64)[g]
    return (q8 * d).astype(np.float32)


def dequantize_bits(packed: np.ndarray, scale8: np.ndarray, scale2: np.ndarray,
                    rows: int, cols: int) -> np.ndarray:
    """bf16 bit patterns (uint16 [rows, cols]) of w' = RN_bf16(RN32(level * s))."""
    levels = nf4_levels().astype(np.float64)
    codes = unpack_codes(packed).reshape(-1, BLOCK)
    s = block_scales(scale8, scale2).astype(np.float64)
    prod = (levels[codes] * s[:, None]).astype(np.float32)       # exact product, one rounding
    return bf16_round_bits(prod.reshape(-1)).reshape(rows, cols)


def dequantize(packed, scale8, scale2, rows: int, cols: int) -> np.ndarray:
    """Dequantised weight as float64 values of the bf16 results."""
    return bf16_bits_to_f64(dequantize_bits(packed, scale8, scale2, rows, cols))


# ---------------------------------------------------------------------------
# Parts of a large matrix (for checks at full size that the oracle cannot
# afford to encode whole). The block constants and the second-level groups
# are computed over the whole matrix (a group of 256 blocks may straddle
# rows); only the requested weights are encoded. The result equals the same
# rows or columns of dequantize(*quantize(W)).
# ---------------------------------------------------------------------------

def _scales_all(W: np.ndarray):
    W = np.ascontiguousarray(W, dtype=np.float32)
    c1 = block_absmax(W)
    scale8, scale2 = double_quantize(c1)
    return W, c1, block_scales(scale8, scale2).astype(np.float64), scale8, scale2


def _dequant_blocks(Wb: np.ndarray, c1b: np.ndarray, sb: np.ndarray) -> np.ndarray:
    """Blocks [nb, 64] of weights -> float64 values of their bf16 dequantisation."""
    codes = encode_blocks(Wb, c1b, nf4_levels()).reshape(-1, BLOCK)
    prod = (nf4_levels().astype(np.float64)[codes] * sb[:, None]).astype(np.float32)
    return bf16_bits_to_f64(bf16_round_bits(prod.reshape(-1))).reshape(-1, BLOCK)


def dequantize_rows(W: np.ndarray, rows) -> np.ndarray:
    """Rows `rows` of the dequantised W (float64 [len(rows), K])."""
    W, c1, s, _, _ = _scales_all(W)
    N, K = W.shape
    kb = K // BLOCK
    rows = np.asarray(rows)
    blocks = (rows[:, None] * kb + np.arange(kb)[None, :]).reshape(-1)
    out = _dequant_blocks(W[rows].reshape(-1, BLOCK), c1[blocks], s[blocks])
    return out.reshape(len(rows), K)


def dequantize_cols(W: np.ndarray, cols) -> np.ndarray:
    """Columns `cols` of the dequantised W (float64 [N, len(cols)])."""
    W, c1, s, _, _ = _scales_all(W)
    N, K = W.shape
    kb = K // BLOCK
    cols = np.asarray(cols)
    cblocks = np.unique(cols // BLOCK)
    blocks = (np.arange(N)[:, None] * kb + cblocks[None, :]).reshape(-1)
    Wb = W.reshape(N, kb, BLOCK)[:, cblocks, :].reshape(-1, BLOCK)
    vals = _dequant_blocks(Wb, c1[blocks], s[blocks]).reshape(N, len(cblocks), BLOCK)
    where = np.searchsorted(cblocks, cols // BLOCK)
    return vals[:, where, cols % BLOCK]


def quantize_rows(W: np.ndarray, rows):
    """(packed codes [len(rows), K/2], scale8 of those rows' blocks [len(rows), K/64],
    scale2 of the whole matrix): the stored format restricted to `rows`."""
    W, c1, _, scale8, scale2 = _scales_all(W)
    N, K = W.shape
    kb = K // BLOCK
    rows = np.asarray(rows)
    blocks = (rows[:, None] * kb + np.arange(kb)[None, :]).reshape(-1)
    codes = encode_blocks(W[rows].reshape(-1, BLOCK), c1[blocks], nf4_levels())
    return pack_codes(codes).reshape(len(rows), K // 2), scale8[blocks].reshape(len(rows), kb), scale2
