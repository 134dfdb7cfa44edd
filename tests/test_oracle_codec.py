"""Pins of the oracle's NF4 codec: brute force in exact rational arithmetic on
tiny blocks, crafted ties, the invariants the pages state, and bounds.

Sources: "QLoRA, in depth", "The mechanism in brief" (blocks of 64, per-block
absmax scale, 8-bit double quantisation with one 32-bit scale per 256 blocks,
dequantisation to bf16); "QLoRA and Fine-Tuning on One Consumer GPU", "Where
24 GB goes" (0.5 byte per weight).
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import nf4
from bit_nf4_quantized_dequant_b200 import inputs


def _f32(x) -> np.float32:
    return np.float32(x)


def brute_force_codes(block: np.ndarray, levels: np.ndarray):
    """Exact: c1 = max|w|; n = float32 rounding of the exact quotient; code =
    the first index attaining the minimal exact distance."""
    c1 = max(abs(Fraction(float(w))) for w in block)
    codes = []
    for w in block:
        if c1 == 0:
            codes.append(7)
            continue
        q = Fraction(float(w)) / c1
        n = Fraction(float(_f32(float(q))))        # int/int division is correctly rounded
        best, best_d = None, None
        for i, lv in enumerate(levels):
            d = abs(n - Fraction(float(lv)))
            if best_d is None or d < best_d:
                best, best_d = i, d
        codes.append(best)
    return c1, codes


def test_encode_matches_brute_force_on_tiny_blocks():
    L = nf4.nf4_levels()
    rng = np.random.Generator(np.random.PCG64(7))
    W = (rng.standard_normal((6, 128)) * 0.02).astype(np.float32)
    W[1, 5] = 0.0
    W[2, 64:128] = -W[2, 64:128]
    W[3, :64] = 0.0                                   # all-zero block
    W[4, 64:] = np.float32(1e-40)                     # subnormal block
    c1 = nf4.block_absmax(W)
    codes = nf4.encode_blocks(W, c1, L).reshape(-1, 64)
    for b, block in enumerate(W.reshape(-1, 64)):
        ref_c1, ref_codes = brute_force_codes(block, L)
        assert Fraction(float(c1[b])) == ref_c1
        assert codes[b].tolist() == ref_codes


def test_midpoint_ties_go_to_lower_index():
    L = nf4.nf4_levels().astype(np.float64)
    ties = 0
    for i in range(15):
        mid = (L[i] + L[i + 1]) / 2.0                  # exact in float64
        m32 = np.float32(mid)
        block = np.zeros(64, dtype=np.float32)
        block[0] = 1.0                                  # absmax 1 -> n = w exactly
        block[1] = m32
        block[2] = np.nextafter(m32, np.float32(-2))
        block[3] = np.nextafter(m32, np.float32(2))
        c = nf4.encode_blocks(block[None, :], nf4.block_absmax(block[None, :]), nf4.nf4_levels())
        if float(m32) == mid:
            ties += 1
            assert c[1] == i, f"exact tie between {i} and {i+1} must pick {i}"
        assert c[2] == i and c[3] == i + 1 if float(m32) == mid else True
        _, ref = brute_force_codes(block[:4], nf4.nf4_levels())
        assert c[:4].tolist() == ref
    assert ties >= 1, "at least one midpoint is a float32 value (exact tie exercised)"


def test_absmax_element_maps_to_extreme_level():
    W = inputs.weight_f32(64, 256, outliers=True)
    c1 = nf4.block_absmax(W)
    codes = nf4.encode_blocks(W, c1, nf4.nf4_levels()).reshape(-1, 64)
    blocks = W.reshape(-1, 64)
    arg = np.argmax(np.abs(blocks), axis=1)
    picked = codes[np.arange(codes.shape[0]), arg]
    sign = blocks[np.arange(blocks.shape[0]), arg] > 0
    assert np.all(picked[sign] == 15) and np.all(picked[~sign] == 0)


def test_zero_is_exact_and_all_zero_block():
    W = np.zeros((2, 128), dtype=np.float32)
    W[0, 64:] = inputs.normal_f32(3, 64, 0.02)
    W[0, 70] = 0.0
    W[0, 71] = -0.0
    packed, s8, s2 = nf4.quantize(W)
    codes = nf4.unpack_codes(packed).reshape(2, 128)
    assert np.all(codes[0, :64] == 7) and np.all(codes[1] == 7)
    assert codes[0, 70] == 7 and codes[0, 71] == 7
    assert s8[0] == 0 and s8[2] == 0 and s8[3] == 0
    bits = nf4.dequantize_bits(packed, s8, s2, 2, 128)
    assert np.all(bits[0, :64] == 0) and bits[0, 70] == 0 and bits[0, 71] == 0
    assert np.all(bits[1] == 0)


def test_packing_high_nibble_first():
    codes = np.array([1, 2, 15, 0, 7, 9], dtype=np.uint8)
    p = nf4.pack_codes(codes)
    assert p.tolist() == [0x12, 0xF0, 0x79]
    assert nf4.unpack_codes(p).tolist() == codes.tolist()


def brute_force_q8(c1: float, c2: float) -> int:
    if c2 == 0:
        return 0
    t = Fraction(255) * Fraction(c1) / Fraction(c2)
    best = min(range(256), key=lambda q: (abs(t - q), q % 2))   # nearest, ties to even
    return best


def test_double_quant_matches_brute_force():
    rng = np.random.Generator(np.random.PCG64(11))
    c1 = np.abs(rng.standard_normal(700) * 0.05).astype(np.float32)   # 3 groups, last one short
    c1[5] = 0.0
    # craft exact half-way ratios: c2 = 255 * 2^-4 makes 255 c1 / c2 = 16 c1
    c1[256:512] = np.float32(0.001)
    c1[300] = np.float32(255.0 / 16.0)                 # group max
    c1[301] = np.float32(2.5 / 16.0)                   # ratio 2.5 -> 2
    c1[302] = np.float32(3.5 / 16.0)                   # ratio 3.5 -> 4
    s8, s2 = nf4.double_quantize(c1)
    assert s8.shape == (700,) and s2.shape == (3,)
    for g in range(3):
        grp = c1[g * 256:(g + 1) * 256]
        c2 = float(grp.max())
        assert s2[g] == np.float32(Fraction(c2) / 255)    # RN32 of the exact quotient
        for j, c in enumerate(grp):
            assert s8[g * 256 + j] == brute_force_q8(float(c), c2)
    assert s8[301] == 2 and s8[302] == 4


def test_group_max_scale_and_monotonicity():
    W = inputs.weight_f32(256, 1024, outliers=True)
    c1 = nf4.block_absmax(W)
    s8, s2 = nf4.double_quantize(c1)
    s = nf4.block_scales(s8, s2)
    for g in range(s2.size):
        sl = slice(g * 256, (g + 1) * 256)
        k = np.argmax(c1[sl])
        assert s8[sl][k] == 255
        c2 = c1[sl][k]
        assert abs(int(np.float32(s[sl][k]).view(np.int32)) - int(np.float32(c2).view(np.int32))) <= 2
        order = np.argsort(c1[sl], kind="stable")
        assert np.all(np.diff(s[sl][order].astype(np.float64)) >= 0)


def test_bf16_rounding_matches_library_cast():
    rng = np.random.Generator(np.random.PCG64(5))
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-40, 30, 100000)).astype(np.float32)
    # exact ties: low 16 bits == 0x8000, both parities of the kept part
    ties = (rng.integers(0, 2**31, 1000, dtype=np.uint32) & 0xFFFF0000) | 0x8000
    x = np.concatenate([x, ties.view(np.float32), np.array([1e-45, -1e-45, 3e-39], np.float32)])
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(nf4.bf16_round_bits(x), ref)


def test_dequant_error_bound():
    """|w' - w| <= (half the widest level gap) c1 + |s - c1| + bf16 rounding."""
    W = inputs.weight_f32(128, 512, outliers=True)
    packed, s8, s2 = nf4.quantize(W)
    Wd = nf4.dequantize(packed, s8, s2, 128, 512).reshape(-1, 64)
    c1 = nf4.block_absmax(W).astype(np.float64)
    s = nf4.block_scales(s8, s2).astype(np.float64)
    half_gap = np.max(np.diff(nf4.nf4_levels_f64())) / 2
    bound = half_gap * c1 + np.abs(s - c1) + 2.0 ** -8 * np.abs(Wd).max(axis=1) + 1e-30
    err = np.abs(Wd - W.reshape(-1, 64).astype(np.float64)).max(axis=1)
    assert np.all(err <= bound)
    # the 8-bit constant is within half a step of the true absmax
    d = np.repeat(s2.astype(np.float64), 256)[: c1.size]
    assert np.all(np.abs(s - c1) <= 0.5 * d + 2 ** -23 * c1 + 1e-30)


def test_dequant_special_values():
    W = np.zeros((1, 64), dtype=np.float32)
    W[0, 0] = 0.75
    W[0, 1] = -0.75
    packed, s8, s2 = nf4.quantize(W)
    bits = nf4.dequantize_bits(packed, s8, s2, 1, 64)
    assert s8[0] == 255
    s = np.float32(np.float64(255) * np.float64(s2[0]))
    assert nf4.bf16_bits_to_f64(bits[0, :2]).tolist() == [float(torch.tensor(float(s)).bfloat16()),
                                                          float(torch.tensor(-float(s)).bfloat16())]
    assert np.all(bits[0, 2:] == 0)


def test_storage_sizes_of_quantize_output():
    W = inputs.weight_f32(96, 1024 + 64)
    packed, s8, s2 = nf4.quantize(W)
    n = W.size
    assert packed.size == n // 2 and s8.size == n // 64 and s2.size == -(-(n // 64) // 256)


def test_non_finite_rejected():
    W = np.zeros((1, 64), dtype=np.float32)
    W[0, 3] = np.inf
    with pytest.raises(nf4.NonFiniteInput):
        nf4.quantize(W)
    W[0, 3] = np.nan
    with pytest.raises(nf4.NonFiniteInput):
        nf4.quantize(W)


def test_planted_tie_rule_is_caught(monkeypatch):
    """A planted mistake in the oracle (ties to the upper index) must fail the
    brute-force pin: the pins are sharp enough to see it."""
    real = nf4.encode_blocks

    def upper_ties(W, c1, levels, chunk=1 << 14):
        flat = np.ascontiguousarray(W, dtype=np.float32).reshape(-1, 64)
        n = (flat.astype(np.float64) / c1[:, None]).astype(np.float32).astype(np.float64)
        d = np.abs(n[..., None] - levels.astype(np.float64))
        return (15 - np.argmin(d[..., ::-1], axis=-1)).astype(np.uint8).reshape(-1)

    monkeypatch.setattr(nf4, "encode_blocks", upper_ties)
    with pytest.raises(AssertionError):
        test_midpoint_ties_go_to_lower_index()
    monkeypatch.setattr(nf4, "encode_blocks", real)


@pytest.mark.parametrize("N,K", [(12, 11008), (12, 704), (33, 4096)])
def test_row_and_column_restrictions_equal_the_whole(N, K):
    """dequantize_rows / dequantize_cols / quantize_rows (used for checks at
    full size) are the whole-matrix encoding restricted to rows or columns,
    including second-level groups that straddle rows (K = 704 and 4096 give
    11 and 64 blocks per row)."""
    g = inputs.rng(31)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[3, 5] = 0.0
    W[7, 64:128] = 0.0
    packed, s8, s2 = nf4.quantize(W)
    full = nf4.dequantize(packed, s8, s2, N, K)
    rows = np.array([0, 3, 7, N - 1])
    cols = np.array([0, 1, 63, 64, 65, K - 1, 130 if K > 130 else 2])
    np.testing.assert_array_equal(nf4.dequantize_rows(W, rows), full[rows])
    np.testing.assert_array_equal(nf4.dequantize_cols(W, cols), full[:, cols])
    pr, s8r, s2r = nf4.quantize_rows(W, rows)
    np.testing.assert_array_equal(pr, packed.reshape(N, K // 2)[rows])
    np.testing.assert_array_equal(s8r, s8.reshape(N, K // 64)[rows])
    np.testing.assert_array_equal(s2r, s2)


def _midpoint_scales(levels: np.ndarray, per_level: int, rng) -> list:
    """Float32 scales s for which RN32(level * s) is exactly halfway between
    two bf16 values (low 16 bits 0x8000) while the exact product is not: the
    products where rounding to float32 first and then to bf16 differs from
    one rounding of the exact product whenever the exact product lies on the
    side of the odd bf16 neighbour. Levels 0 and +-1 have exact products and
    are skipped."""
    out = []
    for i, L in enumerate(levels.astype(np.float64)):
        if L == 0.0 or abs(L) == 1.0:
            continue
        found = 0
        for _ in range(50 * per_level):
            if found == per_level:
                break
            t_bits = (int(rng.integers(0x3C000000, 0x3F000000)) & 0xFFFF0000) | 0x8000
            t = float(np.array([t_bits], np.uint32).view(np.float32)[0]) * (1.0 if L > 0 else -1.0)
            s0 = np.float32(t / L)
            for k in range(-3, 4):
                s = s0
                for _ in range(abs(k)):
                    s = np.nextafter(s, np.float32(np.inf) if k > 0 else np.float32(-np.inf))
                exact = Fraction(float(L)) * Fraction(float(s))
                if float(np.float32(float(exact))) == t and exact != Fraction(t):
                    out.append((i, np.float32(s)))
                    found += 1
                    break
    return out


def _bf16_single_rounding(x: Fraction) -> int:
    """bf16 bits of one round-to-nearest-even rounding of an exact value
    (finite, within the normal float32 range or zero)."""
    if x == 0:
        return 0
    sign = 0x8000 if x < 0 else 0
    m = abs(x)
    b = int(np.array([np.float32(float(m))], np.float32).view(np.uint32)[0]) & 0xFFFF0000
    cands = []
    for hi in (b - 0x10000, b, b + 0x10000):
        if hi < 0:
            continue
        v = Fraction(float(np.array([hi], np.uint32).view(np.float32)[0]))
        cands.append((abs(v - m), (hi >> 16) & 1, hi >> 16))
    cands.sort()
    if cands[0][0] == cands[1][0]:                # exact tie: the even one
        return (min(cands[:2], key=lambda c: c[1])[2] & 0x7FFF) | sign
    return (cands[0][2] & 0x7FFF) | sign


def _rounding_case():
    """Blocks that each hold all 16 codes four times, with block scales
    s = RN32(q8 * d) that vary per block: 512 groups of random scales, then one
    group per crafted midpoint scale (its first block has q8 = 1, so s = d).
    Returns the codec inputs, torch's float32-then-bf16 bits and the crafted
    (block, level) pairs with their exact single-rounding bits."""
    rng = np.random.Generator(np.random.PCG64(11))
    levels = nf4.nf4_levels()
    crafted = _midpoint_scales(levels, 12, rng)
    n_groups = 512 + len(crafted)
    codes = np.tile(np.arange(16, dtype=np.uint8), 4)
    nb = n_groups * 256
    q8 = rng.integers(1, 256, nb).astype(np.uint8)
    d = (rng.uniform(0.5, 2.0, n_groups) * 10.0 ** rng.integers(-6, 1, n_groups)).astype(np.float32)
    for g, (_, s) in enumerate(crafted):
        q8[(512 + g) * 256] = 1
        d[512 + g] = s
    packed = nf4.pack_codes(np.tile(codes, nb))
    s_t = torch.from_numpy(q8.astype(np.float32)) * torch.from_numpy(np.repeat(d, 256))   # float32 products
    w_t = torch.from_numpy(levels)[torch.from_numpy(codes.astype(np.int64))][None, :] * s_t[:, None]
    ref = w_t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    single = [((512 + g) * 256, i, _bf16_single_rounding(Fraction(float(levels[i])) * Fraction(float(s))))
              for g, (i, s) in enumerate(crafted)]
    return packed, q8, d, nb, ref, single


def test_dequant_rounding_matches_float32_then_bf16_in_torch():
    """The dequantiser's rounding reading, w' = RN_bf16(RN32(level * s)) with
    s = RN32(q8 * d) ("QLoRA, in depth", "The mechanism in brief": the weight
    is dequantised to the bf16 compute dtype through the float32 block
    constant), against torch's own float32 multiplies and bf16 cast: all 16
    levels times about 1.3e5 float32 scales, plus crafted scales whose float32
    product sits exactly on a bf16 midpoint while the exact product does not.
    One rounding of the exact product straight to bf16 (the neighbouring
    reading) gives other bits on part of the crafted cases."""
    packed, q8, d, nb, ref, single = _rounding_case()
    bits = nf4.dequantize_bits(packed, q8, d, nb, 64).reshape(nb, 64)
    assert np.array_equal(bits, ref)
    differ = sum(1 for b, i, sb in single if sb != int(bits[b, i]))
    assert len(single) >= 150 and differ >= len(single) // 4


def test_planted_single_rounding_is_caught(monkeypatch):
    """A dequantiser that rounds the exact product once, straight to bf16,
    passes every bound and special value but fails the pin above."""
    def one_rounding(packed, scale8, scale2, rows, cols):
        levels = nf4.nf4_levels().astype(np.float64)
        codes = nf4.unpack_codes(packed).reshape(-1, nf4.BLOCK)
        s = nf4.block_scales(scale8, scale2).astype(np.float64)
        v = (levels[codes] * s[:, None]).reshape(-1)        # exact in float64
        a = np.abs(v)
        ulp = np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7)
        lo = np.floor(a / ulp)                              # exact: scaling by powers of two
        frac = a / ulp - lo
        up = (frac > 0.5) | ((frac == 0.5) & (lo % 2 == 1))
        r = np.where(a > 0, (lo + up) * ulp, 0.0) * np.sign(v)
        return nf4.bf16_round_bits(r.astype(np.float32)).reshape(rows, cols)   # r is already on the bf16 grid

    packed, q8, d, nb, ref, single = _rounding_case()
    # the crafted groups alone keep the planted version fast
    sel = slice(512 * 256, nb)
    sub = nf4.pack_codes(nf4.unpack_codes(packed).reshape(nb, 64)[sel].reshape(-1))
    monkeypatch.setattr(nf4, "dequantize_bits", one_rounding)
    bits = nf4.dequantize_bits(sub, q8[sel], d[512:], nb - 512 * 256, 64)
    assert not np.array_equal(bits, ref[sel])
