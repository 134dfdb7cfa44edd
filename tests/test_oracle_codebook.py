"""Pins of the oracle's NF4 codebook.

The pages fix: 16 levels placed at quantiles of a normal distribution
("QLoRA, in depth", "The mechanism in brief"; "QLoRA and Fine-Tuning on One
Consumer GPU", "NF4 and double quantisation"), the block's absmax element maps
to a +-1 level (the block constant is the absmax), and zero must be exactly
representable. The offset of the outermost quantile is NOT fixed by the pages
(parity unpinned for that one constant); everything around it is pinned here.
"""

import numpy as np
import pytest
import scipy.special
import scipy.stats

from oracle import nf4


def test_shape_order_and_exact_points():
    L = nf4.nf4_levels()
    assert L.dtype == np.float32 and L.shape == (16,)
    assert np.all(np.diff(L.astype(np.float64)) > 0), "levels strictly increasing"
    assert L[0] == np.float32(-1.0) and L[15] == np.float32(1.0)
    assert L[7] == np.float32(0.0) and not np.signbit(L[7])
    assert int(np.sum(L < 0)) == 7 and int(np.sum(L > 0)) == 8


def test_equal_probability_spacing():
    """Phi(level * Phi^{-1}(o)) must step by the same probability on each side:
    (o - 1/2)/8 on the positive side and (o - 1/2)/7 on the negative side."""
    L = nf4.nf4_levels_f64()
    o = nf4.NF4_OFFSET
    z = scipy.stats.norm.ppf(o)
    p = scipy.stats.norm.cdf(L * z)
    pos = p[7:] - 0.5            # 0, then 8 positive levels
    neg = 0.5 - p[:8][::-1]      # 0, then 7 negative levels (nearest zero first)
    np.testing.assert_allclose(np.diff(pos), (o - 0.5) / 8, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(np.diff(neg), (o - 0.5) / 7, rtol=1e-12, atol=1e-15)


def test_matches_library_quantile_function_bitwise():
    """Our bisection quantile function against scipy's ndtri: the float32
    levels must agree bit for bit."""
    o = nf4.NF4_OFFSET
    top = scipy.special.ndtri(o)
    pos = [scipy.special.ndtri(0.5 + (o - 0.5) * j / 8) / top for j in range(1, 9)]
    neg = [-scipy.special.ndtri(0.5 + (o - 0.5) * j / 7) / top for j in range(1, 8)]
    ref = np.array(sorted(neg) + [0.0] + pos).astype(np.float32)
    assert np.array_equal(ref.view(np.uint32), nf4.nf4_levels().view(np.uint32))


@pytest.mark.parametrize("p", [0.5, 0.5 + 1e-9, 0.6, 0.84134474606854293, 0.9677083333, 0.999])
def test_quantile_function(p):
    assert nf4.normal_quantile(p) == pytest.approx(scipy.special.ndtri(p), rel=1e-14, abs=1e-15)


def test_known_first_levels():
    """The levels nearest zero of the published NF4 table are about 0.0796 and
    -0.0911; a wrong offset or step count moves them well beyond 1e-4."""
    L = nf4.nf4_levels_f64()
    assert L[8] == pytest.approx(0.0796, abs=1e-4)
    assert L[6] == pytest.approx(-0.0911, abs=1e-4)


def test_nf4_beats_uniform_int4_on_normal_blocks():
    """'Why NF4 and not plain int4?' (mantramindai.in, Follow-up questions):
    on normally distributed weights NF4's error is lower than evenly spaced
    int4 levels at the same 4 bits. Both use per-block absmax scaling."""
    rng = np.random.Generator(np.random.PCG64(123))
    w = rng.standard_normal((4096, 64))
    c1 = np.abs(w).max(axis=1, keepdims=True)
    n = w / c1
    L = nf4.nf4_levels_f64()
    nf4_q = L[np.argmin(np.abs(n[..., None] - L), axis=-1)] * c1
    int4_levels = np.arange(-7, 8) / 7.0           # symmetric absmax int4
    int4_q = int4_levels[np.argmin(np.abs(n[..., None] - int4_levels), axis=-1)] * c1
    rmse_nf4 = np.sqrt(np.mean((nf4_q - w) ** 2))
    rmse_int4 = np.sqrt(np.mean((int4_q - w) ** 2))
    assert rmse_nf4 < rmse_int4
