"""Pins of the int4 comparison codec: its levels, brute-force encoding on
tiny blocks in exact rationals, the absmax element at +-1, zero at code 8,
and the error ordering the pages state (NF4 below int4 on normal weights)."""

from fractions import Fraction

import numpy as np

from oracle import codebooks, nf4
from bit_nf4_quantized_dequant_b200 import inputs


def test_int4_levels():
    L = codebooks.int4_levels()
    assert L.dtype == np.float32 and len(L) == 16
    assert np.all(np.diff(L) > 0)
    assert L[8] == 0.0 and L[1] == -1.0 and L[15] == 1.0
    for k in range(16):
        assert abs(float(L[k]) - (k - 8) / 7) <= 2.0 ** -24   # float32 rounding of (k-8)/7


def test_encode_brute_force_tiny_blocks():
    g = inputs.rng(600)
    L = [Fraction(float(v)) for v in codebooks.int4_levels()]
    for trial in range(20):
        w = (g.standard_normal(64) * 0.03).astype(np.float32)
        if trial == 3:
            w[10] = 0.0
        packed, s8, s2 = codebooks.quantize_int4(w.reshape(1, 64))
        codes = nf4.unpack_codes(packed)
        c1 = Fraction(float(np.max(np.abs(w))))
        for i, wi in enumerate(w):
            n = Fraction(float(np.float32(Fraction(float(wi)) / c1)))   # RN32 of the exact quotient
            d = [abs(n - l) for l in L]
            best = min(range(16), key=lambda k: (d[k], k))               # ties to the lower index
            assert codes[i] == best
        assert codes[int(np.argmax(np.abs(w)))] in (1, 15)


def test_zero_block_and_zero_weights():
    W = np.zeros((1, 128), dtype=np.float32)
    W[0, 64:] = np.linspace(-0.1, 0.1, 64, dtype=np.float32)
    W[0, 100] = 0.0
    codes = nf4.unpack_codes(codebooks.quantize_int4(W)[0])
    assert np.all(codes[:64] == 8) and codes[100] == 8


def test_nf4_error_below_int4_on_normal_weights():
    """The pages' claim, with both codecs in the same stored format."""
    W = (inputs.rng(601).standard_normal((64, 4096)) * 0.02).astype(np.float32)
    e_nf4 = nf4.dequantize(*nf4.quantize(W), *W.shape) - W
    p, s8, s2 = codebooks.quantize_int4(W)
    e_int4 = nf4.bf16_bits_to_f64(codebooks.dequantize_int4_bits(p, s8, s2, *W.shape)) - W
    assert np.sqrt(np.mean(e_nf4 ** 2)) < 0.9 * np.sqrt(np.mean(e_int4 ** 2))
