"""Pins of the comparison format's oracle (oracle/dq_fp8.py): NF4 codes with
an 8-bit-float, mean-centred second level. Each check rests on something
other than the oracle itself: the E4M3 format's definition and a library
cast, exact sums, closed-form error bounds of the 8-bit float, the storage
arithmetic the pages quote."""

import math

import numpy as np
import pytest

from oracle import dq_fp8 as odq, nf4 as onf4


def test_e4m3_table_is_the_format():
    """254 finite values and two NaNs; largest 448 (1.75 * 2^8), smallest
    positive 2^-9 (subnormal), smallest normal 2^-6; codes 0..0x7E increase."""
    t = odq.e4m3_table()
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.sum(np.isfinite(t)) == 254
    pos = t[:127]
    assert np.all(np.diff(pos) > 0)
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9 and pos[8] == 2.0 ** -6
    assert np.array_equal(t[0x80:0xFF], -pos)


def test_e4m3_encode_matches_library_cast():
    """Round to nearest, ties to even, for magnitudes up to 448: the same codes
    as torch's float8_e4m3fn cast (a library routine), on random values, on
    every exact midpoint between neighbours and on the values themselves."""
    torch = pytest.importorskip("torch")
    pos = odq.e4m3_table()[:127]
    mids = 0.5 * (pos[1:] + pos[:-1])
    g = np.random.default_rng(11)
    rnd = np.concatenate([g.uniform(-448, 448, 4000), g.standard_normal(4000) * 0.01,
                          g.standard_normal(2000) * 2.0 ** -8])
    x = np.concatenate([pos, -pos, mids, -mids, rnd]).astype(np.float32)
    ours = odq.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e6, -500.0, 3.4e38], dtype=np.float32)
    assert list(odq.e4m3_encode(x)) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E]


def test_group_mean_within_one_ulp_of_exact_mean():
    """mu is the rounded block-order sum divided by n: within one float32 ulp
    of the exact mean (math.fsum is exact)."""
    g = np.random.default_rng(12)
    for scale in (1e-3, 1.0, 1e20):
        c1 = (np.abs(g.standard_normal(256)) * scale).astype(np.float32)
        mu = odq.group_mean(c1)
        exact = math.fsum(float(v) for v in c1) / 256.0
        assert abs(float(mu) - exact) <= float(np.spacing(np.float32(exact)))


def test_constant_group_decodes_exactly():
    """All constants equal: nothing to centre, d = 0, every code +0 and the
    decoded constant is the mean, i.e. exact."""
    c1 = np.full(256, 0.0371, dtype=np.float32)
    q, s2 = odq.double_quantize_fp8(c1)
    assert not q.any() and s2[0, 0] == 0 and s2[0, 1] == c1[0]
    assert np.array_equal(odq.block_scales_fp8(q, s2), c1)


@pytest.mark.parametrize("kind", ["spread", "clustered", "outlier", "ragged"])
def test_decoded_constants_within_e4m3_bound(kind):
    """|s_b - c1_b| <= 2^-4 |c1_b - mu| + 2^-10 d + a few float32 ulps: the
    8-bit float keeps 3 mantissa bits (half-ulp relative error 2^-4 for
    normals, 2^-10 absolute below 2^-6, in units of d). A clustered group
    (constants 1 +- 1 %) fails this bound if the centring is dropped."""
    g = np.random.default_rng({"spread": 1, "clustered": 2, "outlier": 3, "ragged": 4}[kind])
    n = 3 * 256 if kind != "ragged" else 2 * 256 + 77
    if kind == "clustered":
        c1 = 1.0 + 0.01 * g.standard_normal(n)
    elif kind == "outlier":
        c1 = np.abs(g.standard_normal(n)) * 0.05
        c1[::97] *= 8.0
    else:
        c1 = np.abs(g.standard_normal(n)) * 0.05
    c1 = c1.astype(np.float32)
    q, s2 = odq.double_quantize_fp8(c1)
    s = odq.block_scales_fp8(q, s2).astype(np.float64)
    grp = np.arange(n) // 256
    mu_true = np.array([np.mean(c1[grp == gi].astype(np.float64)) for gi in range(grp.max() + 1)])[grp]
    mu, d = s2[grp, 1].astype(np.float64), s2[grp, 0].astype(np.float64)
    assert np.all(np.abs(mu - mu_true) <= np.spacing(np.float32(np.max(c1))))
    cen = np.abs(c1.astype(np.float64) - mu_true)
    ulp = np.spacing(np.float32(np.max(c1))).astype(np.float64)
    bound = 2.0 ** -4 * cen + 2.0 ** -10 * d + 4 * ulp
    assert np.all(np.abs(s - c1) <= bound)
    # the extreme block of each group maps to +-448 d
    for gi in range(grp.max() + 1):
        sl = grp == gi
        k = np.argmax(np.abs(c1[sl].astype(np.float64) - mu[sl]))
        assert odq.e4m3_decode(q[sl][k:k + 1])[0] in (448.0, -448.0)


def test_storage_saving_is_the_quoted_037_bits():
    """4 + 8/64 + 64/16384 bits per weight; against 4.5 without double
    quantisation that saves 0.371 bits, the pages' "about 0.37"."""
    assert odq.BITS_PER_WEIGHT == 4.12890625
    assert abs((4.5 - odq.BITS_PER_WEIGHT) - 0.37) < 0.005


def test_codes_are_the_nf4_codes_and_dequant_uses_decoded_scales():
    """Only the second level differs from the NF4 format: the packed codes are
    identical, and with the decoded constants in place of the linear ones the
    dequantised weight follows the same rule, element for element."""
    g = np.random.default_rng(21)
    W = (g.standard_normal((48, 320)) * 0.02).astype(np.float32)
    W[3, :64] = 0.0
    p8, q8, s28 = odq.quantize_fp8dq(W)
    p, _, _ = onf4.quantize(W)
    assert np.array_equal(p8, p)
    bits = odq.dequantize_fp8dq_bits(p8, q8, s28, 48, 320)
    s = odq.block_scales_fp8(q8, s28).astype(np.float64)
    lv = onf4.nf4_levels().astype(np.float64)
    codes = onf4.unpack_codes(p8).reshape(-1, 64)
    for b in (0, 5, 17, 239):
        want = onf4.bf16_round_bits((lv[codes[b]] * s[b]).astype(np.float32))
        assert np.array_equal(bits.reshape(-1, 64)[b], want)
    # the all-zero block dequantises to zeros of either sign
    assert np.all((bits[3, :64] & 0x7FFF) == 0)
