"""GPU parity of the NF4 codec against the oracle: packed codes, 8-bit block
scales, fp32 second-level scales and the dequantised bf16 weight must be
bit-exact ("QLoRA, in depth", "The mechanism in brief")."""

import numpy as np
import pytest

from oracle import nf4 as onf4
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import bf16_dev_bits

pytestmark = pytest.mark.gpu

SHAPES = [
    (1024, 1024, False),    # single linear 1024x1024
    (4096, 4096, True),     # attention projection with 0.1% x8 outliers
    (48, 192, False),       # 144 blocks: one short group
    (16, 64, False),        # one block per row
    (272, 320, True),       # ragged: 1360 blocks = 5 groups + 80
    (11008, 128, False),    # tall
]


def _quantize_gpu(lib, W):
    import torch
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    q = lib.nf4_quantize(torch.from_numpy(W).cuda(), status=status)
    torch.cuda.synchronize()
    return q, int(status.item())


@pytest.mark.parametrize("N,K,outliers", SHAPES)
def test_quantize_bit_exact(lib, N, K, outliers):
    W = inputs.weight_f32(N, K, outliers=outliers)
    q, st = _quantize_gpu(lib, W)
    assert st == 0
    codes, s8, s2 = onf4.quantize(W)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.scale8.cpu().numpy(), s8)
    assert np.array_equal(q.scale2.cpu().numpy().view(np.uint32), s2.view(np.uint32))


@pytest.mark.parametrize("N,K,outliers", SHAPES)
def test_dequantize_bit_exact(lib, N, K, outliers):
    W = inputs.weight_f32(N, K, index=1, outliers=outliers)
    q, _ = _quantize_gpu(lib, W)
    out = lib.nf4_dequantize(q)
    import torch
    torch.cuda.synchronize()
    codes, s8, s2 = onf4.quantize(W)
    ref = onf4.dequantize_bits(codes, s8, s2, N, K)
    assert np.array_equal(bf16_dev_bits(out), ref)


def test_special_blocks(lib):
    """All-zero blocks, signed zeros, subnormals, a block whose max is negative,
    exact midpoint ties between levels."""
    W = np.zeros((4, 256), dtype=np.float32)
    W[0, 64:128] = inputs.normal_f32(9, 64, 1e-39)        # subnormal block
    W[1, :64] = -np.abs(inputs.normal_f32(10, 64, 0.5))
    W[1, 5] = -3.0                                         # negative absmax -> code 0
    W[2, 64] = -0.0
    L = onf4.nf4_levels().astype(np.float64)
    mids = [np.float32((L[i] + L[i + 1]) / 2) for i in range(15)]
    W[3, :15] = mids
    W[3, 15] = 1.0
    W[3, 64:79] = [np.nextafter(m, np.float32(2)) for m in mids]
    W[3, 79] = -1.0
    q, st = _quantize_gpu(lib, W)
    assert st == 0
    codes, s8, s2 = onf4.quantize(W)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    assert np.array_equal(q.scale8.cpu().numpy(), s8)
    assert np.array_equal(q.scale2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    out = lib.nf4_dequantize(q)
    assert np.array_equal(bf16_dev_bits(out), onf4.dequantize_bits(codes, s8, s2, 4, 256))


@pytest.mark.parametrize("bad", [np.inf, -np.inf, np.nan])
def test_nonfinite_sets_device_status(lib, bad):
    W = inputs.weight_f32(32, 128)
    W[7, 33] = bad
    _, st = _quantize_gpu(lib, W)
    assert st == 5  # QLORA_ERR_NONFINITE


def test_status_is_cleared_by_next_quantize(lib):
    W = inputs.weight_f32(32, 128)
    _, st = _quantize_gpu(lib, W)
    assert st == 0


@pytest.mark.parametrize("N,K", [(256, 1024), (272, 320), (4096, 4096)])
def test_int4_comparison_codec_bit_exact(lib, N, K):
    """The int4 comparison codec (same format, evenly spaced levels): codes,
    block constants and the dequantised bf16 weight bit for bit against
    oracle.codebooks, and its levels as the oracle's."""
    import torch
    from oracle import codebooks
    W = inputs.weight_f32(N, K, index=7, outliers=(N == 4096))
    q = lib.codec_quantize(torch.from_numpy(W).cuda(), lib.CODEBOOK_INT4)
    out = lib.codec_dequantize(q, lib.CODEBOOK_INT4)
    torch.cuda.synchronize()
    p, s8, s2 = codebooks.quantize_int4(W)
    np.testing.assert_array_equal(q.codes.cpu().numpy(), p)
    np.testing.assert_array_equal(q.scale8.cpu().numpy(), s8)
    np.testing.assert_array_equal(q.scale2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    np.testing.assert_array_equal(bf16_dev_bits(out), codebooks.dequantize_int4_bits(p, s8, s2, N, K))
    np.testing.assert_array_equal(np.array(lib.codec_levels(lib.CODEBOOK_INT4), dtype=np.float32),
                                  codebooks.int4_levels())


def test_nf4_error_below_int4_on_the_gpu(lib):
    """The error ordering the pages state, measured on the GPU codecs for a
    4096 x 4096 weight from N(0, 0.02) with 0.1% x8 outliers."""
    import torch
    W = torch.from_numpy(inputs.weight_f32(4096, 4096, index=8, outliers=True)).cuda()
    err = {}
    for book in (lib.CODEBOOK_NF4, lib.CODEBOOK_INT4):
        back = lib.codec_dequantize(lib.codec_quantize(W, book), book).float()
        err[book] = torch.sqrt(torch.mean((back - W) ** 2)).item()
    assert err[lib.CODEBOOK_NF4] < 0.9 * err[lib.CODEBOOK_INT4]


def _fp8dq_case(kind):
    g = inputs.rng(40)
    if kind == "ragged":            # 240 blocks: one short group
        return (g.standard_normal((48, 320)) * 0.02).astype(np.float32)
    if kind == "constant":          # every block's absmax 0.03: d = 0, codes +0
        W = (g.uniform(-0.03, 0.03, (64, 512))).astype(np.float32)
        W.reshape(-1, 64)[:, 5] = 0.03
        return W
    if kind == "zeros":             # all-zero blocks inside groups of non-zero ones
        W = (g.standard_normal((256, 1024)) * 0.02).astype(np.float32)
        W[7, :] = 0.0
        W[100, 64:192] = 0.0
        return W
    return inputs.weight_f32(1024, 4096, index=9, outliers=True)


@pytest.mark.parametrize("kind", ["outliers", "ragged", "constant", "zeros"])
def test_fp8_second_level_bit_exact(lib, kind):
    """The comparison second level (E4M3 codes of mean-centred block
    constants, (d, mu) per group): codes, E4M3 codes, the float32 pairs and
    the dequantised bf16 weight bit for bit against oracle.dq_fp8."""
    import torch
    from oracle import dq_fp8
    W = _fp8dq_case(kind)
    N, K = W.shape
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = lib.dqfp8_quantize(torch.from_numpy(W).cuda(), status=st)
    out = lib.dqfp8_dequantize(q)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    p, s8, s2 = dq_fp8.quantize_fp8dq(W)
    np.testing.assert_array_equal(q.codes.cpu().numpy(), p)
    np.testing.assert_array_equal(q.scale8.cpu().numpy(), s8)
    np.testing.assert_array_equal(q.scale2.cpu().numpy().view(np.uint32), s2.reshape(-1).view(np.uint32))
    np.testing.assert_array_equal(bf16_dev_bits(out), dq_fp8.dequantize_fp8dq_bits(p, s8, s2, N, K))


def test_fp8_and_linear_second_levels_err_alike(lib):
    """Both second levels on the same 4096 x 4096 weight (N(0, 0.02), 0.1 %
    x8 outliers): the dequantisation error of the two differs by a few
    percent at most, since both keep the block constants to about 8 bits."""
    import torch
    W = torch.from_numpy(inputs.weight_f32(4096, 4096, index=8, outliers=True)).cuda()
    lin = lib.nf4_dequantize(lib.nf4_quantize(W)).float()
    f8 = lib.dqfp8_dequantize(lib.dqfp8_quantize(W)).float()
    e_lin = torch.sqrt(torch.mean((lin - W) ** 2)).item()
    e_f8 = torch.sqrt(torch.mean((f8 - W) ** 2)).item()
    assert abs(e_f8 - e_lin) < 0.03 * e_lin


def _boundary_weights(levels, seed):
    """Blocks whose quotients w / c1 fall within a few float32 steps of every
    decision point between adjacent levels, and of every multiple of 1/128
    (where an implementation may switch between internal search ranges), for
    block maxima of very different magnitudes, down to subnormal products. Element 0 of each block is +-c1
    so that c1 is the block's absmax."""
    rng = np.random.default_rng(seed)
    lv = np.asarray(levels, dtype=np.float64)
    points = [0.5 * (lv[i] + lv[i + 1]) for i in range(15)] + [k / 128.0 for k in range(-127, 128)]
    vals = []
    for p in points:
        x = np.float32(p)
        for k in range(-4, 5):
            y = x
            for _ in range(abs(k)):
                y = np.nextafter(y, np.float32(np.inf if k > 0 else -np.inf))
            vals.append(y)
    vals = np.clip(np.array(vals, dtype=np.float32), -1, 1)
    rows = []
    # maxima either side of 2^-125 and 2^126, where a quotient taken through
    # the reciprocal of c1 would leave the normal range
    edges = (2.0 ** -125, 2.0 ** -125 * 0.75, 2.0 ** 126, 2.0 ** 126 * 1.5)
    for c1 in (1.0, 0.0371, 3.0517578e-5, 7.5e3, float(rng.uniform(0.01, 0.2))) + edges:
        c1 = np.float32(c1)
        q = (vals.astype(np.float64) * np.float64(c1)).astype(np.float32)   # w near c1 * point
        pad = (-q.size) % 63
        q = np.concatenate([q, np.zeros(pad, np.float32)]).reshape(-1, 63)
        blk = np.concatenate([np.full((q.shape[0], 1), c1, np.float32), q], axis=1)
        blk[::2, 0] = -c1
        rows.append(blk)
    flat = np.concatenate(rows).reshape(-1)
    flat = np.concatenate([flat, np.zeros((-flat.size) % 512, np.float32)])
    return flat.reshape(-1, 512)


def test_quantize_codes_at_decision_points(lib):
    """Codes of quotients a few float32 steps either side of each level
    midpoint (and of the multiples of 1/128) match the oracle for NF4 and for
    the int4 comparison codebook ("QLoRA, in depth", "The mechanism in brief":
    nearest of the 16 levels)."""
    import torch
    from oracle import codebooks
    W = _boundary_weights(onf4.nf4_levels(), 21)
    q, st = _quantize_gpu(lib, W)
    assert st == 0
    codes, s8, s2 = onf4.quantize(W)
    assert np.array_equal(q.codes.cpu().numpy(), codes)
    W4 = _boundary_weights(codebooks.int4_levels(), 22)
    q4 = lib.codec_quantize(torch.from_numpy(W4).cuda(), lib.CODEBOOK_INT4)
    torch.cuda.synchronize()
    p4, _, _ = codebooks.quantize_int4(W4)
    np.testing.assert_array_equal(q4.codes.cpu().numpy(), p4)
