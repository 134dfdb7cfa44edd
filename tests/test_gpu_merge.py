"""GPU parity of the adapter merge W' + s B A (bf16 and fp32 outputs) against
oracle.merge, and of the merge -> re-quantisation path's drift against the
oracle's. bf16 results may differ from the float64 merge rounded to bf16 by
one bf16 unit in the last place (the kernel sums s B A in fp32 first)."""

import numpy as np
import pytest

from oracle import merge as omerge, nf4 as onf4
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu

CASES = [
    # N, K, r, s
    (128, 320, 16, 2.0),     # two column strips, the second with one of four blocks
    (512, 1024, 8, 4.0),
    (64, 256, 64, 0.5),      # largest rank: four MMA K-steps
    (1040, 768, 24, 1.5),    # rank not a multiple of 16, 65 row tiles
]


def _inputs(N, K, r, seed):
    g = inputs.rng(seed)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    A = onf4.bf16_round_bits((g.standard_normal((r, K)) / r).astype(np.float32))
    B = onf4.bf16_round_bits((g.standard_normal((N, r)) * 0.01).astype(np.float32))
    return W, A, B


@pytest.mark.parametrize("N,K,r,s", CASES)
def test_merge_bf16_and_f32(lib, N, K, r, s):
    import torch
    W, A, B = _inputs(N, K, r, 500 + N + K + r)
    q = lib.nf4_quantize(torch.from_numpy(W).cuda())
    Ad, Bd = to_dev_bf16(A), to_dev_bf16(B)
    out16 = lib.nf4_merge(q, Ad, Bd, s)
    out32 = lib.nf4_merge(q, Ad, Bd, s, f32=True)
    torch.cuda.synchronize()
    Wd = onf4.dequantize(*onf4.quantize(W), N, K)
    ref = omerge.merge(Wd, onf4.bf16_bits_to_f64(A), onf4.bf16_bits_to_f64(B), s)
    got16 = bf16_dev_to_f64(out16)
    ulp = np.abs(onf4.bf16_bits_to_f64(onf4.bf16_round_bits(ref.astype(np.float32)))) * 2.0 ** -7
    assert np.all(np.abs(got16 - ref) <= ulp + 1e-30)
    # fp32 result: a few fp32 roundings of the operands' magnitudes (the sum can cancel)
    Ah, Bh = onf4.bf16_bits_to_f64(A), onf4.bf16_bits_to_f64(B)
    bound = 8 * 2.0 ** -24 * (np.abs(Wd) + s * (np.abs(Bh) @ np.abs(Ah)))
    assert np.all(np.abs(out32.double().cpu().numpy() - ref) <= bound)


def test_merge_then_requantise_drift(lib):
    """Merging into the 4-bit base means quantising the merged weight again:
    the drift of that re-quantised merge from the exact merge, relative to the
    merge and to the adapter's own contribution, matches the oracle's."""
    import torch
    N, K, r, s = 1024, 2048, 16, 2.0
    W, A, B = _inputs(N, K, r, 510)
    q = lib.nf4_quantize(torch.from_numpy(W).cuda())
    Ad, Bd = to_dev_bf16(A), to_dev_bf16(B)
    m32 = lib.nf4_merge(q, Ad, Bd, s, f32=True)
    q2 = lib.nf4_quantize(m32)
    back = lib.nf4_dequantize(q2)
    torch.cuda.synchronize()
    Wd = onf4.dequantize(*onf4.quantize(W), N, K)
    Ah, Bh = onf4.bf16_bits_to_f64(A), onf4.bf16_bits_to_f64(B)
    exact = omerge.merge(Wd, Ah, Bh, s)
    err = np.linalg.norm(bf16_dev_to_f64(back) - exact)
    rel, rel_delta = err / np.linalg.norm(exact), err / np.linalg.norm(exact - Wd)
    orel, orel_delta = omerge.requant_drift(exact.astype(np.float32), Wd, Ah, Bh, s)
    assert abs(rel - orel) <= 0.02 * orel and abs(rel_delta - orel_delta) <= 0.02 * orel_delta
