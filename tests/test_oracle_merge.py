"""Pins of the merge oracle: the merged weight against torch's matmul on the
same operands, a zero adapter leaving W' unchanged, and the re-quantisation
drift: zero when the merge already lies on the NF4 grid (zero adapter), and
positive otherwise."""

import numpy as np
import torch

from oracle import merge, nf4
from bit_nf4_quantized_dequant_b200 import inputs


def _case(N=64, K=256, r=16, seed=400):
    g = inputs.rng(seed)
    W = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wd = nf4.dequantize(*nf4.quantize(W), N, K)
    A = nf4.bf16_bits_to_f64(nf4.bf16_round_bits((g.standard_normal((r, K)) / r).astype(np.float32)))
    B = nf4.bf16_bits_to_f64(nf4.bf16_round_bits((g.standard_normal((N, r)) * 0.01).astype(np.float32)))
    return Wd, A, B


def test_merge_matches_torch():
    Wd, A, B = _case()
    ref = torch.from_numpy(Wd) + 2.0 * (torch.from_numpy(B) @ torch.from_numpy(A))
    np.testing.assert_allclose(merge.merge(Wd, A, B, 2.0), ref.numpy(), rtol=1e-14, atol=1e-17)


def test_zero_adapter_is_identity():
    Wd, A, B = _case(seed=401)
    np.testing.assert_array_equal(merge.merge(Wd, A, np.zeros_like(B), 2.0), Wd)


def test_requant_of_the_base_alone_is_not_exact():
    """Re-quantising W' itself is not the identity (its block absmax is the
    bf16 of level 1 times the block scale, and the 8-bit constants round
    again), so even a zero adapter drifts by a little: the pages' warning
    about requantising merged weights holds before any adapter is added."""
    Wd, A, B = _case(seed=403)
    rel, rel_delta = merge.requant_drift(Wd.astype(np.float32), Wd, A, np.zeros_like(B), 0.0)
    assert 0.0 < rel < 0.05
    assert rel_delta == np.inf          # drift against an adapter contribution of zero


def test_requant_drift_is_positive_with_an_adapter():
    Wd, A, B = _case(seed=402)
    m = merge.merge(Wd, A, B, 2.0).astype(np.float32)
    rel, rel_delta = merge.requant_drift(m, Wd, A, B, 2.0)
    assert 0.0 < rel < 0.2
    assert rel_delta > 0.0
