"""Pins of the SwiGLU oracle: silu against torch's, its derivative and the
chain's gradients against central finite differences, and the forward with
zero adapters against torch's own matmul, bf16 cast and silu."""

import numpy as np
import pytest
import torch

from oracle import linear as olin, nf4, swiglu
from bit_nf4_quantized_dequant_b200 import inputs


def test_silu_matches_torch():
    x = inputs.rng(90).standard_normal(10_000) * 6.0
    x = np.concatenate([x, [0.0, 40.0, -40.0, 1e-8, -1e-8]])
    np.testing.assert_allclose(swiglu.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                               rtol=1e-13, atol=1e-300)
    assert swiglu.silu(np.array([0.0]))[0] == 0.0


def test_silu_grad_finite_differences():
    x = inputs.rng(91).standard_normal(2000) * 4.0
    h = 1e-6
    fd = (swiglu.silu(x + h) - swiglu.silu(x - h)) / (2 * h)
    np.testing.assert_allclose(swiglu.silu_grad(x), fd, rtol=1e-7, atol=1e-9)


def test_swiglu_bwd_finite_differences():
    g = inputs.rng(92)
    G, U, dH = g.standard_normal((3, 5, 7))
    dG, dU = swiglu.swiglu_bwd(G, U, dH)
    L = lambda G_, U_: float(np.sum(dH * swiglu.silu(G_) * U_))
    h = 1e-6
    for (i, j) in [(0, 0), (2, 3), (4, 6)]:
        E = np.zeros_like(G)
        E[i, j] = h
        assert abs((L(G + E, U) - L(G - E, U)) / (2 * h) - dG[i, j]) < 1e-7
        assert abs((L(G, U + E) - L(G, U - E)) / (2 * h) - dU[i, j]) < 1e-7


def test_swiglu_fwd_zero_adapters_matches_torch():
    """A = B = 0: H = silu(bf16(X Wg^T)) bf16(X Wu^T), here with torch's matmul,
    bf16 cast and silu on float32 values."""
    g = inputs.rng(93)
    F, K, M, r = 64, 128, 9, 8
    Wg, Wu = (nf4.bf16_bits_to_f64(nf4.bf16_round_bits((g.standard_normal((F, K)) * 0.05).astype(np.float32)))
              for _ in range(2))
    X = nf4.bf16_bits_to_f64(nf4.bf16_round_bits(g.standard_normal((M, K)).astype(np.float32)))
    Z = np.zeros((r, K)), np.zeros((F, r))
    H, G, U = swiglu.swiglu_fwd(Wg, Wu, X, Z[0], Z[1], Z[0], Z[1], 2.0)
    t = lambda a: torch.from_numpy(a)
    Gt = (t(X) @ t(Wg).T).float().bfloat16().double()
    Ut = (t(X) @ t(Wu).T).float().bfloat16().double()
    Ht = torch.nn.functional.silu(Gt) * Ut
    np.testing.assert_array_equal(G, Gt.numpy())
    np.testing.assert_array_equal(U, Ut.numpy())
    np.testing.assert_allclose(H, Ht.numpy(), rtol=1e-12)


def test_planted_derivative_mistake_is_caught(monkeypatch):
    """A plausible slip in the derivative (sigma(x) alone, dropping the
    x sigma (1 - sigma) term) fails the finite-difference pin."""
    monkeypatch.setattr(swiglu, "silu_grad", lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64))))
    with pytest.raises(AssertionError):
        test_silu_grad_finite_differences()
