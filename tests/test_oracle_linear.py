"""Pins of the oracle's QLoRA linear forward and backward.

Source: "QLoRA, in depth", "The mechanism in brief": y = W x + (alpha/r) B A x
with W dequantised; backward gives gradients for A, B and the activations,
never for W. Pinned by exact rational brute force on tiny shapes, adjoint
identities, finite differences, and special cases that reduce to a library
matrix product (torch, a different library from the oracle's numpy).
"""

from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import linear, nf4
from bit_nf4_quantized_dequant_b200 import inputs


def _case(N, K, M, r, seed=0):
    W = inputs.weight_f32(N, K, index=seed)
    packed, s8, s2 = nf4.quantize(W)
    Wd = nf4.dequantize(packed, s8, s2, N, K)
    c = inputs.linear_case(N, K, M, r, index=seed)
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    return Wd, f(c["X"]), f(c["A"]), f(c["B"]), f(c["dY"])


def _frac(a):
    return [[Fraction(float(v)) for v in row] for row in np.atleast_2d(a)]


def _mm(a, b_t):
    """a [p, q] times b_t^T where b_t is [s, q] (lists of Fractions)."""
    return [[sum(x * y for x, y in zip(ra, rb)) for rb in b_t] for ra in a]


def _t(a):
    return [list(col) for col in zip(*a)]


def test_forward_backward_match_exact_brute_force():
    N, K, M, r, s = 4, 64, 3, 2, 2.0
    Wd, X, A, B, dY = _case(N, K, M, r)
    Y, U = linear.linear_fwd(Wd, X, A, B, s)
    dX, dA, dB = linear.linear_bwd(Wd, X, A, B, s, dY)
    Wf, Xf, Af, Bf, dYf = map(_frac, (Wd, X, A, B, dY))
    S = Fraction(s)
    Uf = _mm(Xf, Af)                                     # X A^T   [M, r]
    base = _mm(Xf, Wf)                                   # X W^T   [M, N]
    lora = _mm(Uf, Bf)                                   # U B^T   [M, N]
    Yf = [[base[m][n] + S * lora[m][n] for n in range(N)] for m in range(M)]
    Tf = _mm(dYf, _t(Bf))                                # dY B    [M, r]
    dXf = [[a + S * b for a, b in zip(ra, rb)] for ra, rb in zip(_mm(dYf, _t(Wf)), _mm(Tf, _t(Af)))]
    dAf = [[S * v for v in row] for row in _mm(_t(Tf), _t(Xf))]
    dBf = [[S * v for v in row] for row in _mm(_t(dYf), _t(Uf))]
    for got, ref in ((Y, Yf), (U, Uf), (dX, dXf), (dA, dAf), (dB, dBf)):
        ref = np.array([[float(v) for v in row] for row in ref])
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_adjoint_identities():
    N, K, M, r, s = 96, 192, 40, 8, 2.0
    Wd, X, A, B, dY = _case(N, K, M, r, seed=3)
    Y, U = linear.linear_fwd(Wd, X, A, B, s)
    dX, dA, dB = linear.linear_bwd(Wd, X, A, B, s, dY)
    # Y is linear in X: <dY, Y(X)> = <dX, X>
    assert np.vdot(dY, Y) == pytest.approx(np.vdot(dX, X), rel=1e-10)
    # the LoRA term is linear in A and in B separately
    lora = s * (X @ A.T) @ B.T
    assert np.vdot(dY, lora) == pytest.approx(np.vdot(dA, A), rel=1e-10)
    assert np.vdot(dY, lora) == pytest.approx(np.vdot(dB, B), rel=1e-10)


def test_finite_differences():
    N, K, M, r, s = 16, 64, 5, 4, 1.5
    Wd, X, A, B, dY = _case(N, K, M, r, seed=4)
    dX, dA, dB = linear.linear_bwd(Wd, X, A, B, s, dY)
    rng = np.random.Generator(np.random.PCG64(9))

    def loss(X_, A_, B_):
        return np.vdot(dY, linear.linear_fwd(Wd, X_, A_, B_, s)[0])

    h = 1e-3
    for grad, which in ((dX, 0), (dA, 1), (dB, 2)):
        args = [X, A, B]
        d = rng.standard_normal(args[which].shape)
        plus = list(args); plus[which] = args[which] + h * d
        minus = list(args); minus[which] = args[which] - h * d
        fd = (loss(*plus) - loss(*minus)) / (2 * h)
        assert fd == pytest.approx(np.vdot(grad, d), rel=1e-7, abs=1e-9)


def test_special_cases_reduce_to_library_products():
    N, K, M, r, s = 64, 128, 24, 8, 2.0
    Wd, X, A, B, dY = _case(N, K, M, r, seed=5)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    # B = 0: a plain GEMM with the dequantised weight
    Y0, _ = linear.linear_fwd(Wd, X, A, np.zeros_like(B), s)
    np.testing.assert_allclose(Y0, torch.matmul(t(X), t(Wd).T).numpy(), rtol=1e-12, atol=1e-12)
    # W' = 0: the pure LoRA path
    Y1, _ = linear.linear_fwd(np.zeros_like(Wd), X, A, B, s)
    ref = s * torch.matmul(torch.matmul(t(X), t(A).T), t(B).T)
    np.testing.assert_allclose(Y1, ref.numpy(), rtol=1e-12, atol=1e-14)
    # B = 0 backward: dX is dY W', dA = 0
    dX, dA, dB = linear.linear_bwd(Wd, X, A, np.zeros_like(B), s, dY)
    np.testing.assert_allclose(dX, torch.matmul(t(dY), t(Wd)).numpy(), rtol=1e-12, atol=1e-12)
    assert np.all(dA == 0)
    # linearity in X
    Ya, _ = linear.linear_fwd(Wd, X, A, B, s)
    Yb, _ = linear.linear_fwd(Wd, 2.0 * X, A, B, s)
    np.testing.assert_allclose(Yb, 2.0 * Ya, rtol=1e-13)


def test_row_helpers_agree_with_full_results():
    N, K, M, r, s = 32, 128, 12, 4, 2.0
    Wd, X, A, B, dY = _case(N, K, M, r, seed=6)
    Y, _ = linear.linear_fwd(Wd, X, A, B, s)
    dX, _, _ = linear.linear_bwd(Wd, X, A, B, s, dY)
    rows = np.array([0, 5, 11])
    np.testing.assert_allclose(linear.linear_fwd_rows(Wd, X[rows], A, B, s), Y[rows], rtol=1e-14)
    np.testing.assert_allclose(linear.linear_dx_rows(Wd, dY[rows], A, B, s), dX[rows], rtol=1e-14)


def test_planted_transpose_is_caught(monkeypatch):
    """Plant a wrong operand (dB from U^T dY) in the oracle: the brute-force pin fails."""
    real = linear.linear_bwd

    def wrong(Wd, X, A, B, s, dY):
        dX, dA, dB = real(Wd, X, A, B, s, dY)
        return dX, dA, s * (dY.T @ (X @ np.roll(A, 1, axis=0).T))

    monkeypatch.setattr(linear, "linear_bwd", wrong)
    with pytest.raises(AssertionError):
        test_forward_backward_match_exact_brute_force()
