"""QLoRA linear layer oracle: forward and backward in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA, in depth" (aicassindra.com), section "The mechanism in brief":
every forward dequantises W to the compute dtype and computes
W x + (alpha / r) B A x, where A and B are the LoRA matrices of rank r;
backward computes gradients for A, B and the activations, never for W.
"What is QLoRA ..." (mantramindai.in), "Follow-up questions to expect": the
adapters train in bf16 or fp32, only the frozen base is 4-bit.

Shapes (row-major, PyTorch convention): W'[N, K] (the dequantised bf16 weight,
given here as float64 values), X[M, K], A[r, K], B[N, r], dY[M, N];
s = alpha / r. The layer is Y = X W'^T + s (X A^T) B^T.

All operands are float64 copies of the bf16 (or float32) inputs; nothing is
rounded in between. A matrix product is the only library step used.
"""

from __future__ import annotations

import numpy as np


def linear_fwd(Wd: np.ndarray, X: np.ndarray, A: np.ndarray, B: np.ndarray,
               s: float):
    """Returns (Y [M, N], U [M, r]) with U = X A^T and Y = X W'^T + s U B^T."""
    X = np.asarray(X, dtype=np.float64)
    U = X @ np.asarray(A, dtype=np.float64).T
    Y = X @ np.asarray(Wd, dtype=np.float64).T + s * (U @ np.asarray(B, dtype=np.float64).T)
    return Y, U


def linear_bwd(Wd: np.ndarray, X: np.ndarray, A: np.ndarray, B: np.ndarray,
               s: float, dY: np.ndarray):
    """Gradients of L = <dY, Y> for the layer above, with W frozen.

    T  = dY B                 [M, r]
    dX = dY W' + s T A        [M, K]
    dA = s T^T X              [r, K]
    dB = s dY^T (X A^T)       [N, r]
    No dW is formed.
    """
    X = np.asarray(X, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    T = dY @ B
    dX = dY @ np.asarray(Wd, dtype=np.float64) + s * (T @ A)
    dA = s * (T.T @ X)
    dB = s * (dY.T @ (X @ A.T))
    return dX, dA, dB


def linear_fwd_rows(Wd: np.ndarray, X_rows: np.ndarray, A, B, s: float) -> np.ndarray:
    """Y for a subset of token rows (the forward is row-independent)."""
    return linear_fwd(Wd, X_rows, A, B, s)[0]


def linear_dx_rows(Wd: np.ndarray, dY_rows: np.ndarray, A, B, s: float) -> np.ndarray:
    """dX for a subset of token rows (dX row m depends only on dY row m)."""
    dY_rows = np.asarray(dY_rows, dtype=np.float64)
    T = dY_rows @ np.asarray(B, dtype=np.float64)
    return dY_rows @ np.asarray(Wd, dtype=np.float64) + s * (T @ np.asarray(A, dtype=np.float64))
