"""Adapter merge oracle, float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA" (guide.dupenodi.dev), section "Walking through the tooling":
at inference the adapter is merged, W' = W + scaled BA, into one weight
file (or kept separate); "QLoRA, in depth" (aicassindra.com), section
"Shipping: merge, re-quantize, verify": the merged model is then quantised
again for serving, a second quantisation of weights trained against the
first; "QLoRA and Fine-Tuning on One Consumer GPU", section "What the paper
reports": a merge into 4-bit weights means dequantising, adding the adapter
and quantising once more, and what comes out is no longer the model that was
evaluated.

Here W is the dequantised NF4 base (the weights the adapter was trained
against), scaled BA = s B A with s = alpha / r.
"""

from __future__ import annotations

import numpy as np

from . import nf4


def merge(Wd: np.ndarray, A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """W' + s B A in float64 (W' given as float64 values of the bf16 weight)."""
    return np.asarray(Wd, dtype=np.float64) + s * (np.asarray(B, dtype=np.float64) @ np.asarray(A, dtype=np.float64))


def requant_drift(merged_f32: np.ndarray, Wd: np.ndarray, A: np.ndarray, B: np.ndarray, s: float):
    """Quantise the merged weight to NF4 again and compare its dequantised
    value with the exact merge. Returns (relative Frobenius error of the
    re-quantised merge against the exact merge, the same error divided by the
    norm of the adapter's contribution s B A). A ratio whose denominator is
    zero (a zero adapter, or a zero merge) is inf when the drift is not zero
    and NaN when it is."""
    N, K = merged_f32.shape
    back = nf4.dequantize(*nf4.quantize(merged_f32), N, K)
    exact = merge(Wd, A, B, s)
    err = np.linalg.norm(back - exact)
    ref = np.linalg.norm(exact)
    delta = np.linalg.norm(exact - np.asarray(Wd, dtype=np.float64))
    # a zero merge or a zero adapter leaves a ratio undefined: inf when there
    # is drift to relate to nothing, NaN when there is none
    ratio = lambda den: err / den if den > 0 else (np.inf if err > 0 else np.nan)
    return ratio(ref), ratio(delta)
