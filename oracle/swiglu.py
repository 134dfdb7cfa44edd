"""SwiGLU MLP oracle (the gate / up / down chain of the pages' Llama-style
models), float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA and Fine-Tuning on One Consumer GPU" (multigrid.ai), section
"Where 24 GB goes": LoRA adapters on the attention and MLP projections of a
7B model, and gradient checkpointing, which keeps each layer's input and
recomputes the layer's MLP intermediates during the backward. The MLP of
those models computes h = silu(g) * u with g = gate(x), u = up(x) (each a
QLoRA linear) and then down(h); silu(x) = x / (1 + exp(-x)).

Reading (the pages name the chain, not its precision): g and u are the
outputs of their layers in the compute dtype, bf16, before silu; h is
compared in float64 against the kernels' bf16 result.
"""

from __future__ import annotations

import numpy as np

from . import linear, nf4


def bf16r(x: np.ndarray) -> np.ndarray:
    """float64 -> bf16 (round to nearest even, through float32) -> float64."""
    return nf4.bf16_bits_to_f64(nf4.bf16_round_bits(np.asarray(x, dtype=np.float64).astype(np.float32)))


def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def silu_grad(x: np.ndarray) -> np.ndarray:
    """d silu / dx = sigma(x) (1 + x (1 - sigma(x)))."""
    x = np.asarray(x, dtype=np.float64)
    sg = 1.0 / (1.0 + np.exp(-x))
    return sg * (1.0 + x * (1.0 - sg))


def swiglu_fwd(Wg, Wu, X, Ag, Bg, Au, Bu, s: float):
    """Returns (H, G, U): G = bf16(gate(X)), U = bf16(up(X)), H = silu(G) U."""
    G = bf16r(linear.linear_fwd(Wg, X, Ag, Bg, s)[0])
    U = bf16r(linear.linear_fwd(Wu, X, Au, Bu, s)[0])
    return silu(G) * U, G, U


def swiglu_bwd(G, U, dH):
    """Gradients of L = <dH, silu(G) U> with respect to G and U."""
    dH = np.asarray(dH, dtype=np.float64)
    return dH * U * silu_grad(G), dH * silu(G)
