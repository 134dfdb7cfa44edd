"""Seeded synthetic inputs for the QLoRA linear workloads.

This module only draws random numbers and shapes them: it holds none of the
NF4 or linear-layer arithmetic. Tests, the benchmark and the CPU reference all
take their inputs from here, so the CUDA library and the CPU oracle see the
same bytes.

Value recipe (the shapes are those of the workloads below):
  * W  ~ N(0, 0.02) float32 ("std 0.02" read as the standard deviation);
    the attention-projection workload also multiplies exactly
    floor(0.001 * N * K) distinct, seeded entries by 8 (outliers).
  * X  ~ N(0, 1) rounded to bf16;   dY ~ N(0, 1) rounded to bf16.
  * A  ~ N(0, 1/r) rounded to bf16 ("1/r" read as the standard deviation).
  * B  ~ N(0, 0.01) rounded to bf16.
Seeds: W 0, X 1, A 2, B 3, dY 4, outliers 5, each offset by 16 * the index of
the matrix inside a multi-matrix workload.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

SEED_W, SEED_X, SEED_A, SEED_B, SEED_DY, SEED_OUTLIER = 0, 1, 2, 3, 4, 5


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_f32(seed: int, shape, std: float) -> np.ndarray:
    x = rng(seed).standard_normal(size=shape, dtype=np.float32)
    return (x * np.float32(std)).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16) via torch's round-to-nearest-even cast."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def with_outliers(W: np.ndarray, seed: int, frac: float = 1e-3, factor: float = 8.0) -> np.ndarray:
    """Multiply exactly floor(frac * W.size) distinct seeded entries by factor."""
    n = int(np.floor(frac * W.size))
    out = W.copy().reshape(-1)
    if n:
        idx = rng(seed).choice(W.size, size=n, replace=False)
        out[idx] = (out[idx] * np.float32(factor)).astype(np.float32)
    return out.reshape(W.shape)


@dataclass
class Linear:
    """One QLoRA linear: W[N, K] is quantised, the adapter has rank r."""
    name: str
    N: int
    K: int


@dataclass
class Workload:
    name: str
    M: int                      # tokens
    r: int
    alpha: float
    linears: list = field(default_factory=list)
    outliers: bool = False
    description: str = ""

    @property
    def s(self) -> float:
        return self.alpha / self.r


def _llama(hidden, kv, mlp):
    return [Linear("q", hidden, hidden), Linear("k", kv, hidden), Linear("v", kv, hidden),
            Linear("o", hidden, hidden), Linear("gate", mlp, hidden), Linear("up", mlp, hidden),
            Linear("down", hidden, mlp)]


WORKLOADS = {
    "linear_1k": Workload(
        "linear_1k", M=64, r=8, alpha=16, linears=[Linear("w", 1024, 1024)],
        description="single QLoRA linear 1024x1024, 64 tokens, r=8, alpha=16"),
    "attn_proj_7b": Workload(
        "attn_proj_7b", M=2048, r=16, alpha=32, linears=[Linear("w", 4096, 4096)], outliers=True,
        description="Llama-7B attention projection 4096x4096 with 0.1% x8 outliers, "
                    "batch 1 x seq 2048 tokens, r=16, alpha=32"),
    "mlp_7b": Workload(
        "mlp_7b", M=4096, r=16, alpha=32,
        linears=[Linear("gate", 11008, 4096), Linear("up", 11008, 4096), Linear("down", 4096, 11008)],
        description="Llama-7B SiLU-gated MLP gate/up 4096->11008, down 11008->4096, "
                    "2x2048 tokens, r=16, alpha=32, forward recomputed before backward"),
    "stack_3b": Workload(
        "stack_3b", M=2048, r=16, alpha=32, linears=_llama(3072, 1024, 8192) * 28,
        description="3B decoder stack: 28 layers x 7 linears (hidden 3072, kv 1024, "
                    "MLP 8192), 2048 tokens, r=16, alpha=32"),
    "set_8b": Workload(
        "set_8b", M=4096, r=16, alpha=32, linears=_llama(4096, 1024, 14336) * 32,
        description="8B linear set: 32 layers x 7 linears (hidden 4096, kv 1024, "
                    "MLP 14336), 4096 tokens, r=16, alpha=32"),
    "set_8b_decode": Workload(
        "set_8b_decode", M=8, r=16, alpha=32, linears=_llama(4096, 1024, 14336) * 32,
        description="8B linear set forward at 8 tokens (memory-bound)"),
}


def weight_f32(N: int, K: int, index: int = 0, outliers: bool = False) -> np.ndarray:
    W = normal_f32(SEED_W + 16 * index, (N, K), 0.02)
    if outliers:
        W = with_outliers(W, SEED_OUTLIER + 16 * index)
    return W


def activations_bf16(M: int, K: int, index: int = 0) -> np.ndarray:
    return to_bf16_bits(normal_f32(SEED_X + 16 * index, (M, K), 1.0))


def lora_a_bf16(r: int, K: int, index: int = 0) -> np.ndarray:
    return to_bf16_bits(normal_f32(SEED_A + 16 * index, (r, K), 1.0 / r))


def lora_b_bf16(N: int, r: int, index: int = 0) -> np.ndarray:
    return to_bf16_bits(normal_f32(SEED_B + 16 * index, (N, r), 0.01))


def grad_out_bf16(M: int, N: int, index: int = 0) -> np.ndarray:
    return to_bf16_bits(normal_f32(SEED_DY + 16 * index, (M, N), 1.0))


def linear_case(N: int, K: int, M: int, r: int, index: int = 0, outliers: bool = False):
    """All inputs of one linear: W float32, X/A/B/dY as bf16 bit patterns."""
    return dict(
        W=weight_f32(N, K, index, outliers),
        X=activations_bf16(M, K, index),
        A=lora_a_bf16(r, K, index),
        B=lora_b_bf16(N, r, index),
        dY=grad_out_bf16(M, N, index),
    )
