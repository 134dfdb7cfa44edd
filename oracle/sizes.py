"""Storage ledger of the NF4 format and LoRA parameter counts.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (page title, section):
  * "QLoRA, in depth", "The mechanism in brief": about 4.127 bits per weight
    with double quantisation instead of 4.5 without it.
  * "QLoRA, in depth", "Where the memory goes in a small model": rank-16 LoRA
    on every linear of a 3B model (28 layers, hidden 3072, 8 KV heads, MLP
    8192) adds 24.3 million parameters; embedding, norms and head stay 16-bit.
  * "What is QLoRA ...", "The three QLoRA ideas" and "Why an 8B model is about
    5-6 GB, not 4 GB".
  * "QLoRA and Fine-Tuning on One Consumer GPU", "NF4 and double
    quantisation" and "Where 24 GB goes".
"""

from __future__ import annotations

BLOCK = 64
GROUP = 256


def nf4_storage_bytes(rows: int, cols: int):
    """(code bytes, 8-bit scale bytes, fp32 second-level scale bytes) of one
    [rows, cols] matrix: half a byte per weight, one byte per block of 64,
    four bytes per group of 256 blocks (the last group may be short)."""
    n = rows * cols
    if cols % BLOCK:
        raise ValueError("cols must be a multiple of 64")
    nb = n // BLOCK
    ng = -(-nb // GROUP)
    return n // 2, nb, 4 * ng


def nf4_total_bytes(rows: int, cols: int) -> int:
    return sum(nf4_storage_bytes(rows, cols))


def bits_per_weight(double_quant: bool = True) -> float:
    """Storage cost per weight for a matrix whose block count is a multiple of
    256: 4 code bits + the per-block constant amortised over 64 weights (8 bits
    with double quantisation, a 32-bit float without) + (with double
    quantisation) one 32-bit second-level scale per 256 * 64 weights."""
    if double_quant:
        return 4.0 + 8.0 / BLOCK + 32.0 / (BLOCK * GROUP)
    return 4.0 + 32.0 / BLOCK


# Linear layers of one decoder layer as (name, out_features N, in_features K).
def llama_linears(hidden: int, kv_dim: int, mlp: int):
    return [
        ("q", hidden, hidden), ("k", kv_dim, hidden), ("v", kv_dim, hidden),
        ("o", hidden, hidden), ("gate", mlp, hidden), ("up", mlp, hidden),
        ("down", hidden, mlp),
    ]


# Model shapes the pages use (layer count, linears, vocabulary, hidden).
MODELS = {
    # Llama-3.2-1B: hidden 2048, 16 layers, 8 KV heads x 64, MLP 8192, tied embedding
    "1B": dict(layers=16, linears=llama_linears(2048, 512, 8192), vocab=128256, hidden=2048, tied=True),
    # Llama-3.2-3B: hidden 3072, 28 layers, 8 KV heads x 128, MLP 8192, tied embedding
    "3B": dict(layers=28, linears=llama_linears(3072, 1024, 8192), vocab=128256, hidden=3072, tied=True),
    # Llama-7B (first/second generation): hidden 4096, 32 layers, full KV, MLP 11008
    "7B": dict(layers=32, linears=llama_linears(4096, 4096, 11008), vocab=32000, hidden=4096, tied=False),
    # Llama-3.1-8B: hidden 4096, 32 layers, 8 KV heads x 128, MLP 14336, untied head
    "8B": dict(layers=32, linears=llama_linears(4096, 1024, 14336), vocab=128256, hidden=4096, tied=False),
}


def linear_weight_count(model: str) -> int:
    m = MODELS[model]
    return m["layers"] * sum(n * k for _, n, k in m["linears"])


def embed_head_params(model: str) -> int:
    m = MODELS[model]
    return (1 if m["tied"] else 2) * m["vocab"] * m["hidden"]


def lora_params(model: str, r: int, names=None) -> int:
    """A is [r, K] and B is [N, r] for every adapted linear: r (N + K) each."""
    m = MODELS[model]
    per_layer = sum(r * (n + k) for name, n, k in m["linears"] if names is None or name in names)
    return m["layers"] * per_layer


def nf4_linear_bytes(model: str) -> int:
    """Packed NF4 bytes of every linear of the model (constants included)."""
    m = MODELS[model]
    return m["layers"] * sum(nf4_total_bytes(n, k) for _, n, k in m["linears"])


def qlora_weight_bytes(model: str) -> int:
    """NF4 linears plus the bf16 embedding/head the pages say stays 16-bit."""
    return nf4_linear_bytes(model) + 2 * embed_head_params(model)


def bf16_weight_bytes(model: str) -> int:
    return 2 * (linear_weight_count(model) + embed_head_params(model))
