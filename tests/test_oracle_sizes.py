"""Pins of the oracle's storage ledger against the figures the pages print
(``tests/golden/pages_figures.txt``, each line citing its page and section)."""

import os

import pytest

from oracle import sizes as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_figures.txt")


def _golden():
    out = {}
    with open(GOLDEN) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            key, val, tol, src = [p.strip() for p in line.split("|")]
            out[key] = (float(val), tol, src)
    return out


def _computed():
    dq_overhead = S.bits_per_weight(True) - 4.0
    saving_bits = S.bits_per_weight(False) - S.bits_per_weight(True)
    params_7b = S.linear_weight_count("7B") + S.embed_head_params("7B")
    return {
        "bits_per_weight_dq": S.bits_per_weight(True),
        "bits_per_weight_no_dq": S.bits_per_weight(False),
        "dq_overhead_bits": dq_overhead,
        "fp32_scale_overhead_bits": S.bits_per_weight(False) - 4.0,
        "dq_saving_bits": saving_bits,
        "dq_saving_8b_bytes": saving_bits * 8e9 / 8,
        "dq_saving_65b_bytes": 0.37 * 65e9 / 8,
        "base_7b_nf4_bytes": params_7b * 0.5,
        "constants_7b_bytes": params_7b * dq_overhead / 8,
        "embed_head_8b_params": S.embed_head_params("8B"),
        "quantized_linears_8b_bytes": S.nf4_linear_bytes("8B"),
        "embed_head_8b_bytes": 2 * S.embed_head_params("8B"),
        "total_8b_qlora_bytes": S.qlora_weight_bytes("8B"),
        "lora_3b_r16_params": S.lora_params("3B", 16),
        "qlora_3b_weight_bytes": S.qlora_weight_bytes("3B"),
        "saving_1b_bytes": S.bf16_weight_bytes("1B") - S.qlora_weight_bytes("1B"),
        "saving_8b_min_bytes": S.bf16_weight_bytes("8B") - S.qlora_weight_bytes("8B"),
        "embed_share_1b": 2 * S.embed_head_params("1B") / S.qlora_weight_bytes("1B"),
    }


@pytest.mark.parametrize("key", sorted(_golden()))
def test_page_figure(key):
    val, tol, src = _golden()[key]
    got = _computed()[key]
    if tol == "lower-bound":
        assert got > val, src
    else:
        assert got == pytest.approx(val, rel=float(tol), abs=0 if float(tol) else 1e-12), src


def test_exact_values():
    # 4 + 8/64 + 32/(64*256) exactly
    assert S.bits_per_weight(True) == 4.126953125
    # rank 16 on all seven linears of the 3B shape: 28 * 868352
    assert S.lora_params("3B", 16) == 24_313_856
    # the 8B linear set and its packed size (N*K/2 + N*K/64 + 4*ceil(N*K/64/256) per matrix)
    assert S.linear_weight_count("8B") == 6_979_321_856
    assert S.nf4_linear_bytes("8B") == 3_600_416_768


def test_storage_of_one_matrix():
    assert S.nf4_storage_bytes(1024, 1024) == (524288, 16384, 256)
    assert S.nf4_storage_bytes(4096, 4096) == (8388608, 262144, 4096)
    assert sum(S.nf4_storage_bytes(11008, 4096)) == 23_259_904
    # a short last group still costs a full 32-bit scale
    assert S.nf4_storage_bytes(1, 64 * 257) == (64 * 257 // 2, 257, 8)
