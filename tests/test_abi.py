"""The C-ABI library builds for sm_100a, loads, exports every symbol that
include/qlora.h declares, and its host-only calls and argument checks behave
as documented. No kernel is launched here (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import nf4 as onf4, sizes as osizes

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "qlora.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    syms = declared_symbols()
    assert syms == sorted(lib.SYMBOLS)
    so = lib.library()
    for s in syms:
        assert getattr(so, s) is not None


def test_sizes_match_oracle(lib):
    for rows, cols in [(1024, 1024), (4096, 4096), (11008, 4096), (1, 64 * 257), (48, 192)]:
        assert lib.nf4_sizes(rows, cols) == osizes.nf4_storage_bytes(rows, cols)


def test_codebook_matches_oracle_derivation_bitwise(lib):
    """The library's hard-coded levels against the oracle's own derivation
    (bisection quantile function): two independent computations."""
    assert np.array_equal(lib.nf4_codebook().view(np.uint32), onf4.nf4_levels().view(np.uint32))


def test_status_strings(lib):
    for code, name in lib.STATUS.items():
        assert lib.status_string(code) == name


def _nf4(rows, cols, codes=0x10000, s8=0x20000, s2=0x30000):
    return lib_struct(rows, cols, codes, s8, s2)


def lib_struct(rows, cols, codes, s8, s2):
    from bit_nf4_quantized_dequant_b200._binding import _NF4
    return _NF4(rows, cols, codes, s8, s2)


def test_argument_errors_are_returned_before_any_launch(lib):
    so = lib.library()
    SZ = ctypes.c_size_t
    a, b, c = SZ(), SZ(), SZ()
    assert so.qlora_nf4_sizes(16, 100, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 2
    assert so.qlora_nf4_sizes(0, 64, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 1
    assert so.qlora_nf4_sizes(16, 64, None, ctypes.byref(b), ctypes.byref(c)) == 1
    assert so.qlora_nf4_codebook(None) == 1
    # quantize: null input, bad shape, misaligned pointers
    q = _nf4(16, 64)
    assert so.qlora_nf4_quantize(None, ctypes.byref(q), None, None) == 1
    assert so.qlora_nf4_quantize(ctypes.c_void_p(0x40008), ctypes.byref(q), None, None) == 3
    q_bad = _nf4(16, 100)
    assert so.qlora_nf4_quantize(ctypes.c_void_p(0x40000), ctypes.byref(q_bad), None, None) == 2
    q_mis = _nf4(16, 64, codes=0x10004)
    assert so.qlora_nf4_dequantize(ctypes.byref(q_mis), ctypes.c_void_p(0x40000), None) == 3
    assert so.qlora_nf4_dequantize(ctypes.byref(q), None, None) == 1
    # linear: unsupported rank, shape, null operands, missing workspace
    P = ctypes.c_void_p
    X, A, B, Y = P(0x50000), P(0x60000), P(0x70000), P(0x80000)
    q = _nf4(32, 64)
    fwd = so.qlora_linear_fwd
    assert fwd(ctypes.byref(q), X, 8, A, B, 12, 2.0, Y, None, None, 0, None, None) == 2
    assert fwd(ctypes.byref(q), X, 8, A, B, 72, 2.0, Y, None, None, 0, None, None) == 2
    assert fwd(ctypes.byref(q), None, 8, A, B, 16, 2.0, Y, None, None, 0, None, None) == 1
    assert fwd(ctypes.byref(q), X, 0, A, B, 16, 2.0, Y, None, None, 0, None, None) == 1
    assert fwd(ctypes.byref(q), X, 8, A, B, 16, float("nan"), Y, None, None, 0, None, None) == 1
    assert fwd(ctypes.byref(q), X, 8, A, B, 16, 2.0, Y, None, None, 0, None, None) == 4
    assert fwd(ctypes.byref(q), P(0x50002), 8, A, B, 16, 2.0, Y, None, None, 0, None, None) == 3
    q_rows = _nf4(40, 64)
    assert fwd(ctypes.byref(q_rows), X, 8, A, B, 16, 2.0, Y, None, None, 0, None, None) == 2
    bwd = so.qlora_linear_bwd
    assert bwd(ctypes.byref(q), X, 8, A, B, 16, 2.0, None, None, None, P(0x90000), P(0xA0000),
               P(0xB0000), 1 << 20, None, None) == 1
    assert so.qlora_linear_workspace(8, 32, 64, 16, None) == 1
    ws = SZ()
    assert so.qlora_linear_workspace(8, 32, 100, 16, ctypes.byref(ws)) == 2
    # fused GEMMs: the optional stream-K workspace is checked before any launch
    assert so.qlora_fused_workspace(0, ctypes.byref(ws)) == 1
    assert so.qlora_fused_workspace(8, None) == 1
    assert so.qlora_fused_workspace(8, ctypes.byref(ws)) == 0 and ws.value > 0
    need = ws.value
    sU, WS = P(0x90000), P(0xC0000)
    assert so.qlora_fused_fwd(ctypes.byref(q), X, 8, B, 16, sU, Y, WS, need - 1, None, None) == 4
    assert so.qlora_fused_dx(ctypes.byref(q), X, 8, A, 16, sU, Y, WS, need - 1, None, None) == 4
    assert so.qlora_fused_fwd(ctypes.byref(q), X, 8, B, 16, sU, Y, P(0xC0008), need, None, None) == 3


def test_fused_workspace_scales_with_token_tile(lib):
    """Stream-K partials hold one [128 x token-tile] fp32 tile per SM: the size
    grows with the token tile (16 .. 256 tokens) and then stays flat; up to 16
    tokens it also covers the few-token launch's partial tiles and flags."""
    sizes = [lib.fused_workspace(m) for m in (1, 16, 17, 128, 256, 4096)]
    assert sizes[0] <= sizes[1] < sizes[2] < sizes[3] < sizes[4] == sizes[5]
    assert lib.linear_workspace(2048, 4096, 4096, 16) > lib.fused_workspace(2048)


def test_workspace_grows_with_tokens(lib):
    small = lib.linear_workspace(64, 1024, 1024, 8)
    big = lib.linear_workspace(2048, 4096, 4096, 16)
    assert 0 < small < big


def test_gemm_schedule_control(lib):
    """qlora_set_gemm_schedule accepts the three documented values and rejects
    anything else with INVALID_ARG (a host-only call)."""
    so = lib.library()
    for v in (lib.SCHEDULE_SINGLE, lib.SCHEDULE_PAIR, lib.SCHEDULE_AUTO):
        assert so.qlora_set_gemm_schedule(v) == 0
    for v in (-1, 3, 1 << 20):
        assert so.qlora_set_gemm_schedule(v) == 1
    with lib.gemm_schedule(lib.SCHEDULE_PAIR):
        pass
    assert so.qlora_set_gemm_schedule(lib.SCHEDULE_AUTO) == 0


def test_argument_errors_of_the_next_scope_calls(lib):
    """The comparison second level, the fused gradient + AdamW launch and the
    failure-path self-test refuse bad arguments before any launch."""
    so = lib.library()
    SZ, P = ctypes.c_size_t, ctypes.c_void_p
    a, b, c = SZ(), SZ(), SZ()
    assert so.qlora_dqfp8_sizes(64, 256, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 0
    assert (a.value, b.value, c.value) == (64 * 128, 256, 8)        # (d, mu) per group: 8 bytes
    n1, n2, n3 = SZ(), SZ(), SZ()
    so.qlora_nf4_sizes(4096, 4096, ctypes.byref(n1), ctypes.byref(n2), ctypes.byref(n3))
    so.qlora_dqfp8_sizes(4096, 4096, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
    assert (a.value, b.value, c.value) == (n1.value, n2.value, 2 * n3.value)
    q = _nf4(16, 64)
    assert so.qlora_dqfp8_quantize(None, ctypes.byref(q), None, None) == 1
    q4 = _nf4(16, 64, s2=0x30004)                                    # 4-byte but not 8-byte aligned
    assert so.qlora_dqfp8_quantize(P(0x40000), ctypes.byref(q4), None, None) == 3
    assert so.qlora_dqfp8_dequantize(ctypes.byref(q4), P(0x40000), None) == 3
    assert so.qlora_dqfp8_dequantize(ctypes.byref(q), None, None) == 1
    # fused gradients + AdamW
    from bit_nf4_quantized_dequant_b200._binding import _Adam8
    st = _Adam8(0x100000, 0, 0x110000, 0x120000, 0x130000, 0x140000)
    X, dY, sU, sT = P(0x50000), P(0x60000), P(0x70000), P(0x80000)
    g = so.qlora_lora_grads_adamw8
    args = lambda **k: dict(dict(r=16, A=ctypes.byref(st), B=ctypes.byref(st), step=1, lr=1e-4, b1=0.9, b2=0.999,
                                 eps=1e-8), **k)
    call = lambda d: g(X, dY, 64, 256, 128, sU, sT, d["r"], None, None, d["A"], d["B"], d["step"], d["lr"],
                       d["b1"], d["b2"], d["eps"], 0.0, None)
    assert call(args(A=None)) == 1
    assert call(args(step=0)) == 1
    assert call(args(b1=1.0)) == 1
    assert call(args(eps=0.0)) == 1
    assert call(args(r=12)) == 2
    bad = _Adam8(0x100000, 0, 0, 0x120000, 0x130000, 0x140000)       # missing m_q
    assert call(args(B=ctypes.byref(bad))) == 1
    # self-test
    assert so.qlora_selftest_bounded_wait(None, None) == 1
    assert so.qlora_selftest_bounded_wait(P(0x50002), None) == 3
