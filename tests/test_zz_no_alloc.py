"""The allocation-free forward, qlora_linear_fwd_noalloc, for callers that
cannot allocate device memory where they run the layer (a plug-in that only
receives inputs and outputs, a server whose device memory is all in a fixed
pool, code that must not call cudaMalloc between launches). Its scratch is a
fixed array inside the library, shared by every call and keeping the previous
call's contents, so the test makes two calls in a row with different inputs
(and once with sU kept in that scratch) and checks each against the ordinary
workspace-taking qlora_linear_fwd, within the tolerance the parity tests use.

This file is collected last on purpose; it also passes alone in a fresh
process (the `lib` fixture builds and loads the library).
"""

import ctypes

import pytest

from bit_nf4_quantized_dequant_b200 import inputs

from helpers import assert_close_fp, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, X, A, B, r, s, Y, sU):
    import torch
    st = q.c_struct()
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return lib.library().qlora_linear_fwd_noalloc(
        ctypes.byref(st), ptr(X), X.shape[0], ptr(A), ptr(B), r, s, ptr(Y), ptr(sU), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_forward_matches_workspace_forward_twice(lib):
    import torch
    N, K, M, r, s = 1024, 2048, 300, 16, 2.0
    for call, index in enumerate((0, 1)):
        c = inputs.linear_case(N, K, M, r, index=index)
        q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
        X, A, B = to_dev_bf16(c["X"]), to_dev_bf16(c["A"]), to_dev_bf16(c["B"])
        Y_ref, sU_ref = lib.linear_fwd(q, X, A, B, s)
        Y = torch.full_like(Y_ref, float("nan"))
        # first call keeps sU in a caller buffer, the second leaves it in the scratch
        sU = torch.full_like(sU_ref, float("nan")) if call == 0 else None
        assert _call_noalloc(lib, q, X, A, B, r, s, Y, sU) == 0
        torch.cuda.synchronize()
        assert_close_fp(bf16_dev_to_f64(Y), bf16_dev_to_f64(Y_ref), f"Y (call {call})")
        if sU is not None:
            assert_close_fp(bf16_dev_to_f64(sU), bf16_dev_to_f64(sU_ref), "sU")


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    """A call whose scratch would exceed the fixed maximum is refused before
    anything is launched (the pointers are never dereferenced)."""
    from bit_nf4_quantized_dequant_b200._binding import _NF4
    q = _NF4(4096, 4096, 0x10000, 0x20000, 0x30000)
    P = ctypes.c_void_p
    rc = lib.library().qlora_linear_fwd_noalloc(ctypes.byref(q), P(0x40000), 1 << 22, P(0x50000), P(0x60000),
                                                64, 2.0, P(0x70000), None, None, None)
    assert rc == 4   # QLORA_ERR_WORKSPACE


def test_noalloc_few_tokens_needs_no_scratch(lib):
    """At 12 tokens the forward is one launch that forms sU itself: the
    allocation-free entry then touches no scratch at all, even for a K whose
    partial sums would not fit in it, and matches the oracle."""
    import numpy as np
    import torch
    from oracle import linear as olin, nf4 as onf4
    N, K, M, r, s = 512, 4096, 12, 16, 2.0
    c = inputs.linear_case(N, K, M, r, index=3)
    q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    X, A, B = to_dev_bf16(c["X"]), to_dev_bf16(c["A"]), to_dev_bf16(c["B"])
    Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    sU = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, q, X, A, B, r, s, Y, sU) == 0
    torch.cuda.synchronize()
    Wd = onf4.dequantize(*onf4.quantize(c["W"]), N, K)
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    Yr, U = olin.linear_fwd(Wd, f(c["X"]), f(c["A"]), f(c["B"]), s)
    assert_close_fp(bf16_dev_to_f64(Y), Yr, "Y")
    assert_close_fp(bf16_dev_to_f64(sU), s * U, "sU")
