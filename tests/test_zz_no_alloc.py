"""The allocation-free forward, qlora_linear_fwd_noalloc, for callers that
cannot allocate device memory where they run the layer (a plug-in that only
receives inputs and outputs, a server whose device memory is all in a fixed
pool, code that must not call cudaMalloc between launches because that call
can synchronise the device). Its scratch is a fixed 8 MiB array inside the
library, shared by every call and keeping the previous call's contents, so the
tests make calls in a row with different inputs and check each one against
the oracle and, bit for bit, against the ordinary workspace-taking
qlora_linear_fwd, which runs the same launches.

This file is collected last on purpose; it also passes alone in a fresh
process (the `lib` fixture builds and loads the library).
"""

import ctypes

import numpy as np
import pytest

from oracle import linear as olin, nf4 as onf4
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import assert_close_fp, bf16_dev_bits, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, X, A, B, r, s, Y, sU, M=None):
    import torch
    st = q.c_struct()
    ptr = lambda t: None if t is None else ctypes.c_void_p(t if isinstance(t, int) else t.data_ptr())
    return lib.library().qlora_linear_fwd_noalloc(
        ctypes.byref(st), ptr(X), X.shape[0] if M is None else M, ptr(A), ptr(B), r, s, ptr(Y), ptr(sU), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(lib, N, K, M, r, index):
    import torch
    c = inputs.linear_case(N, K, M, r, index=index)
    q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    Wd = onf4.dequantize(*onf4.quantize(c["W"]), N, K)
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    ref = olin.linear_fwd(Wd, f(c["X"]), f(c["A"]), f(c["B"]), 2.0)
    return q, to_dev_bf16(c["X"]), to_dev_bf16(c["A"]), to_dev_bf16(c["B"]), ref


@pytest.mark.parametrize("M", [300, 40, 12])
def test_noalloc_forward_matches_oracle_and_workspace_forward(lib, M):
    """Two calls in a row (sU kept by the caller, then left in the scratch)
    at 300 tokens (whole GEMM tiles), 40 tokens (stream-K partials in the
    scratch) and 12 tokens (the few-token launch, all its scratch there)."""
    import torch
    N, K, r, s = 1024, 2048, 16, 2.0
    for call in (0, 1):
        q, X, A, B, (Yr, U) = _case(lib, N, K, M, r, index=call + 3 * M)
        Y_ref, sU_ref = lib.linear_fwd(q, X, A, B, s)
        Y = torch.full_like(Y_ref, float("nan"))
        sU = torch.full_like(sU_ref, float("nan")) if call == 0 else None
        assert _call_noalloc(lib, q, X, A, B, r, s, Y, sU) == 0
        torch.cuda.synchronize()
        assert_close_fp(bf16_dev_to_f64(Y), Yr, f"Y (call {call})")
        assert np.array_equal(bf16_dev_bits(Y), bf16_dev_bits(Y_ref)), f"Y bits (call {call})"
        if sU is not None:
            assert_close_fp(bf16_dev_to_f64(sU), s * U, "sU")
            assert np.array_equal(bf16_dev_bits(sU), bf16_dev_bits(sU_ref))


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    """Just over the limit: beyond 16 tokens and at more than 64 the scratch
    is the 256-byte counter page plus round_up(M * r * 2, 256) for sU when the
    caller does not keep it. 65,600 tokens at rank 64 need 8,397,056 bytes >
    8 MiB; 65,534 tokens need exactly 8 MiB. Every pointer is a real device
    buffer, so even a regression that launched would compute on valid memory;
    the call must refuse before launching."""
    import torch
    N = K = 1024
    M, r = 65600, 64
    c = inputs.linear_case(N, K, 1, r, index=9)
    q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((r, K), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, q, X, A, B, r, 2.0, Y, None) == 4   # QLORA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((Y[:: 4099] == 7.0).all())                        # nothing was written
    assert _call_noalloc(lib, q, X, A, B, r, 2.0, Y, None, M=65535) == 4
    assert _call_noalloc(lib, q, X, A, B, r, 2.0, Y, None, M=65534) == 0
    torch.cuda.synchronize()


def test_noalloc_validates_everything_before_launching(lib):
    """A misaligned Y or a weight whose rows are not a multiple of 16 is
    refused before any kernel runs: the caller's sU buffer stays untouched."""
    import torch
    N, K, M, r = 256, 512, 40, 16
    q, X, A, B, _ = _case(lib, N, K, M, r, index=11)
    sU = torch.full((M, r), 7.0, dtype=torch.bfloat16, device="cuda")
    Ybuf = torch.empty(M * N + 8, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, q, X, A, B, r, 2.0, Ybuf.data_ptr() + 2, sU, M=M) == 3   # QLORA_ERR_MISALIGNED
    c = inputs.linear_case(24, K, 1, r, index=12)
    q24 = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    Y24 = torch.empty((M, 24), dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, q24, X, A, B, r, 2.0, Y24, sU) == 2                      # UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert bool((sU == 7.0).all())
