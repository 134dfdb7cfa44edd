"""GPU parity of the few-token forward of a group of linears in one launch
(qlora_linear_fwd_group) against the fp64 oracle ("QLoRA, in depth", "The
mechanism in brief": y = W x + (alpha/r) B A x; "QLoRA and Fine-Tuning on One
Consumer GPU", "Where 24 GB goes": adapters on every attention and MLP
projection). Tolerance as everywhere for GEMM outputs: relative Frobenius
error <= 5e-3, per-element |err| <= 1e-2 max|ref| (helpers.py)."""

import numpy as np
import pytest

from oracle import linear as olin, nf4 as onf4
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import assert_close_fp, bf16_dev_bits, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _f(bits):
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


def _group(lib, shapes, M, index0=0, shared_x=False, keep_su=None, alpha=32.0):
    """Quantised weights, device inputs and the oracle's Y and sU for each
    (N, K, r) of `shapes`; problems with shared_x use the first X (same K)."""
    import torch
    probs, refs = [], []
    X0 = X0_dev = None
    for i, (N, K, r) in enumerate(shapes):
        c = inputs.linear_case(N, K, M, r, index=index0 + i)
        q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
        Wd = onf4.dequantize(*onf4.quantize(c["W"]), N, K)
        if shared_x and X0 is not None:
            xb, xd = X0, X0_dev                 # the same device buffer
        else:
            xb, xd = c["X"], to_dev_bf16(c["X"])
        if X0 is None:
            X0, X0_dev = xb, xd
        s = alpha / r
        Yr, U = olin.linear_fwd(Wd, _f(xb), _f(c["A"]), _f(c["B"]), s)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        ks = keep_su[i] if keep_su is not None else True
        sU = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device="cuda") if ks else None
        probs.append(lib.LinearProblem(q, xd, to_dev_bf16(c["A"]), to_dev_bf16(c["B"]), s, Y, sU))
        refs.append((Yr, s * U))
    return probs, refs


def _check(probs, refs):
    for i, (p, (Yr, sUr)) in enumerate(zip(probs, refs)):
        assert_close_fp(bf16_dev_to_f64(p.Y), Yr, f"Y[{i}]")
        if p.sU is not None:
            assert_close_fp(bf16_dev_to_f64(p.sU), sUr, f"sU[{i}]")


GROUPS = [
    # (shapes (N, K, r), M, shared X)
    ([(512, 1024, 16), (128, 1024, 16), (128, 1024, 16)], 8, True),     # q, k, v of one attention layer
    ([(1792, 512, 16), (1792, 512, 16)], 5, True),                      # gate, up
    ([(256, 1792, 16)], 1, False),                                      # down, one token
    ([(272, 320, 24), (48, 2048, 64), (16, 64, 8)], 12, False),         # ragged rows, K not 256-aligned, r 8..64
    ([(400, 832, 32), (144, 4160, 8)], 16, False),                      # 16 tokens, K with a short last chunk
]


@pytest.mark.parametrize("shapes,M,shared", GROUPS)
def test_group_forward_matches_oracle(lib, shapes, M, shared):
    import torch
    probs, refs = _group(lib, shapes, M, shared_x=shared)
    lib.linear_fwd_group(probs)
    torch.cuda.synchronize()
    _check(probs, refs)


def test_group_is_deterministic_and_equals_single_calls(lib):
    """Two calls give the same bits, and a group gives the bits of one call
    per linear through qlora_linear_fwd (the same launch with one problem)."""
    import torch
    shapes = [(640, 1024, 16), (128, 1024, 16), (384, 768, 32)]
    probs, _ = _group(lib, shapes, 7)
    lib.linear_fwd_group(probs)
    first = [bf16_dev_bits(p.Y).copy() for p in probs]
    lib.linear_fwd_group(probs)
    torch.cuda.synchronize()
    for a, p in zip(first, probs):
        assert np.array_equal(a, bf16_dev_bits(p.Y))
    for p, a in zip(probs, first):
        Y1, sU1 = lib.linear_fwd(p.q, p.X, p.A, p.B, p.s)
        torch.cuda.synchronize()
        assert np.array_equal(bf16_dev_bits(Y1), a)
        assert np.array_equal(bf16_dev_bits(sU1), bf16_dev_bits(p.sU))


def test_group_sU_kept_in_workspace_and_more_than_16_linears(lib):
    """sU left in the workspace for some linears, and 20 linears (two launches
    of up to 16 on the stream sharing one workspace)."""
    import torch
    shapes = [(16 * (1 + i % 5), 64 * (1 + i % 4), 8 * (1 + i % 3)) for i in range(20)]
    keep = [i % 2 == 0 for i in range(20)]
    probs, refs = _group(lib, shapes, 3, index0=40, keep_su=keep)
    lib.linear_fwd_group(probs)
    torch.cuda.synchronize()
    _check(probs, refs)


def test_group_graph_replay_with_changing_inputs(lib):
    """A captured launch replays with the same per-launch value: every flag
    and counter it used must be clear again, or the second replay would read
    the first replay's partial sums and sU."""
    import torch
    shapes = [(512, 2048, 16), (256, 2048, 16)]
    probs, _ = _group(lib, shapes, 8, shared_x=True)
    ws = torch.zeros(lib.linear_fwd_group_workspace(probs, 8), dtype=torch.uint8, device="cuda")
    arr = lib._binding._problem_array(probs)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        lib.linear_fwd_group(probs, ws=ws, arr=arr)   # warm-up outside capture
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        lib.linear_fwd_group(probs, ws=ws, arr=arr)
    for trial in range(3):
        c = inputs.activations_bf16(8, 2048, index=100 + trial)
        probs[0].X.copy_(to_dev_bf16(c))
        g.replay()
        torch.cuda.synchronize()
        xh = _f(c)
        for p in probs:
            N, K = p.q.rows, p.q.cols
            Wd = onf4.dequantize(p.q.codes.cpu().numpy(), p.q.scale8.cpu().numpy(), p.q.scale2.cpu().numpy(), N, K)
            Yr, U = olin.linear_fwd(Wd, xh, bf16_dev_to_f64(p.A), bf16_dev_to_f64(p.B), p.s)
            assert_close_fp(bf16_dev_to_f64(p.Y), Yr, f"Y replay {trial}")
            assert_close_fp(bf16_dev_to_f64(p.sU), p.s * U, f"sU replay {trial}")
    del g


def test_group_overlap_flag_sees_the_preceding_kernel(lib):
    """With QLORA_FWD_OVERLAP_PREVIOUS the launch may start streaming weights
    early, but X written by the kernel just before it on the stream must be
    the value it reads."""
    import torch
    shapes = [(1024, 1024, 16), (256, 1024, 16)]
    probs, refs = _group(lib, shapes, 8, shared_x=True)
    X_true = probs[0].X.clone()
    ws = torch.zeros(lib.linear_fwd_group_workspace(probs, 8), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        probs[0].X.zero_()
        torch.cuda.synchronize()
        probs[0].X.copy_(X_true)           # a kernel on the stream right before the forward
        lib.linear_fwd_group(probs, ws=ws, flags=lib.FWD_OVERLAP_PREVIOUS)
        torch.cuda.synchronize()
        _check(probs, refs)


def test_group_rejects_bad_arguments(lib):
    import torch
    probs, _ = _group(lib, [(128, 256, 16)], 8)
    ws = torch.zeros(lib.linear_fwd_group_workspace(probs, 8), dtype=torch.uint8, device="cuda")
    arr = lib._binding._problem_array(probs)
    L = lib.library()
    st = lambda **kw: L.qlora_linear_fwd_group(arr, kw.get("count", 1), kw.get("M", 8), kw.get("flags", 0),
                                               kw.get("ws", ws.data_ptr()), kw.get("ws_bytes", ws.numel()), None,
                                               None)
    assert st() == 0
    assert st(M=17) == 2            # beyond the few-token range
    assert st(count=0) == 1
    assert st(flags=2) == 1
    assert st(ws_bytes=ws.numel() - 1) == 4
    assert st(ws=ws.data_ptr() + 8) == 3
    torch.cuda.synchronize()
