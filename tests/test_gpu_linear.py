"""GPU parity of the fused QLoRA linear forward and backward against the fp64
oracle ("QLoRA, in depth", "The mechanism in brief": y = W x + (alpha/r) B A x;
backward gives dX, dA and dB, never dW). Tolerance: relative Frobenius error
<= 5e-3 and per-element |err| <= 1e-2 max|ref| (see helpers.py)."""

import numpy as np
import pytest

from oracle import linear as olin, nf4 as onf4
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import assert_close_fp, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _setup(lib, N, K, M, r, index=0, outliers=False):
    import torch
    c = inputs.linear_case(N, K, M, r, index=index, outliers=outliers)
    q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    codes, s8, s2 = onf4.quantize(c["W"])
    Wd = onf4.dequantize(codes, s8, s2, N, K)
    f = lambda b: inputs.bf16_bits_to_f32(b).astype(np.float64)
    host = dict(Wd=Wd, X=f(c["X"]), A=f(c["A"]), B=f(c["B"]), dY=f(c["dY"]))
    dev = dict(q=q, X=to_dev_bf16(c["X"]), A=to_dev_bf16(c["A"]), B=to_dev_bf16(c["B"]), dY=to_dev_bf16(c["dY"]))
    return host, dev


CASES = [
    # N, K, M, r, alpha
    (1024, 1024, 64, 8, 16.0),     # single linear 1024x1024, 64 tokens, r=8, alpha=16
    (272, 320, 100, 16, 32.0),     # ragged rows, tokens and K tiles
    (128, 64, 1, 8, 16.0),         # one token, one K block
    (64, 192, 33, 24, 48.0),       # r not a multiple of 16
    (256, 512, 300, 32, 64.0),     # two token tiles, the second ragged
    (160, 256, 17, 64, 64.0),      # largest rank
    (512, 1024, 8, 16, 32.0),      # decode-sized token count
    (384, 2048, 520, 16, 32.0),    # several row tiles x three token tiles
]


@pytest.mark.parametrize("N,K,M,r,alpha", CASES)
def test_forward_backward_parity(lib, N, K, M, r, alpha):
    import torch
    s = alpha / r
    h, d = _setup(lib, N, K, M, r)
    Y, sU = lib.linear_fwd(d["q"], d["X"], d["A"], d["B"], s)
    dX, dA, dB = lib.linear_bwd(d["q"], d["X"], d["A"], d["B"], s, d["dY"], sU=sU)
    torch.cuda.synchronize()
    Yr, U = olin.linear_fwd(h["Wd"], h["X"], h["A"], h["B"], s)
    dXr, dAr, dBr = olin.linear_bwd(h["Wd"], h["X"], h["A"], h["B"], s, h["dY"])
    assert_close_fp(bf16_dev_to_f64(Y), Yr, "Y")
    assert_close_fp(bf16_dev_to_f64(sU), s * U, "sU")
    assert_close_fp(bf16_dev_to_f64(dX), dXr, "dX")
    assert_close_fp(dA.cpu().numpy(), dAr, "dA")
    assert_close_fp(dB.cpu().numpy(), dBr, "dB")


def test_backward_recompute_and_skip_paths(lib):
    """sU omitted -> recomputed bit-identically; dX omitted -> dA/dB unchanged."""
    import torch
    N, K, M, r, s = 256, 512, 96, 16, 2.0
    _, d = _setup(lib, N, K, M, r, index=2)
    Y, sU = lib.linear_fwd(d["q"], d["X"], d["A"], d["B"], s)
    dX1, dA1, dB1 = lib.linear_bwd(d["q"], d["X"], d["A"], d["B"], s, d["dY"], sU=sU)
    dX2, dA2, dB2 = lib.linear_bwd(d["q"], d["X"], d["A"], d["B"], s, d["dY"], sU=None)
    _, dA3, dB3 = lib.linear_bwd(d["q"], d["X"], d["A"], d["B"], s, d["dY"], sU=sU, want_dX=False)
    torch.cuda.synchronize()
    assert torch.equal(dX1, dX2)
    for a, b in ((dA1, dA2), (dB1, dB2), (dA1, dA3), (dB1, dB3)):
        assert torch.equal(a, b)


def test_zero_lora_up_reduces_to_plain_gemm(lib):
    """B = 0: Y must equal X W'^T; compared with torch's bf16 matmul on the
    library's own dequantised weight (a library routine), within tolerance."""
    import torch
    N, K, M, r = 512, 1024, 256, 16
    _, d = _setup(lib, N, K, M, r, index=3)
    Bz = torch.zeros_like(d["B"])
    Y, _ = lib.linear_fwd(d["q"], d["X"], d["A"], Bz, 2.0)
    Wd = lib.nf4_dequantize(d["q"])
    ref = torch.matmul(d["X"].float(), Wd.float().T)
    torch.cuda.synchronize()
    assert_close_fp(bf16_dev_to_f64(Y), ref.double().cpu().numpy(), "Y(B=0)")


def test_attention_projection_full_size_sampled(lib):
    """4096x4096 with 0.1% x8 outliers, 2048 tokens, r=16, alpha=32, in the
    launch configuration the benchmark times. Y and dX on 64 seeded rows; sU,
    dA and dB in full."""
    import torch
    N = K = 4096
    M, r, s = 2048, 16, 2.0
    h, d = _setup(lib, N, K, M, r, outliers=True)
    Y, sU = lib.linear_fwd(d["q"], d["X"], d["A"], d["B"], s)
    dX, dA, dB = lib.linear_bwd(d["q"], d["X"], d["A"], d["B"], s, d["dY"], sU=sU)
    torch.cuda.synchronize()
    rows = np.sort(inputs.rng(77).choice(M, size=64, replace=False))
    Yr = olin.linear_fwd_rows(h["Wd"], h["X"][rows], h["A"], h["B"], s)
    dXr = olin.linear_dx_rows(h["Wd"], h["dY"][rows], h["A"], h["B"], s)
    assert_close_fp(bf16_dev_to_f64(Y)[rows], Yr, "Y rows")
    assert_close_fp(bf16_dev_to_f64(dX)[rows], dXr, "dX rows")
    U = h["X"] @ h["A"].T
    T = h["dY"] @ h["B"]
    assert_close_fp(bf16_dev_to_f64(sU), s * U, "sU")
    assert_close_fp(dA.cpu().numpy(), s * (T.T @ h["X"]), "dA")
    assert_close_fp(dB.cpu().numpy(), s * (h["dY"].T @ U), "dB")


def test_no_timeout_status(lib):
    import torch
    N, K, M, r = 256, 256, 64, 16
    _, d = _setup(lib, N, K, M, r, index=4)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.linear_fwd(d["q"], d["X"], d["A"], d["B"], 2.0, status=st)
    lib.linear_bwd(d["q"], d["X"], d["A"], d["B"], 2.0, d["dY"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


# Shapes for the two schedules of the fused GEMMs: tiles split over many CTAs
# (fewer tiles than SMs), a ragged second wave (more tiles than SMs), decode.
# With a workspace, token tiles of at most 64 (M <= 64) take the stream-K path.
SCHEDULE_CASES = [
    # N, K, M, r
    (2048, 1024, 300, 16),    # whole tiles: 32 FWD tiles of 16 K-steps
    (2560, 256, 4000, 16),    # whole tiles: 320 FWD tiles, a ragged second wave; pairs: 80 FWD
                              # pair tiles of 256 rows x 512 tokens, ragged last token tile
    (4032, 512, 1100, 8),     # pairs: the last FWD pair tile's odd CTA holds 64 rows
    (512, 4096, 1100, 32),    # pairs: 16 DX pair tiles of 256 dX columns, rank 32
    (256, 4608, 1500, 64),    # pairs: rank 64 (the LoRA slices at 128-row offsets)
    (4096, 512, 8, 16),       # stream-K: each tile cut between about five CTAs
    (512, 4096, 64, 16),      # stream-K: 4 FWD tiles of 64 K-steps, ~37 CTAs per tile, more
                              # partials than fit in shared memory
    (1024, 256, 40, 32),      # stream-K: ragged token tile, 8 FWD / 2 DX tiles
]


@pytest.mark.parametrize("N,K,M,r", SCHEDULE_CASES)
def test_fused_gemm_whole_tile_and_stream_k(lib, N, K, M, r):
    """qlora_fused_fwd / qlora_fused_dx with the automatic schedule, forced to
    single-CTA whole tiles, with a workspace (stream-K for short token tiles,
    partial tiles summed through the workspace) and forced to CTA pairs
    (cta_group::2) all match the oracle; they differ only in fp32 summation
    order."""
    import torch
    s = 2.0
    h, d = _setup(lib, N, K, M, r, index=5)
    U = h["X"] @ h["A"].T
    T = h["dY"] @ h["B"]
    sU = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    sT = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    lws = torch.zeros(lib.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")
    lib.lora_xa(d["X"], d["A"], s, sU, lws)
    lib.lora_dyb(d["dY"], d["B"], s, sT, lws)
    gws = torch.full((lib.fused_workspace(M),), 0xAB, dtype=torch.uint8, device="cuda")
    gws[:256].zero_()   # the counter page starts at zero; the rest needs no initialisation
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = {}
    for name, ws, schedule in (("auto", None, lib.SCHEDULE_AUTO), ("single", None, lib.SCHEDULE_SINGLE),
                               ("streamk", gws, lib.SCHEDULE_AUTO), ("pair", None, lib.SCHEDULE_PAIR)):
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dX = torch.full((M, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        with lib.gemm_schedule(schedule):
            lib.fused_fwd(d["q"], d["X"], d["B"], sU, Y, status=st, ws=ws)
            lib.fused_dx(d["q"], d["dY"], d["A"], sT, dX, status=st, ws=ws)
        out[name] = (Y, dX)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Yr = olin.linear_fwd(h["Wd"], h["X"], h["A"], h["B"], s)[0]
    dXr = h["dY"] @ h["Wd"] + s * (T @ h["A"])
    for name, (Y, dX) in out.items():
        assert_close_fp(bf16_dev_to_f64(Y), Yr, f"Y ({name})")
        assert_close_fp(bf16_dev_to_f64(dX), dXr, f"dX ({name})")


def test_stream_k_graph_replays(lib):
    """A CUDA graph replays the stream-K forward with the same launch values
    each time, so the flags in the workspace must be cleared by the kernel that
    consumed them: three replays on changing inputs each match the oracle."""
    import torch
    N, K, M, r, s = 2048, 512, 40, 16, 2.0
    h, d = _setup(lib, N, K, M, r, index=6)
    sU = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    lws = torch.zeros(lib.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")
    gws = torch.zeros(lib.fused_workspace(M), dtype=torch.uint8, device="cuda")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    X = d["X"].clone()
    lib.lora_xa(X, d["A"], s, sU, lws)
    lib.fused_fwd(d["q"], X, d["B"], sU, Y, ws=gws)    # warm-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lib.lora_xa(X, d["A"], s, sU, lws)
        lib.fused_fwd(d["q"], X, d["B"], sU, Y, ws=gws)
    for rep in range(3):
        c = inputs.linear_case(N, K, M, r, index=10 + rep)
        X.copy_(to_dev_bf16(c["X"]))
        Y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        Xh = inputs.bf16_bits_to_f32(c["X"]).astype(np.float64)
        Yr = olin.linear_fwd(h["Wd"], Xh, h["A"], h["B"], s)[0]
        assert_close_fp(bf16_dev_to_f64(Y), Yr, f"Y (replay {rep})")
    del g


# Few-token forwards take the persistent weight-streaming kernel (codes,
# activations and block constants through a shared-memory ring, warp-level MMAs,
# tiles split between CTAs). The block constants come by TMA when a row's 8-bit
# constants are a multiple of 16 bytes and a chunk's second-level constants fit
# one 256-entry window (at most 480 blocks a row), else by cp.async.
FEW_TOKEN_CASES = [
    # N, K, M, r
    (1024, 7168, 5, 16),    # 112 blocks a row: constants by TMA
    (512, 4096, 16, 32),    # 16 tokens (two MMA token tiles)
    (2048, 1024, 9, 8),     # second token tile nearly empty
    (64, 192, 3, 64),       # one tile, three blocks (byte-wise constants), largest rank
    (256, 32768, 8, 16),    # 512 blocks a row: constants by cp.async; 256 pieces of X A^T
    (384, 11008, 7, 24),    # 172 blocks a row (not a multiple of 16): cp.async; rank 24
]


@pytest.mark.parametrize("N,K,M,r", FEW_TOKEN_CASES)
def test_few_token_forward(lib, N, K, M, r):
    import torch
    s = 2.0
    h, d = _setup(lib, N, K, M, r, index=7)
    Y, sU = lib.linear_fwd(d["q"], d["X"], d["A"], d["B"], s)
    torch.cuda.synchronize()
    Yr, U = olin.linear_fwd(h["Wd"], h["X"], h["A"], h["B"], s)
    assert_close_fp(bf16_dev_to_f64(sU), s * U, "sU")
    assert_close_fp(bf16_dev_to_f64(Y), Yr, "Y")


def test_bounded_wait_reports_timeout_and_context_survives(lib):
    """A kernel wait that can never complete (qlora_selftest_bounded_wait)
    gives up after the library's limit, writes QLORA_ERR_TIMEOUT to the
    device status and returns; the same context then runs a linear forward
    that matches the oracle."""
    import time
    import torch
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.time()
    lib.selftest_bounded_wait(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 6                      # QLORA_ERR_TIMEOUT
    assert time.time() - t0 < 30
    N, K, M, r, s = 256, 512, 40, 16, 2.0
    h, d = _setup(lib, N, K, M, r, index=11)
    Y, sU = lib.linear_fwd(d["q"], d["X"], d["A"], d["B"], s)
    torch.cuda.synchronize()
    Yr, _ = olin.linear_fwd(h["Wd"], h["X"], h["A"], h["B"], s)
    assert_close_fp(bf16_dev_to_f64(Y), Yr, "Y after the timeout")
