"""GPU parity on the full-size workloads beyond the attention projection: the
Llama-7B SiLU-gated MLP chain with the forward recomputed before the backward,
one layer of the 3B decoder stack, the 8B linear shapes at 4096 tokens and at
8 tokens, and the standalone dequantisation of the 8B shapes.

"QLoRA, in depth", section "The mechanism in brief": the layer dequantises W
to bf16 on every forward (and again when the forward is recomputed) and its
backward gives dX, dA and dB, never dW. Tolerances as in test_gpu_linear
(relative Frobenius error <= 5e-3, per-element |err| <= 1e-2 max|ref|); the
codec is compared bit for bit.

Where the oracle cannot afford the whole product in float64, it is checked on
sampled outputs that it computes exactly: 64 seeded output columns of Y (from
the dequantised rows of W), 64 seeded columns of dX in 4 NF4 block-columns
(from the dequantised columns of W), and dA, dB, sU in full (they are thin).
"""

import numpy as np
import pytest

from oracle import linear as olin, nf4 as onf4
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import assert_close_fp, bf16_dev_bits, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _f64(bits):
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


def _bf16r(x):
    """Round float64 values to bf16 (the compute dtype at the harness's
    boundaries between layers) and back to float64."""
    return onf4.bf16_bits_to_f64(onf4.bf16_round_bits(np.asarray(x, dtype=np.float64).astype(np.float32)))


def _sampled_linear(lib, N, K, M, r, alpha, index):
    """fwd + bwd of one full-size linear against the oracle on sampled outputs."""
    import torch
    s = alpha / r
    c = inputs.linear_case(N, K, M, r, index=index)
    q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    X, A, B, dY = (to_dev_bf16(c[k]) for k in ("X", "A", "B", "dY"))
    Y, sU = lib.linear_fwd(q, X, A, B, s)
    dX, dA, dB = lib.linear_bwd(q, X, A, B, s, dY, sU=sU)
    torch.cuda.synchronize()
    g = inputs.rng(1000 + index)
    ns = np.sort(g.choice(N, size=min(64, N), replace=False))
    # 64 dX columns from 4 NF4 block-columns, so that the oracle encodes only those
    kb = np.sort(g.choice(K // 64, size=4, replace=False))
    ks = np.sort((kb[:, None] * 64 + np.stack([g.choice(64, size=16, replace=False) for _ in kb])).reshape(-1))
    Xh, Ah, Bh, dYh = (_f64(c[k]) for k in ("X", "A", "B", "dY"))
    U = Xh @ Ah.T
    T = dYh @ Bh
    Wr = onf4.dequantize_rows(c["W"], ns)
    Wc = onf4.dequantize_cols(c["W"], ks)
    tag = f"{N}x{K} M={M}"
    assert_close_fp(bf16_dev_to_f64(Y)[:, ns], Xh @ Wr.T + s * U @ Bh[ns].T, f"Y cols ({tag})")
    assert_close_fp(bf16_dev_to_f64(sU), s * U, f"sU ({tag})")
    assert_close_fp(bf16_dev_to_f64(dX)[:, ks], dYh @ Wc + s * T @ Ah[:, ks], f"dX cols ({tag})")
    assert_close_fp(dA.cpu().numpy(), s * (T.T @ Xh), f"dA ({tag})")
    assert_close_fp(dB.cpu().numpy(), s * (dYh.T @ U), f"dB ({tag})")


LAYER_3B = [(3072, 3072), (1024, 3072), (8192, 3072), (3072, 8192)]   # q/o, k/v, gate/up, down


@pytest.mark.parametrize("N,K", LAYER_3B)
def test_stack_3b_layer_shapes(lib, N, K):
    """3B decoder stack (hidden 3072, kv 1024, MLP 8192), 2048 tokens, r=16,
    alpha=32: every distinct linear shape of a layer."""
    _sampled_linear(lib, N, K, 2048, 16, 32.0, index=40 + LAYER_3B.index((N, K)))


LAYER_8B = [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]   # q/o, k/v, gate/up, down


@pytest.mark.parametrize("N,K", LAYER_8B)
def test_set_8b_shapes_4096_tokens(lib, N, K):
    """8B linear set (hidden 4096, kv 1024, MLP 14336) fwd+bwd at 4096 tokens."""
    _sampled_linear(lib, N, K, 4096, 16, 32.0, index=50 + LAYER_8B.index((N, K)))


@pytest.mark.parametrize("N,K", LAYER_8B)
def test_set_8b_shapes_8_tokens(lib, N, K):
    """8B linear set forward at 8 tokens (one launch per linear): Y on 64
    sampled output columns and sU in full."""
    import torch
    M, r, s = 8, 16, 2.0
    c = inputs.linear_case(N, K, M, r, index=60 + LAYER_8B.index((N, K)))
    q = lib.nf4_quantize(torch.from_numpy(c["W"]).cuda())
    X, A, B = (to_dev_bf16(c[k]) for k in ("X", "A", "B"))
    Y, sU = lib.linear_fwd(q, X, A, B, s)
    torch.cuda.synchronize()
    ns = np.sort(inputs.rng(1100 + N + K).choice(N, size=64, replace=False))
    Xh, Ah, Bh = (_f64(c[k]) for k in ("X", "A", "B"))
    U = Xh @ Ah.T
    Wr = onf4.dequantize_rows(c["W"], ns)
    assert_close_fp(bf16_dev_to_f64(Y)[:, ns], Xh @ Wr.T + s * U @ Bh[ns].T, "Y cols")
    assert_close_fp(bf16_dev_to_f64(sU), s * U, "sU")


@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_set_8b_dequant_bit_exact_on_sampled_rows(lib, N, K):
    """Standalone quantise + dequantise of full-size 8B MLP weights: packed
    codes and block constants of 32 sampled rows, every second-level scale,
    and the dequantised bf16 rows, all bit for bit."""
    import torch
    W = inputs.weight_f32(N, K, index=70 + (N > K))
    q = lib.nf4_quantize(torch.from_numpy(W).cuda())
    Wd = lib.nf4_dequantize(q)
    torch.cuda.synchronize()
    rows = np.sort(inputs.rng(1200 + N).choice(N, size=32, replace=False))
    pr, s8r, s2 = onf4.quantize_rows(W, rows)
    codes = q.codes.cpu().numpy().reshape(N, K // 2)
    scale8 = q.scale8.cpu().numpy().reshape(N, K // 64)
    np.testing.assert_array_equal(codes[rows], pr)
    np.testing.assert_array_equal(scale8[rows], s8r)
    np.testing.assert_array_equal(q.scale2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    ref_bits = onf4.bf16_round_bits(onf4.dequantize_rows(W, rows).astype(np.float32))
    np.testing.assert_array_equal(bf16_dev_bits(Wd)[rows], ref_bits)


@pytest.fixture(scope="module")
def mlp_7b():
    """Inputs and the float64 oracle of the Llama-7B SiLU-gated MLP chain
    (gate/up 4096->11008, down 11008->4096), 4096 tokens, r=16, alpha=32,
    computed once for the unfused and the fused chain. The oracle rounds to
    bf16 at the layer boundaries the kernels round at (g, u, h, dH, dg, du)."""
    H, Fd, M, r, alpha = 4096, 11008, 4096, 16, 32.0
    s = alpha / r

    def case(N, K, index):   # only the inputs the chain uses
        return dict(W=inputs.weight_f32(N, K, index), A=inputs.lora_a_bf16(r, K, index),
                    B=inputs.lora_b_bf16(N, r, index))
    cg, cu, cd = case(Fd, H, 80), case(Fd, H, 81), case(H, Fd, 82)
    X, dY = inputs.activations_bf16(M, H, 80), inputs.grad_out_bf16(M, H, 82)
    Wg, Wu, Wd = (onf4.dequantize(*onf4.quantize(c["W"]), *c["W"].shape) for c in (cg, cu, cd))
    Xh, dYh = _f64(X), _f64(dY)
    (Ag, Bg), (Au, Bu), (Ad, Bd) = ((_f64(c["A"]), _f64(c["B"])) for c in (cg, cu, cd))
    go = _bf16r(olin.linear_fwd(Wg, Xh, Ag, Bg, s)[0])
    uo = _bf16r(olin.linear_fwd(Wu, Xh, Au, Bu, s)[0])
    silu = go / (1.0 + np.exp(-go))
    ho = _bf16r(silu * uo)
    yo = olin.linear_fwd(Wd, ho, Ad, Bd, s)[0]
    dho, dAdo, dBdo = olin.linear_bwd(Wd, ho, Ad, Bd, s, dYh)
    dho = _bf16r(dho)
    sg = 1.0 / (1.0 + np.exp(-go))
    dgo = _bf16r(dho * uo * sg * (1 + go * (1 - sg)))
    duo = _bf16r(dho * silu)
    dXgo, dAgo, dBgo = olin.linear_bwd(Wg, Xh, Ag, Bg, s, dgo)
    dXuo, dAuo, dBuo = olin.linear_bwd(Wu, Xh, Au, Bu, s, duo)
    return dict(s=s, r=r, cg=cg, cu=cu, cd=cd, X=X, dY=dY,
                ref=dict(g=go, h=ho, y=yo, dh=dho, dX=dXgo + dXuo, dAd=dAdo, dBd=dBdo, dAg=dAgo, dBg=dBgo,
                         dAu=dAuo, dBu=dBuo))


def test_mlp_7b_chain_with_recompute(lib, mlp_7b):
    """The chain through three separate QLoRA linears with the
    gradient-checkpointing pattern: the forward runs, is recomputed
    (dequantising every weight again) and must give the same bits, then the
    backward runs through SiLU(g) * u. The glue between the layers is plain
    torch in bf16."""
    import torch
    import torch.nn.functional as F
    d, s = mlp_7b, mlp_7b["s"]
    cg, cu, cd = d["cg"], d["cu"], d["cd"]
    X = to_dev_bf16(d["X"])
    dY = to_dev_bf16(d["dY"])
    qs, lora = [], []
    for c in (cg, cu, cd):
        qs.append(lib.nf4_quantize(torch.from_numpy(c["W"]).cuda()))
        lora.append((to_dev_bf16(c["A"]), to_dev_bf16(c["B"])))

    def forward():
        g, sUg = lib.linear_fwd(qs[0], X, *lora[0], s)
        u, sUu = lib.linear_fwd(qs[1], X, *lora[1], s)
        h = (F.silu(g.float()) * u.float()).bfloat16()
        y, sUd = lib.linear_fwd(qs[2], h, *lora[2], s)
        return g, u, h, y, (sUg, sUu, sUd)

    g, u, h, y, sUs = forward()
    g2, u2, h2, y2, _ = forward()          # recompute before the backward
    torch.cuda.synchronize()
    for a, b in ((g, g2), (u, u2), (h, h2), (y, y2)):
        assert torch.equal(a, b)
    dh, dAd, dBd = lib.linear_bwd(qs[2], h2, *lora[2], s, dY, sU=sUs[2])
    gf, uf, dhf = g2.float(), u2.float(), dh.float()
    sig = torch.sigmoid(gf)
    dg = (dhf * uf * sig * (1 + gf * (1 - sig))).bfloat16()
    du = (dhf * F.silu(gf)).bfloat16()
    dXg, dAg, dBg = lib.linear_bwd(qs[0], X, *lora[0], s, dg, sU=sUs[0])
    dXu, dAu, dBu = lib.linear_bwd(qs[1], X, *lora[1], s, du, sU=sUs[1])
    dX = dXg.float() + dXu.float()
    torch.cuda.synchronize()
    ref = d["ref"]
    assert_close_fp(bf16_dev_to_f64(g), ref["g"], "gate output")
    assert_close_fp(bf16_dev_to_f64(h), ref["h"], "SiLU(g) * u")
    assert_close_fp(bf16_dev_to_f64(y), ref["y"], "MLP output")
    assert_close_fp(bf16_dev_to_f64(dh), ref["dh"], "dH")
    assert_close_fp(dX.double().cpu().numpy(), ref["dX"], "dX")
    for name, got in (("dAd", dAd), ("dBd", dBd), ("dAg", dAg), ("dBg", dBg), ("dAu", dAu), ("dBu", dBu)):
        assert_close_fp(got.cpu().numpy(), ref[name], name)


def test_mlp_7b_chain_fused_swiglu(lib, mlp_7b):
    """The same chain with gate and up fused: one GEMM over the interleaved
    NF4 weight writes h = silu(g) * u, the recompute repeats it (same bits),
    and the backward's fused GEMM recomputes g and u to write dg and du; dX
    and the adapter gradients follow from the existing kernels over the fused
    operands. Checked against the same oracle chain."""
    import torch
    d, s, r = mlp_7b, mlp_7b["s"], mlp_7b["r"]
    cg, cu, cd = d["cg"], d["cu"], d["cd"]
    X = to_dev_bf16(d["X"])
    dY = to_dev_bf16(d["dY"])
    M, K = X.shape
    Fd = cg["W"].shape[0]
    qgu = lib.nf4_quantize(lib.swiglu_interleave(torch.from_numpy(cg["W"]), torch.from_numpy(cu["W"])).cuda())
    qd = lib.nf4_quantize(torch.from_numpy(cd["W"]).cuda())
    Agu = to_dev_bf16(np.concatenate([cg["A"], cu["A"]]))
    Bgu = lib.swiglu_pack_b(to_dev_bf16(cg["B"]), to_dev_bf16(cu["B"]))
    Ad, Bd = to_dev_bf16(cd["A"]), to_dev_bf16(cd["B"])
    ws = torch.zeros(lib.linear_workspace(M, 2 * Fd, K, 2 * r), dtype=torch.uint8, device="cuda")
    sUgu = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
    lib.lora_xa(X, Agu, s, sUgu, ws)
    h = lib.swiglu_fwd(qgu, X, Bgu, sUgu)
    y, sUd = lib.linear_fwd(qd, h, Ad, Bd, s)
    h2 = lib.swiglu_fwd(qgu, X, Bgu, sUgu)        # recompute before the backward
    torch.cuda.synchronize()
    assert torch.equal(h, h2)
    dh, dAd, dBd = lib.linear_bwd(qd, h2, Ad, Bd, s, dY, sU=sUd)
    dGU = lib.swiglu_bwd(qgu, X, Bgu, sUgu, dh)
    sTgu = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
    lib.lora_dyb(dGU, Bgu, s, sTgu, ws)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    lib.fused_dx(qgu, dGU, Agu, sTgu, dX)
    dAgu = torch.empty((2 * r, K), dtype=torch.float32, device="cuda")
    dBgu = torch.empty((2 * Fd, 2 * r), dtype=torch.float32, device="cuda")
    lib.lora_grads(X, dGU, sUgu, sTgu, dAgu, dBgu, ws)
    dBg, dBu = lib.swiglu_unpack_db(dBgu)
    torch.cuda.synchronize()
    ref = d["ref"]
    assert_close_fp(bf16_dev_to_f64(h), ref["h"], "SiLU(g) * u (fused)")
    assert_close_fp(bf16_dev_to_f64(y), ref["y"], "MLP output")
    assert_close_fp(bf16_dev_to_f64(dh), ref["dh"], "dH")
    assert_close_fp(bf16_dev_to_f64(dX), ref["dX"], "dX (fused)")
    dA = dAgu.cpu().numpy()
    for name, got in (("dAd", dAd.cpu().numpy()), ("dBd", dBd.cpu().numpy()), ("dAg", dA[:r]), ("dAu", dA[r:]),
                      ("dBg", dBg.cpu().numpy()), ("dBu", dBu.cpu().numpy())):
        assert_close_fp(got, ref[name], name + " (fused)")
