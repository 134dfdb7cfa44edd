"""GPU parity of the fused SwiGLU projection (gate and up in one tcgen05 GEMM
over the row-interleaved NF4 weight; h = silu(g) * u in the epilogue) and of
its backward, which recomputes g and u inside the GEMM and writes dg, du.
The oracle is oracle.swiglu on the same stored NF4 weight, de-interleaved;
the rest of the backward (dX, adapter gradients) runs through the existing
kernels over the fused operands and is compared with the two separate
linears' oracle gradients. Tolerances as in test_gpu_linear."""

import numpy as np
import pytest

from oracle import linear as olin, nf4 as onf4, swiglu as osw
from bit_nf4_quantized_dequant_b200 import inputs

from helpers import assert_close_fp, bf16_dev_to_f64, to_dev_bf16

pytestmark = pytest.mark.gpu


def _f64(bits):
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


def _deinterleave(Wgu):
    """Rows of the [2F, K] interleaved matrix back to (Wg, Wu)."""
    F2, K = Wgu.shape
    v = Wgu.reshape(F2 // 128, 2, 64, K)
    return v[:, 0].reshape(F2 // 2, K), v[:, 1].reshape(F2 // 2, K)


CASES = [
    # F, K, M, r
    (128, 256, 40, 16),     # one row tile pair, ragged token tile of 64
    (576, 512, 300, 16),    # 9 gate/up tiles, two token tiles, ragged
    (256, 1024, 200, 8),    # smallest rank (2r = 16)
    (192, 320, 17, 32),     # largest rank (2r = 64), 5 K blocks per row (groups straddle rows)
]


@pytest.mark.parametrize("F,K,M,r", CASES)
def test_swiglu_fused_forward_and_backward(lib, F, K, M, r):
    import torch
    s = 2.0
    g = inputs.rng(300 + F + K + M + r)
    Wg = (g.standard_normal((F, K)) * 0.02).astype(np.float32)
    Wu = (g.standard_normal((F, K)) * 0.02).astype(np.float32)
    bf = lambda a: onf4.bf16_round_bits(a.astype(np.float32))
    X = bf(g.standard_normal((M, K)))
    Ag, Au = bf(g.standard_normal((r, K)) / r), bf(g.standard_normal((r, K)) / r)
    Bg, Bu = bf(g.standard_normal((F, r)) * 0.01), bf(g.standard_normal((F, r)) * 0.01)
    dH = bf(g.standard_normal((M, F)))

    Wgu32 = lib.swiglu_interleave(torch.from_numpy(Wg), torch.from_numpy(Wu))
    q = lib.nf4_quantize(Wgu32.cuda())
    Xd, dHd = to_dev_bf16(X), to_dev_bf16(dH)
    Agu = to_dev_bf16(np.concatenate([Ag, Au]))
    Bgu = lib.swiglu_pack_b(to_dev_bf16(Bg), to_dev_bf16(Bu))
    ws = torch.zeros(lib.linear_workspace(M, 2 * F, K, 2 * r), dtype=torch.uint8, device="cuda")
    sUgu = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
    lib.lora_xa(Xd, Agu, s, sUgu, ws)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    H = lib.swiglu_fwd(q, Xd, Bgu, sUgu, status=st)
    dGU = lib.swiglu_bwd(q, Xd, Bgu, sUgu, dHd, status=st)
    sTgu = torch.empty((M, 2 * r), dtype=torch.bfloat16, device="cuda")
    lib.lora_dyb(dGU, Bgu, s, sTgu, ws)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    lib.fused_dx(q, dGU, Agu, sTgu, dX, status=st)
    dAgu = torch.empty((2 * r, K), dtype=torch.float32, device="cuda")
    dBgu = torch.empty((2 * F, 2 * r), dtype=torch.float32, device="cuda")
    lib.lora_grads(Xd, dGU, sUgu, sTgu, dAgu, dBgu, ws)
    dBg, dBu = lib.swiglu_unpack_db(dBgu)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    # oracle on the same stored weight
    Wgu_d = onf4.dequantize(*onf4.quantize(Wgu32.numpy()), 2 * F, K)
    Wgd, Wud = _deinterleave(Wgu_d)
    Xh, Agh, Auh, Bgh, Buh, dHh = (onf4.bf16_bits_to_f64(a) for a in (X, Ag, Au, Bg, Bu, dH))
    Ho, Go, Uo = osw.swiglu_fwd(Wgd, Wud, Xh, Agh, Bgh, Auh, Buh, s)
    dGo, dUo = osw.swiglu_bwd(Go, Uo, dHh)
    assert_close_fp(bf16_dev_to_f64(H), Ho, "H")
    dg, du = _deinterleave(bf16_dev_to_f64(dGU).T)
    assert_close_fp(dg.T, dGo, "dg")
    assert_close_fp(du.T, dUo, "du")
    dGb, dUb = osw.bf16r(dGo), osw.bf16r(dUo)   # the backward's inputs are the bf16 dg, du
    dXg, dAg_o, dBg_o = olin.linear_bwd(Wgd, Xh, Agh, Bgh, s, dGb)
    dXu, dAu_o, dBu_o = olin.linear_bwd(Wud, Xh, Auh, Buh, s, dUb)
    assert_close_fp(bf16_dev_to_f64(dX), dXg + dXu, "dX")
    dA = dAgu.cpu().numpy()
    assert_close_fp(dA[:r], dAg_o, "dA gate")
    assert_close_fp(dA[r:], dAu_o, "dA up")
    assert_close_fp(dBg.cpu().numpy(), dBg_o, "dB gate")
    assert_close_fp(dBu.cpu().numpy(), dBu_o, "dB up")


def test_swiglu_pack_and_unpack_layout(lib):
    """The block-diagonal adapter operand and the diagonal-block extraction,
    element by element (layout only, bit for bit)."""
    import torch
    F, r = 192, 8
    g = inputs.rng(310)
    Bg = torch.from_numpy(g.standard_normal((F, r)).astype(np.float32)).bfloat16().cuda()
    Bu = torch.from_numpy(g.standard_normal((F, r)).astype(np.float32)).bfloat16().cuda()
    Bgu = lib.swiglu_pack_b(Bg, Bu).cpu().float().numpy()
    for f in (0, 63, 64, 191):
        i_g, i_u = (f // 64) * 128 + f % 64, (f // 64) * 128 + 64 + f % 64
        np.testing.assert_array_equal(Bgu[i_g, :r], Bg[f].cpu().float().numpy())
        np.testing.assert_array_equal(Bgu[i_u, r:], Bu[f].cpu().float().numpy())
        assert not Bgu[i_g, r:].any() and not Bgu[i_u, :r].any()
    dBgu = torch.from_numpy(g.standard_normal((2 * F, 2 * r)).astype(np.float32)).cuda()
    dBg, dBu = lib.swiglu_unpack_db(dBgu)
    host = dBgu.cpu().numpy()
    for f in (0, 65, 191):
        i_g, i_u = (f // 64) * 128 + f % 64, (f // 64) * 128 + 64 + f % 64
        np.testing.assert_array_equal(dBg[f].cpu().numpy(), host[i_g, :r])
        np.testing.assert_array_equal(dBu[f].cpu().numpy(), host[i_u, r:])
