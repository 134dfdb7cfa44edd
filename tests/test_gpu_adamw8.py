"""GPU parity of the 8-bit AdamW step against oracle.adamw8 over several
steps: parameters (fp32 bits), their bf16 copy, the int8 / uint8 state codes
and the block scales, all bit for bit (every operation on both sides is a
single IEEE-rounded fp32 operation in the same order)."""

import numpy as np
import pytest

from oracle import adamw8 as oadam
from bit_nf4_quantized_dequant_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,wd", [(1000, 0.01), (16 * 4096, 0.0), (4096 * 16 + 77, 0.1)])
def test_adamw8_steps_bit_exact(lib, n, wd):
    import torch
    g = inputs.rng(800 + n)
    p0 = (g.standard_normal(n) * 0.05).astype(np.float32)
    grads = [(g.standard_normal(n) * 0.01 * (1 + (i % 3))).astype(np.float32) for i in range(5)]
    hp = dict(lr=2e-4, b1=0.9, b2=0.999, eps=1e-8, wd=wd)
    p = torch.from_numpy(p0.copy()).cuda()
    pb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    st = lib.AdamW8State(n)
    ph, mq, vq = p0.copy(), np.zeros(n, np.int8), np.zeros(n, np.uint8)
    ms, vs = np.zeros(-(-n // 256), np.float32), np.zeros(-(-n // 256), np.float32)
    for t, gr in enumerate(grads, start=1):
        lib.adamw8_step(p, torch.from_numpy(gr).cuda(), st, hp["lr"], hp["b1"], hp["b2"], hp["eps"], hp["wd"],
                        p_bf16=pb)
        ph, pbits, mq, vq, ms, vs = oadam.step(ph, gr, mq, vq, ms, vs, t, **hp)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(p.cpu().numpy().view(np.uint32), ph.view(np.uint32))
        np.testing.assert_array_equal(pb.view(torch.int16).cpu().numpy().view(np.uint16), pbits)
        np.testing.assert_array_equal(st.m_q.cpu().numpy(), mq)
        np.testing.assert_array_equal(st.v_q.cpu().numpy(), vq)
        np.testing.assert_array_equal(st.m_scale.cpu().numpy().view(np.uint32), ms.view(np.uint32))
        np.testing.assert_array_equal(st.v_scale.cpu().numpy().view(np.uint32), vs.view(np.uint32))


FUSED_CASES = [
    # N, K, M, r
    (4096, 1024, 300, 16),   # 32 + 8 gradient tiles, cluster-split reduction
    (272, 320, 100, 8),      # ragged last tiles of both adapters; 32-row state blocks
    (160, 256, 17, 32),
    (1024, 4096, 64, 64),
]


def _exact_inputs(g, M, N, K, r):
    """bf16 inputs of the form k / 8, |k| <= 3: every product and every sum of
    the adapter gradients is exact in fp32, whatever the summation order, so
    the oracle's gradients equal the kernel's bit for bit."""
    import torch
    f = lambda *shape: torch.from_numpy((g.integers(-3, 4, shape) / 8.0).astype(np.float32)).bfloat16().cuda()
    return f(M, K), f(M, N), f(M, r), f(M, r)


@pytest.mark.parametrize("N,K,M,r", FUSED_CASES)
def test_fused_grads_adamw8_matches_oracle(lib, N, K, M, r):
    """qlora_lora_grads_adamw8 over three steps against oracle.adamw8 on the
    oracle's gradients (dA^T for A's d-major state, dB for B's): parameters,
    bf16 operands (A written back as [r, K]), state codes and block scales
    bit for bit; the fp32 gradients it writes equal the exact ones."""
    import torch
    g = inputs.rng(900 + N + K + r)
    hp = dict(lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.01)
    A0 = (g.standard_normal((K, r)) / r).astype(np.float32)        # master of A^T
    B0 = (g.standard_normal((N, r)) * 0.01).astype(np.float32)
    Am, Bm = torch.from_numpy(A0.copy()).cuda(), torch.from_numpy(B0.copy()).cuda()
    Ab = torch.empty((r, K), dtype=torch.bfloat16, device="cuda")
    Bb = torch.empty((N, r), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
    dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
    sA, sB = lib.AdamW8State(K * r), lib.AdamW8State(N * r)
    ref = {}
    for name, p0, n in (("A", A0, K * r), ("B", B0, N * r)):
        nb = -(-n // 256)
        ref[name] = [p0.reshape(-1).copy(), np.zeros(n, np.int8), np.zeros(n, np.uint8),
                     np.zeros(nb, np.float32), np.zeros(nb, np.float32)]
    for t in range(1, 4):
        X, dY, sU, sT = _exact_inputs(g, M, N, K, r)
        lib.lora_grads_adamw8(X, dY, sU, sT, Am, Bm, sA, sB, hp["lr"], hp["b1"], hp["b2"], hp["eps"], hp["wd"],
                              A_bf16=Ab, B_bf16=Bb, dA=dA, dB=dB)
        f64 = lambda x: x.float().cpu().numpy().astype(np.float64)
        gA = (f64(sT).T @ f64(X)).astype(np.float32)                 # [r, K], exact
        gB = (f64(dY).T @ f64(sU)).astype(np.float32)                # [N, r], exact
        torch.cuda.synchronize()
        np.testing.assert_array_equal(dA.cpu().numpy(), gA)
        np.testing.assert_array_equal(dB.cpu().numpy(), gB)
        outs = {}
        for name, grad in (("A", gA.T.reshape(-1)), ("B", gB.reshape(-1))):
            p, mq, vq, ms, vs = ref[name]
            p, pbits, mq, vq, ms, vs = oadam.step(p, np.ascontiguousarray(grad), mq, vq, ms, vs, t, **hp)
            ref[name] = [p, mq, vq, ms, vs]
            outs[name] = pbits
        for name, pm, pb, st, shape in (("A", Am, Ab, sA, (K, r)), ("B", Bm, Bb, sB, (N, r))):
            p, mq, vq, ms, vs = ref[name]
            np.testing.assert_array_equal(pm.cpu().numpy().reshape(-1).view(np.uint32), p.view(np.uint32))
            bits = pb.view(torch.int16).cpu().numpy().view(np.uint16)
            want = outs[name].reshape(shape)
            np.testing.assert_array_equal(bits, want.T if name == "A" else want)
            np.testing.assert_array_equal(st.m_q.cpu().numpy(), mq)
            np.testing.assert_array_equal(st.v_q.cpu().numpy(), vq)
            np.testing.assert_array_equal(st.m_scale.cpu().numpy().view(np.uint32), ms.view(np.uint32))
            np.testing.assert_array_equal(st.v_scale.cpu().numpy().view(np.uint32), vs.view(np.uint32))


def test_fused_equals_gradients_then_step(lib):
    """On random inputs (gradients rounded in the kernel's summation order)
    the fused launch equals qlora_lora_grads followed by two
    qlora_adamw8_step calls, bit for bit."""
    import torch
    N, K, M, r = 2048, 1536, 700, 16
    g = inputs.rng(950)
    bf = lambda *shape: torch.from_numpy(g.standard_normal(shape).astype(np.float32)).bfloat16().cuda()
    X, dY, sU, sT = bf(M, K), bf(M, N), bf(M, r), bf(M, r)
    A0 = torch.from_numpy((g.standard_normal((K, r)) / r).astype(np.float32)).cuda()
    B0 = torch.from_numpy((g.standard_normal((N, r)) * 0.01).astype(np.float32)).cuda()
    # fused
    Am, Bm = A0.clone(), B0.clone()
    Ab = torch.empty((r, K), dtype=torch.bfloat16, device="cuda")
    Bb = torch.empty((N, r), dtype=torch.bfloat16, device="cuda")
    sA, sB = lib.AdamW8State(K * r), lib.AdamW8State(N * r)
    lib.lora_grads_adamw8(X, dY, sU, sT, Am, Bm, sA, sB, 1e-3, weight_decay=0.01, A_bf16=Ab, B_bf16=Bb)
    # separate
    dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
    dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
    ws = torch.zeros(lib.linear_workspace(M, N, K, r), dtype=torch.uint8, device="cuda")
    lib.lora_grads(X, dY, sU, sT, dA, dB, ws)
    Am2, Bm2 = A0.clone(), B0.clone()
    Ab2 = torch.empty(K * r, dtype=torch.bfloat16, device="cuda")
    Bb2 = torch.empty(N * r, dtype=torch.bfloat16, device="cuda")
    sA2, sB2 = lib.AdamW8State(K * r), lib.AdamW8State(N * r)
    lib.adamw8_step(Am2.view(-1), dA.t().contiguous().view(-1), sA2, 1e-3, weight_decay=0.01, p_bf16=Ab2)
    lib.adamw8_step(Bm2.view(-1), dB.view(-1), sB2, 1e-3, weight_decay=0.01, p_bf16=Bb2)
    torch.cuda.synchronize()
    eq = lambda a, b: torch.equal(a.contiguous().view(torch.int8), b.contiguous().view(torch.int8))
    assert eq(Am, Am2) and eq(Bm, Bm2)
    assert eq(Ab, Ab2.view(K, r).t()) and eq(Bb, Bb2.view(N, r))
    for s1, s2 in ((sA, sA2), (sB, sB2)):
        assert eq(s1.m_q, s2.m_q) and eq(s1.v_q, s2.v_q) and eq(s1.m_scale, s2.m_scale) and eq(s1.v_scale, s2.v_scale)
