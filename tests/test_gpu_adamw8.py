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
