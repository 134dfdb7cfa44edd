"""Pins of the 8-bit AdamW oracle: the first step from zero states against
torch.optim.AdamW (whose states are exact fp32), the code ranges and the
block maximum's code, and a multi-step run staying close to fp32-state
AdamW."""

import numpy as np
import torch

from oracle import adamw8
from bit_nf4_quantized_dequant_b200 import inputs

HP = dict(lr=1e-3, b1=0.9, b2=0.999, eps=1e-8, wd=0.01)


def _torch_adamw(p0, grads):
    p = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([p], lr=HP["lr"], betas=(HP["b1"], HP["b2"]), eps=HP["eps"], weight_decay=HP["wd"])
    for g in grads:
        p.grad = torch.from_numpy(g.copy())
        opt.step()
    return p.detach().numpy()


def _run(p0, grads):
    n = p0.size
    nb = -(-n // 256)
    p, mq, vq = p0.copy(), np.zeros(n, np.int8), np.zeros(n, np.uint8)
    ms, vs = np.zeros(nb, np.float32), np.zeros(nb, np.float32)
    for t, g in enumerate(grads, start=1):
        p, _, mq, vq, ms, vs = adamw8.step(p, g, mq, vq, ms, vs, t, **HP)
    return p, mq, vq, ms, vs


def test_first_step_matches_torch():
    g = inputs.rng(700)
    p0 = (g.standard_normal(1000) * 0.1).astype(np.float32)
    grad = (g.standard_normal(1000) * 0.01).astype(np.float32)
    p, *_ = _run(p0, [grad])
    np.testing.assert_allclose(p, _torch_adamw(p0, [grad]), rtol=1e-6, atol=1e-9)


def test_codes_and_block_maxima():
    g = inputs.rng(701)
    p0 = (g.standard_normal(700) * 0.1).astype(np.float32)
    grads = [(g.standard_normal(700) * 0.01).astype(np.float32) for _ in range(3)]
    p, mq, vq, ms, vs = _run(p0, grads)
    for b in range(3):
        sl = slice(256 * b, min(256 * (b + 1), 700))
        assert np.max(np.abs(mq[sl].astype(int))) == 127
        assert np.max(vq[sl]) == 255
        assert ms[b] > 0 and vs[b] > 0


def test_multi_step_close_to_fp32_states():
    g = inputs.rng(702)
    p0 = (g.standard_normal(2048) * 0.1).astype(np.float32)
    grads = [(g.standard_normal(2048) * 0.01).astype(np.float32) for _ in range(20)]
    p8, *_ = _run(p0, grads)
    p32 = _torch_adamw(p0, grads)
    drift = np.abs(p8 - p32).max()
    moved = np.abs(p32 - p0).max()
    assert drift < 0.2 * moved


def test_linear_8bit_second_moment_would_blow_up():
    """Why v is coded in its square-root domain: with linear 8-bit codes a
    small second moment next to a large one in its block decodes to zero and
    the step becomes m / eps. Shown on the reading's alternative, computed here."""
    v = np.array([1e-2, 1e-7], np.float32)
    linear_code = np.rint(np.float32(255) * v / v.max())
    assert linear_code[1] == 0                     # the small v would decode to 0
    sqrt_code = np.clip(np.rint(np.float32(255) * np.sqrt(v / v.max())), 1, 255)
    assert sqrt_code[1] >= 1                       # the reading keeps it nonzero
