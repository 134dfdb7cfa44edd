"""AdamW with 8-bit optimiser states, float32 oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA, in depth" (aicassindra.com), section "A complete run on a 12
GB-class GPU": training uses the paged 8-bit AdamW, whose optimiser states
are held in 8 bits; "QLoRA and Fine-Tuning on One Consumer GPU", section
"Where 24 GB goes": adapter gradients plus Adam's m and v.

AdamW (decoupled weight decay):
    m = b1 m + (1 - b1) g,   v = b2 v + (1 - b2) g^2,
    p = p - lr (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd p).

Reading (the pages say only "8 bits"): blocks of 256 elements; m stored as
int8 codes q with m = q / 127 * (block absmax of m), codes rint(127 m /
absmax); v stored as uint8 codes of its square root, v = (q / 255)^2 * (block
max of v), codes clamp(rint(255 sqrt(v / max)), 1, 255) for v > 0 and 0 for
v = 0 (half to even). The square-root domain and the floor of 1 keep a small
nonzero second moment from decoding to zero, which a linear 8-bit v would do
(and its update would become m / eps: test_oracle_adamw8 shows the blow-up). The method computes in float32, and the codes are decisions
taken on float32 values, so this oracle computes in float32 too, every
operation rounded once, in the order written above (precision as in the
pages' setting: the update runs in the optimiser's fp32).
"""

from __future__ import annotations

import numpy as np

BLOCK = 256
f32 = np.float32


def step(p, g, mq, vq, mscale, vscale, t: int, lr, b1, b2, eps, wd):
    """One step; returns new (p, p_bf16_bits, mq, vq, mscale, vscale)."""
    from .nf4 import bf16_round_bits
    p, g = np.asarray(p, f32), np.asarray(g, f32)
    n = p.size
    nb = -(-n // BLOCK)
    b1, b2, lr, eps, wd = f32(b1), f32(b2), f32(lr), f32(eps), f32(wd)
    omb1, omb2 = f32(f32(1) - b1), f32(f32(1) - b2)
    bc1 = f32(1.0 - float(b1) ** t)
    bc2 = f32(1.0 - float(b2) ** t)
    blk = np.arange(n) // BLOCK
    m0 = (np.asarray(mq, np.int8).astype(f32) / f32(127)) * np.asarray(mscale, f32)[blk]
    tq = np.asarray(vq, np.uint8).astype(f32) / f32(255)
    v0 = (tq * tq) * np.asarray(vscale, f32)[blk]
    m = (b1 * m0) + (omb1 * g)
    v = (b2 * v0) + (omb2 * (g * g))
    mh, vh = m / bc1, v / bc2
    upd = (mh / (np.sqrt(vh) + eps)) + (wd * p)
    pn = p - (lr * upd)
    pad = nb * BLOCK - n
    mmax = np.max(np.abs(np.concatenate([m, np.zeros(pad, f32)])).reshape(nb, BLOCK), axis=1)
    vmax = np.max(np.concatenate([v, np.zeros(pad, f32)]).reshape(nb, BLOCK), axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        mq_n = np.where(mmax[blk] > 0, np.rint((m * f32(127)) / mmax[blk]), f32(0)).astype(np.int8)
        qv = np.clip(np.rint(f32(255) * np.sqrt(v / vmax[blk])), f32(1), f32(255))
        vq_n = np.where(v > 0, qv, f32(0)).astype(np.uint8)
    return pn, bf16_round_bits(pn), mq_n, vq_n, mmax.astype(f32), vmax.astype(f32)
