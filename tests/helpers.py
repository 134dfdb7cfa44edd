"""Shared helpers of the test suite (comparison rules and device upload)."""

import numpy as np

# Tolerances for floating-point results of the GEMM path: relative Frobenius
# error <= 5e-3 and per-element |err| <= 1e-2 * max|ref|.
REL_FRO = 5e-3
ELEM = 1e-2


def assert_close_fp(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = got - ref
    ref_norm = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / ref_norm if ref_norm > 0 else np.linalg.norm(err)
    scale = np.abs(ref).max()
    emax = np.abs(err).max()
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert emax <= ELEM * scale + 1e-30, f"{what}: max |err| {emax:.3e} > {ELEM} * {scale:.3e}"
    return rel, emax / scale if scale > 0 else 0.0


def to_dev_bf16(bits):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def bf16_dev_to_f64(t):
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def bf16_dev_bits(t):
    import torch
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
