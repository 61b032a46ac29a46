"""Tolerances and comparison helpers for CUDA-vs-oracle parity tests.

Bars (stated for this library): fp32 outputs max-abs <= 1e-5; bf16 outputs and
gradients max-abs <= 2e-2 and relative Frobenius error <= 5e-3; lse abs <= 1e-3.
"""
import numpy as np

F32_ATOL = 1e-5
BF16_ATOL = 2e-2
BF16_REL_FRO = 5e-3
LSE_ATOL = 1e-3


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_f32(got, ref, what=""):
    err = np.abs(to_np(got) - ref).max()
    assert err <= F32_ATOL, f"{what}: fp32 max-abs {err:.3e} > {F32_ATOL}"
    return err


def check_bf16(got, ref, what=""):
    g = to_np(got)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - ref).max()
    fro = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= BF16_ATOL, f"{what}: max-abs {err:.3e} > {BF16_ATOL}"
    assert fro <= BF16_REL_FRO, f"{what}: rel-Frobenius {fro:.3e} > {BF16_REL_FRO}"
    return err, fro


def check_lse(got, ref, what=""):
    err = np.abs(to_np(got) - ref).max()
    assert err <= LSE_ATOL, f"{what}: lse max-abs {err:.3e} > {LSE_ATOL}"
    return err
