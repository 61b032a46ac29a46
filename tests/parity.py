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
    if isinstance(t, np.ndarray):
        return t.astype(np.float64, copy=False)
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_f32(got, ref, what=""):
    err = np.abs(to_np(got) - ref).max()
    assert err <= F32_ATOL, f"{what}: fp32 max-abs {err:.3e} > {F32_ATOL}"
    return err


def _exactly_zero(ref):
    """A reference that is zero up to fp64 rounding (e.g. dQ and dK when a row sees a
    single key: dS = P (dP - D) = 0); a relative error against it is undefined, so only
    the max-abs bar applies."""
    return np.linalg.norm(ref) <= 1e-9 * np.sqrt(max(ref.size, 1))


def check_bf16(got, ref, what=""):
    g = to_np(got)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - ref).max()
    assert err <= BF16_ATOL, f"{what}: max-abs {err:.3e} > {BF16_ATOL}"
    if _exactly_zero(ref):
        return err, 0.0
    fro = np.linalg.norm(g - ref) / np.linalg.norm(ref)
    assert fro <= BF16_REL_FRO, f"{what}: rel-Frobenius {fro:.3e} > {BF16_REL_FRO}"
    return err, fro


def check_lse(got, ref, what=""):
    err = np.abs(to_np(got) - ref).max()
    assert err <= LSE_ATOL, f"{what}: lse max-abs {err:.3e} > {LSE_ATOL}"
    return err


def bf16_half_ulp(x):
    """Half a unit in the last place of bf16 (8 significant bits) at |x|."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 0.5 * 2.0 ** (np.floor(np.log2(ax)) - 7)


def check_bf16_stored(got, ref, what=""):
    """Bar for results *stored* in bf16: 2e-2 plus the unavoidable final rounding.

    A bf16 output of magnitude in [4, 8) can be off by half an ulp (0.0156) from the exact
    value even when perfectly rounded, and by 0.031 in [8, 16), so each element may exceed
    the 2e-2 bar by at most half an ulp at its reference value; the relative Frobenius bar
    is unchanged.  Returns the number of elements that needed the allowance.
    """
    g = to_np(got)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    err = np.abs(g - ref)
    allow = BF16_ATOL + bf16_half_ulp(ref)
    worst = (err - allow).max()
    assert worst <= 0, f"{what}: max excess over 2e-2 + half-ulp {worst:.3e}"
    if not _exactly_zero(ref):
        fro = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        assert fro <= BF16_REL_FRO, f"{what}: rel-Frobenius {fro:.3e} > {BF16_REL_FRO}"
    return int((err > BF16_ATOL).sum())
