"""Backward parity: CUDA kernels vs the fp64 oracle's gradients on the same seeded inputs.

The GPU backward consumes the GPU forward's O and lse (as a training step would); the
oracle computes everything from q, k, v, dO in fp64.
"""
import numpy as np
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import D256_TRAIN, TRAIN_CAUSAL, DenseCase
from oracle import attention_fp64 as ora
from parity import check_bf16, check_bf16_stored, to_np

pytestmark = pytest.mark.gpu


def run(case, grad_dtype=torch.float32):
    q, k, v, do = case.make(with_grad_output=True)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.fwd(qd, kd, vd, causal=case.causal, scale=case.scale)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, lse, dod, causal=case.causal, scale=case.scale, grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return (q, k, v, do), (dq, dk, dv)


def test_train_causal_full_size_sampled_heads():
    """B=8, H=16, N=4096, d=64, causal: 8 whole heads (each key/value head's full gradients)."""
    case = TRAIN_CAUSAL
    (q, k, v, do), (dq, dk, dv) = run(case)
    heads = [(0, 0), (7, 15), (3, 5), (1, 9), (5, 2), (6, 11), (2, 14), (4, 7)]
    rq, rk, rv = ora.attention_bwd(q, k, v, do, case.scale, True, heads=heads)
    for b, h in heads:
        check_bf16(dq[b, h], rq[b, h], f"dQ[{b},{h}]")
        check_bf16(dk[b, h], rk[b, h], f"dK[{b},{h}]")
        check_bf16(dv[b, h], rv[b, h], f"dV[{b},{h}]")


def test_train_d256_causal_sampled_heads():
    """Head dimension 256 training workload (B=2, Hq=16, Hkv=4, N=4096, causal): the full
    gradients of two key/value groups (their four query heads each)."""
    case = D256_TRAIN
    (q, k, v, do), (dq, dk, dv) = run(case)
    groups = [(0, 0), (1, 3)]
    rq, rk, rv = ora.attention_bwd(q, k, v, do, case.scale, True, heads=groups)
    for b, g in groups:
        check_bf16(dk[b, g], rk[b, g], f"dK[{b},{g}]")
        check_bf16(dv[b, g], rv[b, g], f"dV[{b},{g}]")
        for h in range(4 * g, 4 * g + 4):
            check_bf16(dq[b, h], rq[b, h], f"dQ[{b},{h}]")


EDGE = [
    # B, Hq, Hkv, Nq, Nkv, d, causal
    (1, 1, 1, 1, 1, 64, False),
    (1, 2, 1, 127, 127, 64, True),
    (2, 4, 2, 200, 200, 64, False),
    (1, 4, 1, 300, 300, 64, True),
    (1, 2, 2, 129, 129, 128, True),
    (1, 4, 2, 256, 384, 128, False),
    (1, 3, 1, 100, 612, 64, True),
    (1, 2, 1, 513, 513, 128, True),
    (1, 4, 2, 200, 200, 96, True),
    (2, 2, 1, 130, 300, 96, False),
    # head dimension 256: 64-row query steps, CTAs per half of the head dimension
    (1, 1, 1, 1, 1, 256, False),
    (1, 2, 1, 63, 63, 256, True),
    (1, 2, 2, 65, 65, 256, True),
    (1, 4, 2, 300, 300, 256, True),
    (2, 2, 1, 129, 517, 256, False),
    (1, 3, 1, 100, 612, 256, True),
    (1, 2, 2, 640, 640, 256, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,d,causal", EDGE)
def test_bwd_edge_shapes(B, Hq, Hkv, Nq, Nkv, d, causal):
    case = DenseCase("bwd_edge", B, Hq, Hkv, Nq, Nkv, d, "bf16", causal, 70 + Nq + Nkv + d)
    (q, k, v, do), (dq, dk, dv) = run(case)
    rq, rk, rv = ora.attention_bwd(q, k, v, do, case.scale, causal)
    check_bf16(dq, rq, "dQ")
    check_bf16(dk, rk, "dK")
    check_bf16(dv, rv, "dV")


def test_bwd_bf16_gradients():
    """bf16 gradients are the fp32 gradients rounded once.  The fp32 gradients meet the flat
    bar against the oracle; dK and dV stored as bf16 equal the round-to-nearest-even cast of
    the fp32 ones bit for bit (same accumulation order); dQ, whose fp32 accumulator takes
    reductions from many CTAs in no fixed order, is within one bf16 ulp of that cast.  A
    bf16-stored value can sit half an ulp (up to 0.031 in [8, 16)) from the exact gradient,
    so bf16 storage alone meets only the relaxed bar of check_bf16_stored."""
    case = DenseCase("bwd_bf16", 1, 4, 2, 640, 640, 64, "bf16", True, 91)
    (q, k, v, do), (dq32, dk32, dv32) = run(case, torch.float32)
    (_, _, _, _), (dq, dk, dv) = run(case, torch.bfloat16)
    assert dq.dtype == dk.dtype == dv.dtype == torch.bfloat16
    rq, rk, rv = ora.attention_bwd(q, k, v, do, case.scale, True)
    for got, ref, n in ((dq32, rq, "dQ"), (dk32, rk, "dK"), (dv32, rv, "dV")):
        check_bf16(got, ref, n + " (fp32)")
    assert torch.equal(dk, dk32.to(torch.bfloat16)) and torch.equal(dv, dv32.to(torch.bfloat16))
    cast = dq32.to(torch.bfloat16).float()
    ulp = torch.exp2(torch.floor(torch.log2(cast.abs().clamp_min(2.0 ** -126))) - 7)
    assert ((dq.float() - cast).abs() <= ulp).all()
    over = 0
    for got, ref, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        over += check_bf16_stored(got, ref, n)
    # the allowance is for a handful of elements next to a rounding midpoint, not a trend
    assert over <= 1e-3 * (dq.numel() + dk.numel() + dv.numel())


def test_bwd_d256_bf16_gradients_and_repeat():
    """Head dimension 256 with bf16 gradients: dK, dV are the round-to-nearest-even cast of
    the fp32 ones; two calls give the same dK, dV bits (each key tile's accumulation order
    is fixed)."""
    case = DenseCase("bwd256_bf16", 1, 4, 1, 384, 384, 256, "bf16", True, 95)
    (q, k, v, do), (dq32, dk32, dv32) = run(case, torch.float32)
    (_, _, _, _), (dq, dk, dv) = run(case, torch.bfloat16)
    rq, rk, rv = ora.attention_bwd(q, k, v, do, case.scale, True)
    for got, ref, n in ((dq32, rq, "dQ"), (dk32, rk, "dK"), (dv32, rv, "dV")):
        check_bf16(got, ref, n + " (fp32, d=256)")
    assert torch.equal(dk, dk32.to(torch.bfloat16)) and torch.equal(dv, dv32.to(torch.bfloat16))
    (_, _, _, _), (_, dk32b, dv32b) = run(case, torch.float32)
    assert torch.equal(dk32, dk32b) and torch.equal(dv32, dv32b)


def test_bwd_gradient_invariants_on_gpu():
    """Softmax ignores a common key shift: sum_j dK_j = 0 per head; sum_j dV_j = sum_i dO_i (G=1)."""
    case = DenseCase("inv", 1, 2, 2, 384, 384, 64, "bf16", True, 93)
    (q, k, v, do), (dq, dk, dv) = run(case)
    s_dk = to_np(dk).sum(axis=2)
    s_dv = to_np(dv).sum(axis=2)
    s_do = do.double().numpy().sum(axis=2)
    assert np.abs(s_dk).max() < 0.05
    assert np.abs(s_dv - s_do).max() < 0.05


F32_EDGE = [
    # B, Hq, Hkv, Nq, Nkv, causal: fp32 inputs take the CUDA-core backward (d = 64)
    (1, 12, 12, 196, 196, False),  # the fp32 ViT-B/16 layer
    (1, 1, 1, 1, 1, False),
    (1, 2, 1, 33, 33, True),
    (2, 4, 2, 100, 161, False),
    (1, 3, 1, 70, 300, True),
    (4, 8, 8, 320, 320, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,causal", F32_EDGE)
def test_bwd_f32(B, Hq, Hkv, Nq, Nkv, causal):
    """fp32 gradients against the fp64 oracle at the fp32 bar (max-abs 1e-5), fed the
    fp32 forward's O and lse as a training step would be."""
    case = DenseCase("bwd_f32", B, Hq, Hkv, Nq, Nkv, 64, "f32", causal, 90 + Nq + Nkv, 0.125)
    (q, k, v, do), (dq, dk, dv) = run(case)
    rq, rk, rv = ora.attention_bwd(q, k, v, do, case.scale, causal)
    for got, ref, name in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        err = np.abs(to_np(got) - ref).max()
        assert err <= 1e-5, f"{name}: fp32 max-abs {err:.3e}"
