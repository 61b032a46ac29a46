"""Forward parity: CUDA kernels vs the fp64 oracle on the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import (GQA_PREFILL_CAUSAL, VIT_BATCHED_BF16, VIT_LAYER_F32, DenseCase,
                                                prefill_sweep)
from oracle import attention_fp64 as ora
from parity import check_bf16, check_f32, check_lse, to_np

pytestmark = pytest.mark.gpu


def run(case):
    q, k, v = case.make()
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=case.causal, scale=case.scale)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return q, k, v, o, lse


def test_vit_layer_f32_full():
    q, k, v, o, lse = run(VIT_LAYER_F32)
    O, L = ora.attention_fwd(q, k, v, VIT_LAYER_F32.scale, False)
    check_f32(o, O, "O")
    check_f32(lse, L, "lse")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_worked_example_through_kernel(dtype):
    """Scores [0,0,ln3,ln3] with values [0,0,1,1] give 0.75 (two 2-key blocks would average to 0.5)."""
    q = torch.zeros(1, 1, 1, 64, dtype=dtype)
    k = torch.zeros(1, 1, 4, 64, dtype=dtype)
    v = torch.zeros(1, 1, 4, 64, dtype=dtype)
    q[0, 0, 0, 0] = 1.0
    k[0, 0, 2:, 0] = 1.0  # q.k = [0,0,1,1]; scale ln3 turns it into [0,0,ln3,ln3]
    v[0, 0, 2:, 0] = 1.0
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), scale=math.log(3.0))
    tol = 1e-6 if dtype == torch.float32 else 4e-3
    assert abs(o[0, 0, 0, 0].item() - 0.75) <= tol
    assert abs(lse[0, 0, 0].item() - math.log(8.0)) <= 1e-5


def test_vit_batched_bf16_full():
    q, k, v, o, lse = run(VIT_BATCHED_BF16)
    O, L = ora.attention_fwd(q, k, v, VIT_BATCHED_BF16.scale, False)
    check_bf16(o, O, "O")
    check_lse(lse, L, "lse")


EDGE = [
    # B, Hq, Hkv, Nq, Nkv, d, causal, dtype
    (1, 1, 1, 1, 1, 64, False, "bf16"),
    (1, 1, 1, 1, 1, 128, True, "bf16"),
    (1, 2, 1, 127, 127, 64, True, "bf16"),
    (1, 2, 2, 129, 129, 128, True, "bf16"),
    (2, 4, 1, 200, 333, 128, False, "bf16"),
    (1, 6, 6, 256, 256, 64, True, "bf16"),
    (1, 4, 2, 257, 257, 128, False, "bf16"),
    (1, 3, 1, 100, 612, 128, True, "bf16"),
    (1, 2, 1, 513, 513, 64, True, "bf16"),
    (1, 8, 2, 1000, 1000, 128, True, "bf16"),
    (1, 2, 1, 1, 300, 128, True, "bf16"),
    (1, 4, 2, 300, 300, 96, True, "bf16"),
    (2, 2, 1, 130, 517, 96, False, "bf16"),
    (1, 2, 1, 300, 300, 256, True, "bf16"),
    (1, 4, 2, 129, 517, 256, False, "bf16"),
    (2, 2, 2, 1, 70, 256, True, "bf16"),
    (1, 2, 1, 700, 1000, 256, True, "bf16"),
    (1, 2, 2, 77, 77, 64, False, "f32"),
    (1, 4, 2, 130, 200, 64, True, "f32"),
    (2, 2, 1, 1, 65, 64, False, "f32"),
    (4, 16, 4, 320, 320, 64, True, "f32"),  # enough rows for the 64-row variant
]


# Partial last query tiles leave warps whose rows are all padding: they skip the
# arithmetic and run ahead of the others, so the protocol that hands P to the tensor core
# must not let an early warp complete another warp's tile.  Each call is checked against
# the oracle, several times over, since such a fault depends on timing.
@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,d,causal", [
    (1, 4, 2, 129, 517, 256, False),
    (1, 2, 1, 300, 300, 256, True),
    (2, 2, 1, 161, 700, 256, True),
    (1, 4, 2, 129, 517, 128, False),
    (1, 3, 1, 97, 400, 64, True),
])
def test_partial_query_tiles_repeated(B, Hq, Hkv, Nq, Nkv, d, causal):
    case = DenseCase("partial", B, Hq, Hkv, Nq, Nkv, d, "bf16", causal, 17 + Nq + Nkv)
    q, k, v = (t.cuda() for t in case.make())
    O, L = ora.attention_fwd(q.cpu(), k.cpu(), v.cpu(), case.scale, causal)
    for _ in range(6):
        o, lse = fa.fwd(q, k, v, causal=causal, scale=case.scale)
        torch.cuda.synchronize()
        assert fa.device_status() == 0
        check_bf16(o, O, "O")
        check_lse(lse, L, "lse")


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,d,causal,dtype", EDGE)
def test_edge_shapes(B, Hq, Hkv, Nq, Nkv, d, causal, dtype):
    case = DenseCase("edge", B, Hq, Hkv, Nq, Nkv, d, dtype, causal, 11 + Nq + Nkv)
    q, k, v, o, lse = run(case)
    O, L = ora.attention_fwd(q, k, v, case.scale, causal)
    if dtype == "f32":
        check_f32(o, O, "O")
        check_f32(lse, L, "lse")
    else:
        check_bf16(o, O, "O")
        check_lse(lse, L, "lse")


# d = 64 with at most 256 keys (the ViT-like regime): ragged key counts inside a 16-key
# MMA step and a 32-column softmax chunk, query counts spanning several work items
SHORT = [
    # B, Hq, Hkv, Nq, Nkv, causal
    (1, 1, 1, 1, 1, False),
    (2, 3, 1, 1, 17, False),
    (1, 2, 2, 15, 15, True),
    (1, 4, 2, 16, 16, False),
    (1, 2, 1, 33, 100, True),
    (2, 4, 4, 196, 196, False),
    (1, 2, 1, 255, 255, True),
    (1, 2, 2, 256, 256, False),
    (1, 3, 3, 300, 256, False),
    (1, 2, 1, 513, 200, False),
    (1, 2, 1, 100, 256, True),
    (3, 2, 2, 600, 17, False),
    (1, 4, 1, 129, 130, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nkv,causal", SHORT)
def test_short_keys_d64(B, Hq, Hkv, Nq, Nkv, causal):
    case = DenseCase("short", B, Hq, Hkv, Nq, Nkv, 64, "bf16", causal, 500 + Nq + 3 * Nkv)
    q, k, v, o, lse = run(case)
    O, L = ora.attention_fwd(q, k, v, case.scale, causal)
    check_bf16(o, O, "O")
    check_lse(lse, L, "lse")


@pytest.mark.parametrize("causal", [False, True])
def test_short_keys_large_jumps_in_the_row_maximum(causal):
    """Later keys whose scores exceed the earlier keys' maximum by about 43 and then about
    100 more (base 2) move the running reference maximum twice; the second jump underflows
    the earlier terms to zero, as the exact softmax does in fp32."""
    case = DenseCase("jump", 1, 2, 1, 196, 196, 64, "bf16", causal, 77)
    q, k, v = case.make()
    q[..., 0] = 4.0
    k[0, 0, 70, 0] = 60.0   # scale * q.k = 30 natural units above the rest
    k[0, 0, 170, 0] = 140.0  # 70 natural units
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=case.scale)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    O, L = ora.attention_fwd(q, k, v, case.scale, causal)
    check_bf16(o, O, "O")
    check_lse(lse, L, "lse")


def test_causal_row0_returns_v0_exactly():
    case = DenseCase("row0", 2, 8, 2, 300, 300, 128, "bf16", True, 21)
    q, k, v, o, lse = run(case)
    vr = v.repeat_interleave(4, dim=1)
    assert torch.equal(o[:, :, 0].cpu(), vr[:, :, 0])


def _sample_rows(n, rng, count=512):
    """Seeded rows of one head: the tile boundaries and ends, plus random rows up to `count`."""
    fixed = [0, 1, 127, 128, 255, 256, 257, n // 2, n - 129, n - 128, n - 2, n - 1]
    rows = set(r for r in fixed if 0 <= r < n)
    rest = np.setdiff1d(np.arange(n), np.fromiter(rows, dtype=np.int64))
    rows.update(int(x) for x in rng.choice(rest, size=min(len(rest), max(0, count - len(rows))), replace=False))
    return sorted(rows)


def _check_sampled_heads(case, q, k, v, o, lse, rows_per_head=512):
    """Every (b, h) head on `rows_per_head` seeded rows: O at the bf16 bar (max-abs and
    relative Frobenius over the sampled block), lse at its bar.  Rows of the forward pass
    are independent, so the oracle's per-row function is exact for them."""
    rng = np.random.default_rng(case.seed)
    qn, kn, vn = ora.to_f64(q), ora.to_f64(k), ora.to_f64(v)
    on, ln = to_np(o), lse.cpu().numpy()
    for b in range(case.B):
        for h in range(case.Hq):
            rows = _sample_rows(case.Nq, rng, rows_per_head)
            O, L = ora.attention_fwd_rows(qn, kn, vn, case.scale, case.causal, b, h, rows)
            check_bf16(on[b, h, rows], O, f"{case.name} O[{b},{h}]")
            check_lse(ln[b, h, rows], L, f"{case.name} lse[{b},{h}]")
    return qn, kn, vn, on, ln


def test_gqa_prefill_causal_full_size():
    """B=4, Hq=32, Hkv=8, N=8192, d=128, causal: every head on 512 seeded rows, four heads in full."""
    case = GQA_PREFILL_CAUSAL
    q, k, v, o, lse = run(case)
    qn, kn, vn, on, ln = _check_sampled_heads(case, q, k, v, o, lse)
    for b, h in ((0, 0), (1, 17), (2, 6), (3, 31)):
        for r0 in range(0, case.Nq, 2048):
            rows = list(range(r0, r0 + 2048))
            O, L = ora.attention_fwd_rows(qn, kn, vn, case.scale, True, b, h, rows)
            check_bf16(on[b, h, r0 : r0 + 2048], O, f"O[{b},{h}]")
            check_lse(ln[b, h, r0 : r0 + 2048], L, "lse")


@pytest.mark.parametrize("case", prefill_sweep(), ids=lambda c: c.name)
def test_noncausal_sweep_sampled(case):
    """Non-causal sweep at B*N = 32768: every head on 512 seeded rows (N = 1024 and 2048:
    half or a quarter of all rows)."""
    q, k, v, o, lse = run(case)
    _check_sampled_heads(case, q, k, v, o, lse)


def test_repeat_calls_are_identical():
    case = DenseCase("repeat", 1, 4, 1, 640, 640, 128, "bf16", True, 31)
    q, k, v = (t.cuda() for t in case.make())
    o1, l1 = fa.fwd(q, k, v, causal=True)
    o2, l2 = fa.fwd(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_wait_timeout_sets_status_without_fault():
    fa.device_status(reset=True)
    fa.set_wait_limit_ns(2_000_000)
    try:
        fa.selftest_wait_timeout()
        assert fa.device_status(reset=True) == fa.FA_ERR_DEVICE_TIMEOUT
    finally:
        fa.set_wait_limit_ns(200_000_000)
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert x.sum().item() == 4.0
