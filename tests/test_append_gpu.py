"""Paged KV-cache append: bit-exact against the oracle's slot writes, then decode on it."""
import numpy as np
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import randn
from oracle import attention_fp64 as ora
from parity import check_bf16, check_lse

pytestmark = pytest.mark.gpu


def make(R=8, Hkv=2, d=128, bs=16, maxb=8, seed=60):
    g = torch.Generator().manual_seed(seed)
    num_blocks = R * maxb + 5
    table = torch.randperm(num_blocks, generator=g)[: R * maxb].reshape(R, maxb).to(torch.int32)
    kc = randn((num_blocks, Hkv, bs, d), seed * 10 + 1, torch.bfloat16)
    vc = randn((num_blocks, Hkv, bs, d), seed * 10 + 2, torch.bfloat16)
    k_new = randn((R, Hkv, d), seed * 10 + 3, torch.bfloat16)
    v_new = randn((R, Hkv, d), seed * 10 + 4, torch.bfloat16)
    pos = torch.randint(0, maxb * bs, (R,), generator=g, dtype=torch.int64).to(torch.int32)
    return table, kc, vc, k_new, v_new, pos


def test_append_matches_oracle_bit_exact():
    table, kc, vc, k_new, v_new, pos = make()
    pos[0], pos[1] = 0, 8 * 16 - 1  # first and last slot of the table
    kd, vd = kc.cuda(), vc.cuda()
    fa.paged_kv_append(k_new.cuda(), v_new.cuda(), kd, vd, table.cuda(), pos.cuda())
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    rk, rv = ora.paged_append(kc.float().numpy(), vc.float().numpy(), table.numpy(), pos.numpy(),
                              k_new.float().numpy(), v_new.float().numpy(), 16)
    assert np.array_equal(kd.float().cpu().numpy(), rk)
    assert np.array_equal(vd.float().cpu().numpy(), rv)


def test_append_then_decode():
    table, kc, vc, k_new, v_new, pos = make(seed=61)
    R, Hq = table.shape[0], 12
    q = randn((R, Hq, 128), 615, torch.bfloat16)
    kd, vd = kc.cuda(), vc.cuda()
    fa.paged_kv_append(k_new.cuda(), v_new.cuda(), kd, vd, table.cuda(), pos.cuda())
    ctx = (pos + 1).to(torch.int32)
    o, lse = fa.paged_decode(q.cuda(), kd, vd, table.cuda(), ctx.cuda())
    torch.cuda.synchronize()
    rk, rv = ora.paged_append(kc.float().numpy(), vc.float().numpy(), table.numpy(), pos.numpy(),
                              k_new.float().numpy(), v_new.float().numpy(), 16)
    O, L = ora.paged_decode(q, rk, rv, table.numpy(), ctx.numpy(), 16, 128 ** -0.5)
    check_bf16(o, O, "O")
    check_lse(lse, L, "lse")


def test_append_out_of_range_is_flagged_not_written():
    table, kc, vc, k_new, v_new, pos = make(seed=62)
    pos[2] = 8 * 16  # past the table
    table[3, int(pos[3]) // 16] = 10_000  # past the pool
    kd, vd = kc.cuda(), vc.cuda()
    fa.device_status(reset=True)
    fa.paged_kv_append(k_new.cuda(), v_new.cuda(), kd, vd, table.cuda(), pos.cuda())
    assert fa.device_status(reset=True) == fa.FA_ERR_INVALID_ARG
    keep = [r for r in range(table.shape[0]) if r not in (2, 3)]
    rk, _ = ora.paged_append(kc.float().numpy(), vc.float().numpy(), table.numpy()[keep], pos.numpy()[keep],
                             k_new.float().numpy()[keep], v_new.float().numpy()[keep], 16)
    assert np.array_equal(kd.float().cpu().numpy(), rk)
