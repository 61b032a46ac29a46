"""Host-side checks of the seeded input generators (no GPU): shapes, seeds, the paged pool
layout and the NaN poison that the parity tests rely on."""
import math

import torch

from exact_attention_128_b200.workloads import (PAGED_DECODE, PAGED_PREFILL, DenseCase, PagedCase,
                                                PagedPrefillCase, paged_pool)


def test_dense_case_is_seeded_and_shaped():
    c = DenseCase("t", 2, 4, 2, 33, 65, 64, "bf16", True, 3)
    a, b = c.make(), c.make()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    q, k, v = a
    assert q.shape == (2, 4, 33, 64) and k.shape == v.shape == (2, 2, 65, 64) and q.dtype == torch.bfloat16
    # causal pairs: query i sees keys 0 .. i + 32
    assert c.allowed_pairs() == sum(min(65, i + 32 + 1) for i in range(33))


def test_paged_pool_is_a_permutation_with_minus_one_padding():
    ctx = torch.tensor([1, 16, 17, 100], dtype=torch.int32)
    g = torch.Generator().manual_seed(5)
    table, kc, vc, total = paged_pool(ctx, 16, 8, 2, 128, g, 5000, poison_unused=True)
    nblk = [math.ceil(int(c) / 16) for c in ctx]
    assert total == sum(nblk) and kc.shape == (total, 2, 16, 128)
    used = torch.cat([table[r, :n] for r, n in enumerate(nblk)])
    assert sorted(used.tolist()) == list(range(total))  # every physical block exactly once
    for r, n in enumerate(nblk):
        assert (table[r, n:] == -1).all()
        last = int(table[r, n - 1])
        filled = int(ctx[r]) - (n - 1) * 16
        assert torch.isfinite(kc[last, :, :filled].float()).all()
        assert torch.isnan(kc[last, :, filled:].float()).all() and torch.isnan(vc[last, :, filled:].float()).all()


def test_paged_decode_case_unchanged_by_refactor():
    inp = PAGED_DECODE.make()
    assert inp["num_blocks"] == sum(math.ceil(int(c) / 16) for c in inp["ctx_lens"])
    assert int(inp["ctx_lens"].min()) >= 512 and int(inp["ctx_lens"].max()) <= 8192
    assert inp["q"].shape == (64, 12, 128)


def test_paged_prefill_lengths_and_poison():
    full = PAGED_PREFILL.make(poison=True)
    ctx, ql = full["ctx_lens"], full["q_lens"]
    assert torch.equal(ctx, ql) and int(ctx.min()) >= 2048 and int(ctx.max()) <= 8192
    assert full["q"].shape == (8, 32, int(ql.max()), 128)
    for r, n in enumerate(ql.tolist()):
        assert torch.isfinite(full["q"][r, :, :n].float()).all()
        assert torch.isnan(full["q"][r, :, n:].float()).all()
    # chunked prompts: 1 <= q_len <= round(q_frac * ctx)
    pc = PagedPrefillCase("chunks", 16, 4, 2, 128, 16, 17, 900, 64, True, 11, q_frac=0.25)
    ctx, ql, _ = pc.lengths()
    assert all(1 <= q <= max(1, round(0.25 * c)) for c, q in zip(ctx.tolist(), ql.tolist()))
    # causal pairs of a chunk: the last q rows of a ctx-long sequence
    one = PagedPrefillCase("one", 1, 1, 1, 64, 16, 1, 64, 8, True, 1, ctx_lens_override=(10,), q_lens_override=(3,))
    assert one.allowed_pairs() == 8 + 9 + 10
    assert PagedCase.kv_bytes([10, 20], 2, 128) == 30 * 2 * 128 * 2 * 2
