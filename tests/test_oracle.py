"""Pins for the fp64 oracle, against facts that do not come from the oracle itself.

Each pin cites what fixes it: the pages' worked example, closed forms of softmax,
brute-force blockwise merges (the pages' recurrence), finite differences, invariants
of the definition, and an independent library routine (torch's fp64 CPU attention).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention_fp64 as ora

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        w = json.load(f)
    scores = np.array([0.0 if s == "0" else math.log(3.0) for s in w["scores"]])
    return w, scores, np.array(w["values"])


# ---------------------------------------------------------------------------------
# The pages' worked example ("FlashAttention", "No basta con promediar ...")
# ---------------------------------------------------------------------------------
def test_worked_example_direct_definition():
    w, s, v = _worked()
    # one query, d = 1: q = 1 and k_j = s_j give the stated scores with scale 1
    O, lse, P = ora.attention_head(np.ones((1, 1)), s[:, None], v[:, None], scale=1.0)
    assert abs(O[0, 0] - w["expected_output"]) < 1e-15
    ratios = P[0] / P[0].min()
    np.testing.assert_allclose(ratios, w["unnormalised_weight_ratios"], rtol=1e-14)
    assert abs(lse[0] - math.log(8.0)) < 1e-15  # e^0 + e^0 + 3 + 3


def test_worked_example_two_block_recurrence():
    w, s, v = _worked()
    out, m, l = ora.online_softmax_blocks([s[:2], s[2:]], [v[:2], v[2:]])
    assert abs(out[0] - w["expected_output"]) < 1e-15
    # each block on its own gives the stated block results; their plain mean is wrong
    blk = [ora.online_softmax_blocks([s[i : i + 2]], [v[i : i + 2]])[0][0] for i in (0, 2)]
    assert blk == pytest.approx(w["block_results"], abs=1e-15)
    assert np.mean(blk) == pytest.approx(w["naive_block_mean_wrong"])
    assert abs(np.mean(blk) - w["expected_output"]) > 0.2


def test_worked_example_partial_merge():
    w, s, v = _worked()
    parts = [ora.attention_head(np.ones((1, 1)), s[i : i + 2, None], v[i : i + 2, None], 1.0) for i in (0, 2)]
    o, lse = ora.merge_partials([p[1][0] for p in parts], [p[0][0] for p in parts])
    assert abs(o[0] - w["expected_output"]) < 1e-15
    assert abs(lse - math.log(8.0)) < 1e-15


# ---------------------------------------------------------------------------------
# Brute force: the blockwise recurrence equals the definition for any partition
# ---------------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(6))
def test_random_block_partitions_match_definition(seed):
    rng = np.random.default_rng(seed)
    n, d = int(rng.integers(1, 40)), int(rng.integers(1, 6))
    q = rng.standard_normal((1, d))
    k = rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    scale = 1.0 / math.sqrt(d)
    O, _, _ = ora.attention_head(q, k, v, scale)
    s = scale * (k @ q[0])
    cuts = np.sort(rng.choice(np.arange(1, n), size=min(n - 1, int(rng.integers(0, 6))), replace=False)) if n > 1 else []
    sb = np.split(s, cuts)
    vb = np.split(v, cuts)
    out, m, l = ora.online_softmax_blocks(sb, vb)
    np.testing.assert_allclose(out, O[0], rtol=0, atol=1e-14)
    assert m == pytest.approx(s.max())
    assert l == pytest.approx(np.exp(s - s.max()).sum(), rel=1e-14)


@pytest.mark.parametrize("bs", [1, 2, 3, 7, 16, 37])
def test_block_size_invariance(bs):
    rng = np.random.default_rng(11)
    n, d = 37, 5
    s = rng.standard_normal(n) * 4
    v = rng.standard_normal((n, d))
    ref, _, _ = ora.online_softmax_blocks([s], [v])
    out, _, _ = ora.online_softmax_blocks([s[i : i + bs] for i in range(0, n, bs)], [v[i : i + bs] for i in range(0, n, bs)])
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------------
# Closed forms and invariants of softmax
# ---------------------------------------------------------------------------------
def test_rows_sum_to_one_and_lse_is_logsumexp():
    rng = np.random.default_rng(3)
    q, k, v = rng.standard_normal((9, 4)), rng.standard_normal((13, 4)), rng.standard_normal((13, 4))
    for causal in (False, True):
        O, lse, P = ora.attention_head(q, k, v, 0.5, causal)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-15)
        S = 0.5 * q @ k.T
        if causal:
            S = np.where(ora.causal_allowed(9, 13), S, -np.inf)
        np.testing.assert_allclose(lse, np.logaddexp.reduce(S, axis=1), rtol=0, atol=1e-13)


def test_equal_scores_give_mean_of_values():
    rng = np.random.default_rng(4)
    v = rng.standard_normal((10, 3))
    O, _, _ = ora.attention_head(np.zeros((2, 3)), rng.standard_normal((10, 3)), v, 1.0)
    np.testing.assert_allclose(O, np.broadcast_to(v.mean(axis=0), O.shape), atol=1e-15)


def test_dominant_score_selects_its_value():
    rng = np.random.default_rng(5)
    k = np.zeros((6, 1))
    k[4, 0] = 1.0
    v = rng.standard_normal((6, 2))
    O, lse, _ = ora.attention_head(np.array([[60.0]]), k, v, 1.0)
    np.testing.assert_allclose(O[0], v[4], atol=1e-20 + 1e-24)
    assert lse[0] == pytest.approx(60.0)


def test_scale_enters_as_inverse_sqrt_dk():
    # "Scores = Q K^T / sqrt(d_k)": with q = k = 1-vectors of length d the score is sqrt(d)
    d = 16
    O, lse, _ = ora.attention_head(np.ones((1, d)), np.ones((1, d)), np.ones((1, 1)), 1 / math.sqrt(d))
    assert lse[0] == pytest.approx(math.sqrt(d), abs=1e-14)


# ---------------------------------------------------------------------------------
# Causal reading, GQA reading, multi-head structure
# ---------------------------------------------------------------------------------
def test_causal_row0_is_v0_and_rows_are_prefix_attention():
    rng = np.random.default_rng(6)
    n, d = 12, 4
    q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
    O, _, _ = ora.attention_head(q, k, v, 0.7, causal=True)
    assert np.array_equal(O[0], v[0])
    for i in range(n):
        Oi, _, _ = ora.attention_head(q[i : i + 1], k[: i + 1], v[: i + 1], 0.7)
        np.testing.assert_allclose(O[i], Oi[0], atol=1e-14)


def test_causal_bottom_right_alignment_for_shorter_query():
    rng = np.random.default_rng(7)
    nq, nkv, d = 3, 8, 4
    q, k, v = rng.standard_normal((nq, d)), rng.standard_normal((nkv, d)), rng.standard_normal((nkv, d))
    O, _, _ = ora.attention_head(q, k, v, 0.5, causal=True)
    for i in range(nq):
        last = nkv - nq + i
        Oi, _, _ = ora.attention_head(q[i : i + 1], k[: last + 1], v[: last + 1], 0.5)
        np.testing.assert_allclose(O[i], Oi[0], atol=1e-14)
    # a single query token sees every key: decode is the nq == 1 case
    O1, _, _ = ora.attention_head(q[:1], k, v, 0.5, causal=True)
    O1n, _, _ = ora.attention_head(q[:1], k, v, 0.5, causal=False)
    np.testing.assert_array_equal(O1, O1n)


def test_gqa_equals_explicitly_repeated_heads():
    rng = np.random.default_rng(8)
    B, Hq, Hkv, N, d = 2, 6, 2, 7, 4
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    O, lse = ora.attention_fwd(q, k, v, 0.5, causal=True)
    kr, vr = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    for b in range(B):
        for h in range(Hq):
            o, l, _ = ora.attention_head(q[b, h], kr[b, h], vr[b, h], 0.5, True)
            np.testing.assert_array_equal(O[b, h], o)
            np.testing.assert_array_equal(lse[b, h], l)
    with pytest.raises(ValueError):
        ora.attention_fwd(q[:, :5], k, v, 0.5)


def test_rows_helper_matches_full_forward():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, 4, 10, 3))
    k = rng.standard_normal((1, 2, 10, 3))
    v = rng.standard_normal((1, 2, 10, 3))
    O, lse = ora.attention_fwd(q, k, v, 0.3, causal=True)
    rows = [0, 3, 9]
    o, l = ora.attention_fwd_rows(q, k, v, 0.3, True, 0, 3, rows)
    np.testing.assert_allclose(o, O[0, 3, rows], atol=1e-15)
    np.testing.assert_allclose(l, lse[0, 3, rows], atol=1e-15)


def test_forward_matches_torch_fp64_library_attention():
    g = torch.Generator().manual_seed(10)
    B, Hq, Hkv, N, d = 2, 4, 2, 9, 8
    q = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64)
    for causal in (False, True):
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), is_causal=causal, scale=0.3
        )
        O, _ = ora.attention_fwd(q, k, v, 0.3, causal)
        np.testing.assert_allclose(O, ref.numpy(), atol=1e-13)


# ---------------------------------------------------------------------------------
# Gradients
# ---------------------------------------------------------------------------------
def _loss(q, k, v, do, scale, causal):
    O, _ = ora.attention_fwd(q, k, v, scale, causal)
    return float((O * do).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_central_finite_differences(causal):
    rng = np.random.default_rng(12)
    B, Hq, Hkv, N, d = 1, 2, 1, 5, 3
    q = rng.standard_normal((B, Hq, N, d))
    k = rng.standard_normal((B, Hkv, N, d))
    v = rng.standard_normal((B, Hkv, N, d))
    do = rng.standard_normal((B, Hq, N, d))
    scale = 0.8
    dq, dk, dv = ora.attention_bwd(q, k, v, do, scale, causal)
    h = 1e-6
    for name, x, gx in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            fm = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            num[idx] = (fp - fm) / (2 * h)
        err = np.abs(num - gx).max() / max(1.0, np.abs(gx).max())
        assert err < 1e-6, (name, err)


def test_gradients_match_torch_fp64_autograd():
    g = torch.Generator().manual_seed(13)
    B, Hq, Hkv, N, d = 2, 4, 2, 11, 8
    q = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64, requires_grad=True)
    k = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64, requires_grad=True)
    v = torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64, requires_grad=True)
    do = torch.randn(B, Hq, N, d, generator=g, dtype=torch.float64)
    for causal in (False, True):
        for t in (q, k, v):
            t.grad = None
        out = torch.nn.functional.scaled_dot_product_attention(
            q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), is_causal=causal, scale=0.25
        )
        out.backward(do)
        dq, dk, dv = ora.attention_bwd(q, k, v, do, 0.25, causal)
        np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12)
        np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12)


@pytest.mark.parametrize("Nq,Nkv,causal", [(3, 9, True), (7, 9, True), (3, 9, False), (9, 4, False)])
def test_gradients_rectangular_match_torch_fp64_autograd(Nq, Nkv, causal):
    """Nq != Nkv, with the causal mask aligned bottom-right (query i sees keys
    j <= i + Nkv - Nq), given to torch as an explicit boolean mask."""
    g = torch.Generator().manual_seed(16)
    B, Hq, Hkv, d = 1, 4, 2, 5
    q = torch.randn(B, Hq, Nq, d, generator=g, dtype=torch.float64, requires_grad=True)
    k = torch.randn(B, Hkv, Nkv, d, generator=g, dtype=torch.float64, requires_grad=True)
    v = torch.randn(B, Hkv, Nkv, d, generator=g, dtype=torch.float64, requires_grad=True)
    do = torch.randn(B, Hq, Nq, d, generator=g, dtype=torch.float64)
    mask = None
    if causal:
        mask = torch.arange(Nkv)[None, :] <= torch.arange(Nq)[:, None] + (Nkv - Nq)
    out = torch.nn.functional.scaled_dot_product_attention(
        q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), attn_mask=mask, scale=0.4
    )
    out.backward(do)
    dq, dk, dv = ora.attention_bwd(q.detach(), k.detach(), v.detach(), do, 0.4, causal)
    np.testing.assert_allclose(dq, q.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, k.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, v.grad.numpy(), atol=1e-12)


def test_gradient_invariants():
    """Softmax ignores a common shift of all keys, and P's rows sum to one."""
    rng = np.random.default_rng(14)
    q, k, v, do = (rng.standard_normal((1, 1, 8, 4)) for _ in range(4))
    for causal in (False, True):
        dq, dk, dv = ora.attention_bwd(q, k, v, do, 0.6, causal)
        np.testing.assert_allclose(dk[0, 0].sum(axis=0), 0.0, atol=1e-13)
        np.testing.assert_allclose(dv[0, 0].sum(axis=0), do[0, 0].sum(axis=0), atol=1e-13)


def test_bwd_head_subset_leaves_others_nan():
    rng = np.random.default_rng(15)
    q, do = rng.standard_normal((1, 4, 5, 3)), rng.standard_normal((1, 4, 5, 3))
    k, v = rng.standard_normal((1, 2, 5, 3)), rng.standard_normal((1, 2, 5, 3))
    full = ora.attention_bwd(q, k, v, do, 0.5, True)
    part = ora.attention_bwd(q, k, v, do, 0.5, True, heads=[(0, 1)])
    np.testing.assert_array_equal(part[1][0, 1], full[1][0, 1])
    np.testing.assert_array_equal(part[0][0, 2:], full[0][0, 2:])
    assert np.isnan(part[1][0, 0]).all() and np.isnan(part[0][0, :2]).all()


# ---------------------------------------------------------------------------------
# Paged decode: equals dense attention on the contiguous keys it was built from
# ---------------------------------------------------------------------------------
def _scatter_to_pages(kv_list, bs, Hkv, d, rng):
    """Build a paged cache from contiguous per-request [Hkv, n, d] arrays (test-side)."""
    nblk = [(x.shape[1] + bs - 1) // bs for x in kv_list]
    total = sum(nblk)
    perm = rng.permutation(total)
    cache = np.full((total, Hkv, bs, d), np.nan)
    table = np.full((len(kv_list), max(nblk) + 2), -1, dtype=np.int64)
    pos = 0
    for r, x in enumerate(kv_list):
        for lb in range(nblk[r]):
            pb = perm[pos]
            pos += 1
            table[r, lb] = pb
            seg = x[:, lb * bs : (lb + 1) * bs]
            cache[pb, :, : seg.shape[1]] = seg
    return cache, table


def test_paged_decode_equals_dense_on_contiguous_kv():
    rng = np.random.default_rng(16)
    R, Hq, Hkv, d, bs = 4, 6, 2, 5, 4
    ctx = [1, 4, 5, 13]
    ks = [rng.standard_normal((Hkv, n, d)) for n in ctx]
    vs = [rng.standard_normal((Hkv, n, d)) for n in ctx]
    q = rng.standard_normal((R, Hq, d))
    kc, table = _scatter_to_pages(ks, bs, Hkv, d, np.random.default_rng(1))
    vc, table2 = _scatter_to_pages(vs, bs, Hkv, d, np.random.default_rng(1))
    assert np.array_equal(table, table2)
    O, lse = ora.paged_decode(q, kc, vc, table, ctx, bs, 0.4)
    for r in range(R):
        for h in range(Hq):
            o, l, _ = ora.attention_head(q[r, h][None], ks[r][h // 3], vs[r][h // 3], 0.4)
            np.testing.assert_allclose(O[r, h], o[0], atol=1e-14)
            np.testing.assert_allclose(lse[r, h], l[0], atol=1e-14)
    assert np.isfinite(O).all()  # unused (NaN) slots never reach the result
    # a different physical placement of the same logical cache changes nothing
    kc2, t2 = _scatter_to_pages(ks, bs, Hkv, d, np.random.default_rng(2))
    vc2, _ = _scatter_to_pages(vs, bs, Hkv, d, np.random.default_rng(2))
    O2, lse2 = ora.paged_decode(q, kc2, vc2, t2, ctx, bs, 0.4)
    np.testing.assert_allclose(O2, O, atol=1e-15)
    with pytest.raises(ValueError):
        ora.paged_decode(q, kc, vc, table, [0, 4, 5, 13], bs, 0.4)


def test_merge_partials_equals_whole_softmax():
    rng = np.random.default_rng(17)
    q, k, v = rng.standard_normal((1, 4)), rng.standard_normal((30, 4)), rng.standard_normal((30, 4))
    O, lse, _ = ora.attention_head(q, k, v, 0.5)
    cuts = [0, 7, 8, 21, 30]
    parts = [ora.attention_head(q, k[a:b], v[a:b], 0.5) for a, b in zip(cuts[:-1], cuts[1:])]
    o, l = ora.merge_partials([p[1][0] for p in parts], [p[0][0] for p in parts])
    np.testing.assert_allclose(o, O[0], atol=1e-14)
    assert l == pytest.approx(lse[0], abs=1e-14)


# ---------------------------------------------------------------------------------
# Planted mistakes: each plausible slip in the oracle is caught by some pin above
# ---------------------------------------------------------------------------------
def _pins_pass():
    checks = [
        test_worked_example_direct_definition,
        test_rows_sum_to_one_and_lse_is_logsumexp,
        test_scale_enters_as_inverse_sqrt_dk,
        test_forward_matches_torch_fp64_library_attention,
        test_gradients_match_torch_fp64_autograd,
        test_causal_bottom_right_alignment_for_shorter_query,
        test_gqa_equals_explicitly_repeated_heads,
        test_gradient_invariants,
    ]
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            return False
    return True


def test_planted_mistakes_are_caught(monkeypatch):
    assert _pins_pass()
    good_scores = ora.scaled_scores
    good_allowed = ora.causal_allowed
    good_bwd = ora.attention_bwd_head

    mutations = {
        "scale dropped": ("scaled_scores", lambda q, k, s: q @ k.T),
        "scale squared": ("scaled_scores", lambda q, k, s: s * s * (q @ k.T)),
        "sign flipped": ("scaled_scores", lambda q, k, s: -good_scores(q, k, s)),
        "top-left causal": ("causal_allowed", lambda nq, nkv: np.arange(nkv)[None, :] <= np.arange(nq)[:, None]),
        "strict causal": ("causal_allowed", lambda nq, nkv: good_allowed(nq, nkv) & ~np.eye(nq, nkv, nkv - nq, dtype=bool)),
    }

    def bwd_no_D(qh, kh, vh, doh, scale, causal=False):
        O, _, P = ora.attention_head(qh, kh, vh, scale, causal)
        dS = P * (doh @ vh.T)
        return scale * dS @ kh, scale * dS.T @ qh, P.T @ doh

    def bwd_untransposed_dv(qh, kh, vh, doh, scale, causal=False):
        dq, dk, _ = good_bwd(qh, kh, vh, doh, scale, causal)
        _, _, P = ora.attention_head(qh, kh, vh, scale, causal)
        return dq, dk, P @ doh

    for label, (attr, fn) in mutations.items():
        monkeypatch.setattr(ora, attr, fn)
        assert not _pins_pass(), label
        monkeypatch.undo()
    for label, fn in (("D term dropped", bwd_no_D), ("P not transposed in dV", bwd_untransposed_dv)):
        monkeypatch.setattr(ora, "attention_bwd_head", fn)
        assert not _pins_pass(), label
        monkeypatch.undo()
    assert _pins_pass()


def test_paged_append_token_by_token_rebuilds_the_sequence():
    """Appending a sequence one token at a time into an empty paged cache, then de-paging,
    gives back the sequence (the cache grows one token at a time through the table)."""
    rng = np.random.default_rng(18)
    Hkv, d, bs, n = 2, 3, 4, 13
    seq_k = rng.standard_normal((n, Hkv, d))
    seq_v = rng.standard_normal((n, Hkv, d))
    nblk = (n + bs - 1) // bs
    table = np.full((1, nblk + 1), -1)
    table[0, :nblk] = rng.permutation(10)[:nblk]
    kc = np.zeros((10, Hkv, bs, d))
    vc = np.zeros((10, Hkv, bs, d))
    for t in range(n):
        kc, vc = ora.paged_append(kc, vc, table, [t], seq_k[t][None], seq_v[t][None], bs)
    for g in range(Hkv):
        np.testing.assert_array_equal(ora.depage(kc, table[0], n, g, bs), seq_k[:, g])
        np.testing.assert_array_equal(ora.depage(vc, table[0], n, g, bs), seq_v[:, g])
    # untouched blocks stay untouched
    used = set(int(x) for x in table[0, :nblk])
    for b in range(10):
        if b not in used:
            assert not kc[b].any()


def test_paged_prefill_equals_dense_and_decode():
    """Full prefill from pages equals dense attention on the contiguous K/V; a one-row
    prefill equals the decode step; rows past q_len are not part of the result."""
    rng = np.random.default_rng(19)
    R, Hq, Hkv, d, bs = 3, 4, 2, 3, 4
    ctx = [1, 9, 13]
    ks = [rng.standard_normal((Hkv, n, d)) for n in ctx]
    vs = [rng.standard_normal((Hkv, n, d)) for n in ctx]
    kc, table = _scatter_to_pages(ks, bs, Hkv, d, np.random.default_rng(3))
    vc, _ = _scatter_to_pages(vs, bs, Hkv, d, np.random.default_rng(3))
    nq_max = 13
    q = rng.standard_normal((R, Hq, nq_max, d))
    for causal in (False, True):
        O, L = ora.paged_prefill(q, kc, vc, table, ctx, ctx, bs, 0.5, causal)  # q_len = ctx
        for r in range(R):
            Od, Ld = ora.attention_fwd(q[r:r + 1, :, :ctx[r]], ks[r][None], vs[r][None], 0.5, causal)
            np.testing.assert_allclose(O[r, :, :ctx[r]], Od[0], atol=1e-14)
            np.testing.assert_allclose(L[r, :, :ctx[r]], Ld[0], atol=1e-14)
            assert np.isnan(O[r, :, ctx[r]:]).all()
    # one query row at the end of each sequence is the decode step (causal or not)
    O1, L1 = ora.paged_prefill(q, kc, vc, table, ctx, [1, 1, 1], bs, 0.5, True)
    Od, Ldd = ora.paged_decode(q[:, :, 0], kc, vc, table, ctx, bs, 0.5)
    np.testing.assert_allclose(O1[:, :, 0], Od, atol=1e-14)
    np.testing.assert_allclose(L1[:, :, 0], Ldd, atol=1e-14)
    with pytest.raises(ValueError):
        ora.paged_prefill(q, kc, vc, table, ctx, [2, 10, 3], bs, 0.5, True)


def test_paged_prefill_chunk_equals_last_rows_of_whole_prompt():
    """A prompt chunk (the last q_len < ctx positions of a sequence whose earlier part is
    cached) gives exactly the last q_len rows of the whole prompt's result, causal or not:
    each chunk row sees the cached prefix and the chunk up to its own position."""
    rng = np.random.default_rng(23)
    Hq, Hkv, d, bs = 4, 2, 3, 4
    ctx, qlen = [5, 9, 13], [2, 4, 7]
    R = len(ctx)
    ks = [rng.standard_normal((Hkv, n, d)) for n in ctx]
    vs = [rng.standard_normal((Hkv, n, d)) for n in ctx]
    kc, table = _scatter_to_pages(ks, bs, Hkv, d, np.random.default_rng(5))
    vc, _ = _scatter_to_pages(vs, bs, Hkv, d, np.random.default_rng(5))
    qw = rng.standard_normal((R, Hq, max(ctx), d))
    qc = np.zeros((R, Hq, max(qlen), d))
    for r in range(R):
        qc[r, :, :qlen[r]] = qw[r, :, ctx[r] - qlen[r]:ctx[r]]
    for causal in (False, True):
        Ow, Lw = ora.paged_prefill(qw, kc, vc, table, ctx, ctx, bs, 0.5, causal)
        Oc, Lc = ora.paged_prefill(qc, kc, vc, table, ctx, qlen, bs, 0.5, causal)
        for r in range(R):
            np.testing.assert_allclose(Oc[r, :, :qlen[r]], Ow[r, :, ctx[r] - qlen[r]:ctx[r]], atol=1e-14)
            np.testing.assert_allclose(Lc[r, :, :qlen[r]], Lw[r, :, ctx[r] - qlen[r]:ctx[r]], atol=1e-14)
    # and the causal chunk is not the non-causal one (the mask reaches into the chunk)
    Oc0, _ = ora.paged_prefill(qc, kc, vc, table, ctx, qlen, bs, 0.5, False)
    Oc1, _ = ora.paged_prefill(qc, kc, vc, table, ctx, qlen, bs, 0.5, True)
    assert not np.allclose(Oc0[2, :, :qlen[2] - 1], Oc1[2, :, :qlen[2] - 1])


def test_single_key_gradients_are_zero_in_the_oracle():
    """With one key every softmax row is [1], so dS = P (dP - D) = 0 and dQ = dK = 0 up to
    fp64 rounding (the case the parity checker compares by max-abs only)."""
    import sys
    import os
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    from parity import _exactly_zero

    rng = np.random.default_rng(3)
    q, k, v, do = (rng.standard_normal((1, 1, n, 8)) for n in (5, 1, 1, 5))
    dq, dk, dv = ora.attention_bwd(q, k, v, do, 0.3, False)
    assert _exactly_zero(dq) and _exactly_zero(dk)
    assert np.allclose(dv[0, 0, 0], do[0, 0].sum(axis=0))
    assert not _exactly_zero(dv)
