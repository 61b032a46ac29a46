"""Plain, slow fp64 CPU oracle for exact attention.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
It shares no code with the CUDA path (no kernels, no headers, no helpers): it is the
definition of the operation written out in NumPy float64, materialising the full
score matrix exactly as the unfused "standard attention" the pages describe.

Sources (three web pages, cited by title and section):
  [AK] "Autoatención, kernels CUDA y FlashAttention" (spanish.itimpress.au),
       §1 "Cómo funciona matemáticamente la autoatención en un transformador de visión"
       and §3 "FlashAttention: solución al cuello de botella de memoria de los Transformers".
  [FA] "FlashAttention" (paweldubiel.com notes), "Mecanismo y detalles" and
       "No basta con promediar los resultados de los bloques".
  [KR] "Kernels de atención rápida y fusión de operadores" (the-ai.news),
       "Atención tipo FlashAttention y atención paginada".

Readings where the pages are silent (the plainest reading the rest of the pages supports):
  * LSE is ``m + ln(l)`` over the *scaled* scores, natural log.
  * GQA maps query head h to key/value head ``h // (Hq // Hkv)`` (contiguous groups).
  * Causal masking is bottom-right aligned: query i sits at key position
    ``Nkv - Nq + i`` and may attend keys j <= that position.
  * Paged decode: the single query token attends to all ``ctx_len`` cached tokens.
  * The gradients are the textbook matrix-calculus gradients of the definition.

Every function is pinned by tests that do not re-type its formula: the pages' worked
example (0.75), closed forms, brute-force block merges, finite differences, and an
independent library routine (torch's fp64 CPU attention).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "to_f64",
    "scaled_scores",
    "causal_allowed",
    "attention_head",
    "attention_fwd",
    "attention_fwd_rows",
    "attention_bwd_head",
    "attention_bwd",
    "depage",
    "paged_decode",
    "online_softmax_blocks",
    "merge_partials",
    "paged_append",
    "paged_prefill",
]


def to_f64(x) -> np.ndarray:
    """Upcast the values as actually stored (fp32 or bf16) to float64, exactly."""
    try:  # torch tensor (bf16 has no NumPy dtype, so go through fp32: exact)
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def scaled_scores(qh: np.ndarray, kh: np.ndarray, scale: float) -> np.ndarray:
    """S = scale * Q K^T for one head ([AK] §1, "Scores=(QK^T)/sqrt(d_k)").

    The full Nq x Nkv matrix is materialised, as in the unfused form of [AK] §3.
    """
    return scale * (qh @ kh.T)


def causal_allowed(nq: int, nkv: int) -> np.ndarray:
    """Boolean [nq, nkv]: query i may see key j iff j <= i + (nkv - nq).

    Causal masking is not on the pages; this is the bottom-right reading, which is
    the usual top-left mask when nq == nkv and makes decode the nq == 1 case.
    """
    i = np.arange(nq)[:, None]
    j = np.arange(nkv)[None, :]
    return j <= i + (nkv - nq)


def attention_head(qh, kh, vh, scale: float, causal: bool = False):
    """Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V for one head ([AK] §1).

    Returns (O [nq,d], lse [nq], P [nq,nkv]).  The row softmax is taken the
    numerically stable way (subtract the row maximum) which is exact in real
    arithmetic; ``lse = m + ln(sum_j e^{s_j - m})`` ([FA] "No basta con promediar").
    """
    qh = np.asarray(qh, dtype=np.float64)
    kh = np.asarray(kh, dtype=np.float64)
    vh = np.asarray(vh, dtype=np.float64)
    S = scaled_scores(qh, kh, scale)
    if causal:
        S = np.where(causal_allowed(S.shape[0], S.shape[1]), S, -np.inf)
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    l = E.sum(axis=1)
    P = E / l[:, None]
    O = P @ vh
    lse = m + np.log(l)
    return O, lse, P


def _check_gqa(hq: int, hkv: int) -> int:
    if hkv <= 0 or hq % hkv != 0:
        raise ValueError(f"Hq={hq} must be a positive multiple of Hkv={hkv}")
    return hq // hkv


def attention_fwd(q, k, v, scale: float, causal: bool = False):
    """Multi-head forward, q [B,Hq,Nq,d], k/v [B,Hkv,Nkv,d] -> (O [B,Hq,Nq,d], lse [B,Hq,Nq]).

    Heads are independent ([AK] §1: the same process runs in parallel over heads);
    grouped-query attention shares one K/V head among G = Hq/Hkv query heads
    ([FA] "Mecanismo y detalles", last paragraph).
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, Hq, Nq, d = q.shape
    G = _check_gqa(Hq, k.shape[1])
    O = np.empty((B, Hq, Nq, v.shape[-1]))
    lse = np.empty((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            O[b, h], lse[b, h], _ = attention_head(q[b, h], k[b, h // G], v[b, h // G], scale, causal)
    return O, lse


def attention_fwd_rows(q, k, v, scale: float, causal: bool, b: int, h: int, rows):
    """Forward for selected query rows of one (b, h) head.

    Rows of the forward pass are independent, so this is exact for those rows.  The
    causal mask uses each row's own index in the full sequence.
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    G = _check_gqa(q.shape[1], k.shape[1])
    rows = np.asarray(rows, dtype=np.int64)
    Nq, Nkv = q.shape[2], k.shape[2]
    qh = q[b, h][rows]
    kh, vh = k[b, h // G], v[b, h // G]
    S = scaled_scores(qh, kh, scale)
    if causal:
        allowed = np.arange(Nkv)[None, :] <= (rows[:, None] + (Nkv - Nq))
        S = np.where(allowed, S, -np.inf)
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    l = E.sum(axis=1)
    O = (E / l[:, None]) @ vh
    return O, m + np.log(l)


def attention_bwd_head(qh, kh, vh, doh, scale: float, causal: bool = False):
    """Gradients of sum(O * dO) for one head, by matrix calculus on the definition.

    The pages say only that the backward pass recomputes the attention blocks from
    saved normalisation statistics ([AK] §3 "Recálculo durante la retropropagación";
    [FA] "Mecanismo y detalles").  The quantities recomputed are these:
        P = softmax(S),  dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
        dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
    Returns (dq, dk, dv) for this head.
    """
    O, _, P = attention_head(qh, kh, vh, scale, causal)
    doh = np.asarray(doh, dtype=np.float64)
    dv = P.T @ doh
    dP = doh @ np.asarray(vh, dtype=np.float64).T
    D = (doh * O).sum(axis=1)
    dS = P * (dP - D[:, None])
    dq = scale * (dS @ np.asarray(kh, dtype=np.float64))
    dk = scale * (dS.T @ np.asarray(qh, dtype=np.float64))
    return dq, dk, dv


def attention_bwd(q, k, v, do, scale: float, causal: bool = False, heads=None):
    """Multi-head backward -> (dq [B,Hq,Nq,d], dk, dv [B,Hkv,Nkv,d]).

    dK and dV of a key/value head are summed over the G query heads that share it.
    ``heads`` optionally restricts the computation to a list of (b, hkv) groups; the
    other entries are left as NaN so that a caller cannot mistake them for results.
    """
    q, k, v, do = to_f64(q), to_f64(k), to_f64(v), to_f64(do)
    B, Hq, Nq, d = q.shape
    Hkv = k.shape[1]
    G = _check_gqa(Hq, Hkv)
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    groups = heads if heads is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for b, g in groups:
        dk[b, g] = 0.0
        dv[b, g] = 0.0
        for h in range(g * G, (g + 1) * G):
            dqh, dkh, dvh = attention_bwd_head(q[b, h], k[b, g], v[b, g], do[b, h], scale, causal)
            dq[b, h] = dqh
            dk[b, g] += dkh
            dv[b, g] += dvh
    return dq, dk, dv


def depage(cache, table_row, ctx_len: int, kv_head: int, block_size: int) -> np.ndarray:
    """Contiguous [ctx_len, d] keys (or values) of one request and one KV head.

    Logical token t lives in physical block ``table_row[t // block_size]`` at slot
    ``t % block_size`` ([KR] "Atención tipo FlashAttention y atención paginada": the
    block table links logical positions to fixed-size physical blocks).  The cache
    layout is [num_blocks, Hkv, block_size, d].
    """
    cache = to_f64(cache)
    out = np.empty((ctx_len, cache.shape[-1]))
    for t in range(ctx_len):
        out[t] = cache[int(table_row[t // block_size]), kv_head, t % block_size]
    return out


def paged_decode(q, k_cache, v_cache, block_table, ctx_lens, block_size: int, scale: float):
    """One decode step over a paged KV cache -> (O [R,Hq,d], lse [R,Hq]).

    q is [R, Hq, d] (one new token per request).  The cache is de-paged request by
    request and then run through the dense definition with Nq = 1, non-causal, over
    the ctx_len cached tokens.
    """
    q = to_f64(q)
    k_cache, v_cache = to_f64(k_cache), to_f64(v_cache)
    table = np.asarray(block_table)
    ctx = np.asarray(ctx_lens)
    R, Hq, d = q.shape
    G = _check_gqa(Hq, k_cache.shape[1])
    O = np.empty((R, Hq, v_cache.shape[-1]))
    lse = np.empty((R, Hq))
    for r in range(R):
        n = int(ctx[r])
        if n <= 0:
            raise ValueError("every request needs at least one cached token")
        for g in range(k_cache.shape[1]):
            kr = depage(k_cache, table[r], n, g, block_size)
            vr = depage(v_cache, table[r], n, g, block_size)
            for h in range(g * G, (g + 1) * G):
                o, l, _ = attention_head(q[r, h][None, :], kr, vr, scale, causal=False)
                O[r, h], lse[r, h] = o[0], l[0]
    return O, lse


def online_softmax_blocks(score_blocks, value_blocks):
    """The pages' blockwise recurrence for one query ([FA] "No basta con promediar").

    Keeps the running maximum m, the sum l = sum_j e^{s_j - m} and the numerator
    u = sum_j e^{s_j - m} v_j.  When a block raises the maximum to m', the old l and
    u are multiplied by e^{m - m'} before the block's own terms are added.  The
    result is u / l.  Returns (u / l, m, l).
    """
    m = -np.inf
    l = 0.0
    u = None
    for s_blk, v_blk in zip(score_blocks, value_blocks):
        s_blk = np.asarray(s_blk, dtype=np.float64)
        v_blk = np.asarray(v_blk, dtype=np.float64)
        if v_blk.ndim == 1:
            v_blk = v_blk[:, None]
        m_new = max(m, float(s_blk.max()))
        alpha = np.exp(m - m_new) if np.isfinite(m) else 0.0
        w = np.exp(s_blk - m_new)
        l = alpha * l + w.sum()
        u_blk = (w[:, None] * v_blk).sum(axis=0)
        u = u_blk if u is None else alpha * u + u_blk
        m = m_new
    return u / l, m, l


def merge_partials(lse_parts, o_parts):
    """Combine normalised partial results of disjoint key sets.

    Each part s carries its own normalised output O_s and lse_s = m_s + ln l_s.  The
    parts are weighted by their unnormalised mass e^{lse_s}, not averaged ([FA]
    "No basta con promediar los resultados de los bloques").  Returns (O, lse).
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    o_parts = np.asarray(o_parts, dtype=np.float64)
    top = lse_parts.max()
    w = np.exp(lse_parts - top)
    lse = top + np.log(w.sum())
    O = (w[:, None] * o_parts.reshape(len(lse_parts), -1)).sum(axis=0) / w.sum()
    return O.reshape(o_parts.shape[1:]), lse


def paged_append(k_cache, v_cache, block_table, positions, k_new, v_new, block_size: int):
    """The caches after appending one token per request ([KR] "Atención tipo FlashAttention
    y atención paginada": the cache grows one token at a time; the block table links the
    logical position to a physical block).  Request r's new key/value for every KV head
    goes to block ``block_table[r][pos // block_size]``, slot ``pos % block_size``.  Works
    on copies of the stored values (no arithmetic); returns (k_cache, v_cache)."""
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    table = np.asarray(block_table)
    for r, pos in enumerate(np.asarray(positions)):
        pb = int(table[r, int(pos) // block_size])
        kc[pb, :, int(pos) % block_size] = np.asarray(k_new)[r]
        vc[pb, :, int(pos) % block_size] = np.asarray(v_new)[r]
    return kc, vc


def paged_prefill(q, k_cache, v_cache, block_table, ctx_lens, q_lens, block_size: int, scale: float,
                  causal: bool):
    """Prefill over a paged KV cache -> (O [R,Hq,Nq_max,d], lse [R,Hq,Nq_max]).

    [KR] "Atención tipo FlashAttention y atención paginada" joins blockwise prefill with
    the paged cache.  Request r has ``ctx_lens[r]`` cached tokens (de-paged through its
    block-table row) and ``q_lens[r]`` query rows, which are the last ``q_lens[r]``
    positions of its sequence (bottom-right causal alignment).  Rows at and past
    ``q_lens[r]`` are left as NaN: they are not part of the result.
    """
    q = to_f64(q)
    k_cache, v_cache = to_f64(k_cache), to_f64(v_cache)
    table = np.asarray(block_table)
    R, Hq, Nq_max, d = q.shape
    G = _check_gqa(Hq, k_cache.shape[1])
    O = np.full((R, Hq, Nq_max, v_cache.shape[-1]), np.nan)
    lse = np.full((R, Hq, Nq_max), np.nan)
    for r in range(R):
        n, nq = int(np.asarray(ctx_lens)[r]), int(np.asarray(q_lens)[r])
        if not (1 <= nq <= n):
            raise ValueError("need 1 <= q_len <= ctx_len")
        for g in range(k_cache.shape[1]):
            kr = depage(k_cache, table[r], n, g, block_size)
            vr = depage(v_cache, table[r], n, g, block_size)
            for h in range(g * G, (g + 1) * G):
                O[r, h, :nq], lse[r, h, :nq], _ = attention_head(q[r, h, :nq], kr, vr, scale, causal)
    return O, lse
