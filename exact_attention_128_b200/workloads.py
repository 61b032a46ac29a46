"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path's tests/benchmarks and the fp64 oracle
can consume the same stored tensors.  Every tensor is drawn on the CPU from
``torch.Generator().manual_seed(seed)`` as N(0, 1) in fp32 and then cast
(round-to-nearest-even) to the workload's dtype; the oracle upcasts the stored
values exactly.

Shapes follow the pages' examples: a ViT-B/16 layer (N = 196 patches of a 224x224
image, 12 heads of d_k = 64; "Autoatención, kernels CUDA y FlashAttention" §1), a
long causal GQA prefill, a training step, and a paged decode step with 16-token
blocks ("Kernels de atención rápida ...", "Atención tipo FlashAttention y atención
paginada", which uses a 1.5B-class decoder with block_size = 16).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def randn(shape, seed: int, dtype: torch.dtype) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)


@dataclass
class DenseCase:
    """One dense attention problem: q [B,Hq,N,d], k/v [B,Hkv,N,d] (Nq may differ)."""

    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nkv: int
    d: int
    dtype: str
    causal: bool
    seed: int
    scale: float = field(default=float("nan"))

    def __post_init__(self):
        if math.isnan(self.scale):
            self.scale = 1.0 / math.sqrt(self.d)

    @property
    def torch_dtype(self) -> torch.dtype:
        return DTYPES[self.dtype]

    def make(self, with_grad_output: bool = False):
        """Return (q, k, v[, do]) as CPU tensors of the case's dtype."""
        t = self.torch_dtype
        s = self.seed * 1000
        q = randn((self.B, self.Hq, self.Nq, self.d), s + 1, t)
        k = randn((self.B, self.Hkv, self.Nkv, self.d), s + 2, t)
        v = randn((self.B, self.Hkv, self.Nkv, self.d), s + 3, t)
        if with_grad_output:
            do = randn((self.B, self.Hq, self.Nq, self.d), s + 4, t)
            return q, k, v, do
        return q, k, v

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4*d per allowed (query, key) pair, per head."""
        return 4.0 * self.d * self.B * self.Hq * self.allowed_pairs()

    def allowed_pairs(self) -> int:
        if not self.causal:
            return self.Nq * self.Nkv
        off = self.Nkv - self.Nq
        # query i sees keys 0 .. i + off
        return sum(min(self.Nkv, i + off + 1) for i in range(self.Nq))


# The ViT-B/16 layer in fp32 (N = 196, 12 heads, d_k = 64, scale 1/8).
VIT_LAYER_F32 = DenseCase("vit_b16_layer_fwd_f32", 1, 12, 12, 196, 196, 64, "f32", False, 1, 0.125)
# The same layer batched over 64 images in bf16.
VIT_BATCHED_BF16 = DenseCase("vit_b16_batched_fwd_bf16", 64, 12, 12, 196, 196, 64, "bf16", False, 2, 0.125)
# Long causal GQA prefill: 32 query heads share 8 K/V heads, d = 128.
GQA_PREFILL_CAUSAL = DenseCase("gqa_prefill_causal_n8192", 4, 32, 8, 8192, 8192, 128, "bf16", True, 3)
# Training step, causal, 16 heads of d = 64.
TRAIN_CAUSAL = DenseCase("train_fwd_bwd_causal_n4096", 8, 16, 16, 4096, 4096, 64, "bf16", True, 4, 0.125)
# Other head dimensions at the prefill sweep's N = 4096 (B*N = 32768 for d = 96).
D96_PREFILL = DenseCase("d96_prefill_noncausal_n4096", 8, 32, 8, 4096, 4096, 96, "bf16", False, 5)
D256_PREFILL = DenseCase("d256_prefill_noncausal_n4096", 4, 16, 4, 4096, 4096, 256, "bf16", False, 7)
# Training step at head dimension 256 (causal, GQA 16/4): the same forward FLOPs as the
# d = 64 training step, a quarter of its heads.
D256_TRAIN = DenseCase("d256_train_fwd_bwd_causal_n4096", 2, 16, 4, 4096, 4096, 256, "bf16", True, 8)


def prefill_sweep():
    """Non-causal sweep at B*N = 32768 with the GQA prefill's heads and d."""
    out = []
    for i, n in enumerate((1024, 2048, 4096, 8192, 16384)):
        out.append(DenseCase(f"gqa_prefill_noncausal_n{n}", 32768 // n, 32, 8, n, n, 128, "bf16", False, 30 + i))
    return out


def paged_pool(ctx, block_size: int, max_blocks_per_seq: int, Hkv: int, d: int, g: torch.Generator, s: int,
               poison_unused: bool):
    """Lay R sequences of ``ctx`` tokens out in a paged K/V pool.

    The pool holds exactly sum_r ceil(ctx_r / block_size) blocks; a random permutation
    (drawn from ``g``) assigns a physical id to each (request, logical block) pair in
    order.  Table entries past a request's last block are -1.  Caches are
    [blocks, Hkv, block_size, d] bf16 drawn with seeds s + 2 (K) and s + 3 (V).  With
    ``poison_unused`` the unused slots of each request's last block hold NaN.
    Returns (table, k_cache, v_cache, num_blocks).
    """
    R = len(ctx)
    nblk = [(int(c) + block_size - 1) // block_size for c in ctx]
    total = sum(nblk)
    if max(nblk) > max_blocks_per_seq:
        raise ValueError("context longer than the block table allows")
    perm = torch.randperm(total, generator=g)
    table = torch.full((R, max_blocks_per_seq), -1, dtype=torch.int32)
    pos = 0
    for r in range(R):
        table[r, : nblk[r]] = perm[pos : pos + nblk[r]].to(torch.int32)
        pos += nblk[r]
    kc = randn((total, Hkv, block_size, d), s + 2, torch.bfloat16)
    vc = randn((total, Hkv, block_size, d), s + 3, torch.bfloat16)
    if poison_unused:
        for r in range(R):
            used = int(ctx[r]) - (nblk[r] - 1) * block_size
            if used < block_size:
                pb = int(table[r, nblk[r] - 1])
                kc[pb, :, used:, :] = float("nan")
                vc[pb, :, used:, :] = float("nan")
    return table, kc, vc, total


@dataclass
class PagedCase:
    """One paged-KV decode step: R requests with one new query token each."""

    name: str
    R: int
    Hq: int
    Hkv: int
    d: int
    block_size: int
    ctx_min: int
    ctx_max: int
    max_blocks_per_seq: int
    seed: int
    ctx_lens_override: tuple | None = None

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def make(self, poison_unused: bool = False):
        """Return dict with q, k_cache, v_cache, block_table, ctx_lens (CPU tensors).

        ctx_r ~ U{ctx_min..ctx_max} (inclusive, seeded).  The pool holds exactly
        sum_r ceil(ctx_r / block_size) blocks; a seeded random permutation assigns a
        physical id to each (request, logical block) pair in order.  Table entries
        past a request's last block are -1.  With ``poison_unused`` the unused slots
        of each request's last block hold NaN (a correct kernel never reads them
        into the result).
        """
        g = torch.Generator().manual_seed(self.seed * 1000)
        if self.ctx_lens_override is not None:
            ctx = torch.tensor(self.ctx_lens_override, dtype=torch.int32)
        else:
            ctx = torch.randint(self.ctx_min, self.ctx_max + 1, (self.R,), generator=g, dtype=torch.int64).to(torch.int32)
        table, kc, vc, total = paged_pool(ctx, self.block_size, self.max_blocks_per_seq, self.Hkv, self.d, g,
                                          self.seed * 1000, poison_unused)
        q = randn((self.R, self.Hq, self.d), self.seed * 1000 + 1, torch.bfloat16)
        return {"q": q, "k_cache": kc, "v_cache": vc, "block_table": table, "ctx_lens": ctx, "num_blocks": total}

    @staticmethod
    def kv_bytes(ctx_lens, Hkv: int, d: int) -> int:
        """Algorithmic K+V bytes of one decode step: every cached token's K and V row, bf16."""
        return int(sum(int(c) for c in ctx_lens)) * Hkv * d * 2 * 2


# 1.5B-class decoder decode step: 64 requests, Hq = 12, Hkv = 2, d = 128, 16-token blocks.
PAGED_DECODE = PagedCase("paged_decode_r64_hq12_hkv2_d128_bs16", 64, 12, 2, 128, 16, 512, 8192, 512, 5)


@dataclass
class PagedPrefillCase:
    """A batch of variable-length prefills over a paged KV cache.

    Request r has ctx_r cached tokens and q_r query rows, the last q_r positions of its
    sequence: q_r = ctx_r for a whole prompt (``q_frac`` = 1), else a seeded chunk
    length q_r ~ U{1..max(1, round(q_frac * ctx_r))}.  q is [R, Hq, Nq_max, d] with
    Nq_max = max_r q_r; rows past q_r are padding.
    """

    name: str
    R: int
    Hq: int
    Hkv: int
    d: int
    block_size: int
    ctx_min: int
    ctx_max: int
    max_blocks_per_seq: int
    causal: bool
    seed: int
    q_frac: float = 1.0
    ctx_lens_override: tuple | None = None
    q_lens_override: tuple | None = None

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def lengths(self):
        g = torch.Generator().manual_seed(self.seed * 1000)
        if self.ctx_lens_override is not None:
            ctx = torch.tensor(self.ctx_lens_override, dtype=torch.int32)
        else:
            ctx = torch.randint(self.ctx_min, self.ctx_max + 1, (self.R,), generator=g, dtype=torch.int64).to(torch.int32)
        if self.q_lens_override is not None:
            ql = torch.tensor(self.q_lens_override, dtype=torch.int32)
        elif self.q_frac >= 1.0:
            ql = ctx.clone()
        else:
            hi = [max(1, round(self.q_frac * int(c))) for c in ctx]
            ql = torch.tensor([int(torch.randint(1, h + 1, (1,), generator=g)) for h in hi], dtype=torch.int32)
        return ctx, ql, g

    def make(self, poison: bool = False):
        """Return dict with q, k_cache, v_cache, block_table, ctx_lens, q_lens, num_blocks (CPU).

        With ``poison`` the unused cache slots of each last block and the padding query
        rows hold NaN (a correct kernel never reads them into the result)."""
        ctx, ql, g = self.lengths()
        s = self.seed * 1000
        table, kc, vc, total = paged_pool(ctx, self.block_size, self.max_blocks_per_seq, self.Hkv, self.d, g, s,
                                          poison)
        nq_max = int(ql.max())
        q = randn((self.R, self.Hq, nq_max, self.d), s + 1, torch.bfloat16)
        if poison:
            for r in range(self.R):
                q[r, :, int(ql[r]):, :] = float("nan")
        return {"q": q, "k_cache": kc, "v_cache": vc, "block_table": table, "ctx_lens": ctx, "q_lens": ql,
                "num_blocks": total}

    def allowed_pairs(self) -> int:
        """(query, key) pairs the prefill computes, summed over requests (per head)."""
        ctx, ql, _ = self.lengths()
        tot = 0
        for c, n in zip(ctx.tolist(), ql.tolist()):
            tot += n * (2 * c - n + 1) // 2 if self.causal else n * c
        return tot

    def fwd_flops(self) -> float:
        return 4.0 * self.d * self.Hq * self.allowed_pairs()

    def io_bytes(self) -> int:
        """Algorithmic bytes: every cached K/V row once per KV head, q and o rows once (bf16)."""
        ctx, ql, _ = self.lengths()
        return int(ctx.sum()) * self.Hkv * self.d * 2 * 2 + int(ql.sum()) * self.Hq * self.d * 2 * 2


# Paged counterpart of the causal GQA prefill: 8 whole prompts of U{2048..8192} tokens,
# Hq = 32, Hkv = 8, d = 128, 16-token blocks.
PAGED_PREFILL = PagedPrefillCase("paged_prefill_r8_hq32_hkv8_d128_bs16_causal", 8, 32, 8, 128, 16, 2048, 8192, 512,
                                 True, 6)
