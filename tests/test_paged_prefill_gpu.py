"""Paged, variable-length prefill: CUDA kernel vs the fp64 oracle (de-paged dense attention)."""
import numpy as np
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import PAGED_PREFILL, PagedPrefillCase
from oracle import attention_fp64 as ora
from parity import check_bf16, check_lse

pytestmark = pytest.mark.gpu

NAMES = ("q", "k_cache", "v_cache", "block_table", "ctx_lens", "q_lens")
PER_REQUEST = ("q", "block_table", "ctx_lens", "q_lens")


def run(inp, causal):
    o, lse = fa.paged_prefill(*(inp[n].cuda() for n in NAMES), causal=causal)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def check_rows(o, lse, O, L, q_lens, what):
    """Compare the defined rows (i < q_lens[r]) of every request."""
    for r, n in enumerate(q_lens.tolist()):
        check_bf16(o[r, :, :n], O[r, :, :n], f"{what} O r={r}")
        check_lse(lse[r, :, :n], L[r, :, :n], f"{what} lse r={r}")


def oracle(inp, causal):
    d = inp["q"].shape[-1]
    return ora.paged_prefill(inp["q"], inp["k_cache"], inp["v_cache"], inp["block_table"], inp["ctx_lens"],
                             inp["q_lens"], 16, 1.0 / np.sqrt(d), causal)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize(
    "d,Hq,Hkv,ctx,ql",
    [
        # whole prompts: ragged tails inside a cache block, inside a 128-key tile, single tokens
        (128, 4, 2, (300, 17, 1000, 1), None),
        # chunks: the last q_len positions of a longer cached sequence
        (128, 4, 2, (300, 17, 1000, 513), (45, 17, 1, 257)),
        (128, 8, 8, (129, 640), (128, 100)),
        (64, 6, 2, (300, 65, 777), None),
        (64, 4, 1, (1000, 200, 33), (1000, 1, 7)),
        (96, 4, 2, (300, 17, 500), (300, 9, 129)),
        # whole cache blocks, but a partial key tile: no slot tail, blocks past the sequence
        (128, 4, 2, (96, 160, 16), None),
        (64, 4, 2, (48, 96, 208), (48, 3, 100)),
    ],
)
def test_paged_prefill_vs_oracle(d, Hq, Hkv, ctx, ql, causal):
    pc = PagedPrefillCase("edge", len(ctx), Hq, Hkv, d, 16, 1, 8192, 128, causal, 60 + Hq + d,
                          ctx_lens_override=ctx, q_lens_override=ql)
    inp = pc.make(poison=True)  # NaN in unused cache slots and padding query rows
    fa.device_status(reset=True)
    o, lse = run(inp, causal)
    assert fa.device_status() == 0
    O, L = oracle(inp, causal)
    check_rows(o, lse, O, L, inp["q_lens"], f"d={d}")


@pytest.mark.parametrize(
    "d,Hq,Hkv,width,ctx,ql",
    [
        # the causal item order takes requests in groups whose K/V, bounded by the block
        # table's width, fits 32 MB: Hkv 2 x 8192 blocks at d = 128 makes groups of one,
        (128, 4, 2, 8192, (300, 1000, 17, 1000, 513), None),
        # 1 x 1536 blocks at d = 128 groups of two (the last one partial), with equal lengths
        (128, 4, 1, 1536, (700, 129, 700, 256, 1), (700, 129, 45, 256, 1)),
        # 2 x 1024 blocks at d = 64 groups of four (the last one partial)
        (64, 4, 2, 1024, (300, 65, 777, 300, 20, 512, 513), (300, 65, 1, 129, 20, 512, 257)),
    ],
)
def test_paged_prefill_causal_request_groups(d, Hq, Hkv, width, ctx, ql):
    """Wide block tables make the causal prefill run its requests in several groups (sorted
    by length inside the kernel): the result matches the oracle and equals, bit for bit,
    the run over the same table cut to the blocks in use (one group), since every item
    computes the same tiles in the same order whatever item order the CTAs follow."""
    pc = PagedPrefillCase("groups", len(ctx), Hq, Hkv, d, 16, 1, 8192, width, True, 80 + Hq + d,
                          ctx_lens_override=ctx, q_lens_override=ql)
    inp = pc.make(poison=True)
    fa.device_status(reset=True)
    o, lse = run(inp, True)
    assert fa.device_status() == 0
    O, L = oracle(inp, True)
    check_rows(o, lse, O, L, inp["q_lens"], f"width={width}")
    narrow = dict(inp, block_table=inp["block_table"][:, :(max(ctx) + 15) // 16].contiguous())
    o1, lse1 = run(narrow, True)
    assert fa.device_status() == 0
    for r, n in enumerate(inp["q_lens"].tolist()):
        assert torch.equal(o[r, :, :n], o1[r, :, :n]), f"request {r}"
        assert torch.equal(lse[r, :, :n], lse1[r, :, :n]), f"request {r}"


def test_paged_prefill_matches_dense_kernel_bitwise():
    """Whole causal prompts over the paged cache give exactly the dense forward's bits on
    the same (de-paged) keys and values: the tiles and their order are the same."""
    pc = PagedPrefillCase("dense_eq", 3, 8, 2, 128, 16, 1, 8192, 64, True, 71, ctx_lens_override=(1000, 129, 700))
    inp = pc.make()
    o, lse = run(inp, True)
    for r, n in enumerate(inp["ctx_lens"].tolist()):
        k = torch.stack([torch.from_numpy(ora.depage(inp["k_cache"], inp["block_table"][r], n, g, 16))
                         for g in range(2)])[None].to(torch.bfloat16)
        v = torch.stack([torch.from_numpy(ora.depage(inp["v_cache"], inp["block_table"][r], n, g, 16))
                         for g in range(2)])[None].to(torch.bfloat16)
        od, ld = fa.fwd(inp["q"][r:r + 1, :, :n].contiguous().cuda(), k.cuda(), v.cuda(), causal=True)
        assert torch.equal(o[r, :, :n], od[0].cpu()), f"request {r}"
        assert torch.equal(lse[r, :, :n], ld[0].cpu()), f"request {r}"


def test_paged_prefill_full_config_sampled():
    """8 prompts of U{2048..8192} tokens, Hq=32, Hkv=8, d=128, causal, permuted pool:
    sampled rows (first, last, ragged tile ends, random) of sampled heads vs the oracle."""
    inp = PAGED_PREFILL.make(poison=True)
    fa.device_status(reset=True)
    o, lse = run(inp, True)
    assert fa.device_status() == 0
    rng = np.random.default_rng(7)
    G = PAGED_PREFILL.Hq // PAGED_PREFILL.Hkv
    for r in range(PAGED_PREFILL.R):
        n, nq = int(inp["ctx_lens"][r]), int(inp["q_lens"][r])
        for h in rng.choice(PAGED_PREFILL.Hq, 2, replace=False):
            kr = ora.depage(inp["k_cache"], inp["block_table"][r], n, h // G, 16)[None, None]
            vr = ora.depage(inp["v_cache"], inp["block_table"][r], n, h // G, 16)[None, None]
            rows = sorted({0, nq - 1, min(nq - 1, 255), min(nq - 1, 256), *rng.integers(0, nq, 4).tolist()})
            O, L = ora.attention_fwd_rows(inp["q"][r:r + 1, h:h + 1, :nq], kr, vr, PAGED_PREFILL.scale, True, 0, 0,
                                          rows)
            check_bf16(o[r, h, rows], O, f"O r={r} h={h}")
            check_lse(lse[r, h, rows], L, f"lse r={r} h={h}")
    # every defined row is finite, whatever the padding held
    for r, nq in enumerate(inp["q_lens"].tolist()):
        assert torch.isfinite(o[r, :, :nq].float()).all()


def test_paged_prefill_bad_lengths_and_blocks_are_flagged():
    """A q_len above ctx_len skips that request; a block id outside the pool is not
    dereferenced.  Both set the device status word; the other requests are unaffected."""
    pc = PagedPrefillCase("bad", 3, 4, 2, 128, 16, 1, 8192, 64, True, 72, ctx_lens_override=(100, 100, 300))
    inp = pc.make()
    inp["q_lens"][1] = 101  # more query rows than cached tokens
    fa.device_status(reset=True)
    o, lse = run(inp, True)
    assert fa.device_status(reset=True) == fa.FA_ERR_INVALID_ARG
    good = {k: (v[[0, 2]] if k in PER_REQUEST else v) for k, v in inp.items()}
    O, L = oracle(good, True)
    check_rows(o[[0, 2]], lse[[0, 2]], O, L, good["q_lens"], "valid requests")

    inp = pc.make()
    inp["block_table"][2, 3] = inp["num_blocks"] + 9
    fa.device_status(reset=True)
    o, lse = run(inp, True)
    assert fa.device_status(reset=True) == fa.FA_ERR_INVALID_ARG
    good = {k: (v[:2] if k in PER_REQUEST else v) for k, v in inp.items()}
    O, L = oracle(good, True)
    check_rows(o[:2], lse[:2], O, L, good["q_lens"], "valid requests")


def test_paged_prefill_rejects_bad_arguments():
    pc = PagedPrefillCase("args", 2, 4, 2, 128, 16, 1, 8192, 16, True, 73, ctx_lens_override=(40, 40))
    inp = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in pc.make().items()}
    with pytest.raises(fa.FAError):  # 3 query heads do not group over 2 KV heads
        fa.paged_prefill(inp["q"][:, :3].contiguous(), *(inp[n] for n in NAMES[1:]))
    kc8 = inp["k_cache"].view(inp["num_blocks"] * 2, 2, 8, 128)  # block_size 8
    with pytest.raises(fa.FAError):
        fa.paged_prefill(inp["q"], kc8, kc8, *(inp[n] for n in NAMES[3:]))
