"""Paged-decode parity: CUDA kernel vs the fp64 oracle (de-paged dense attention)."""
import numpy as np
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import PAGED_DECODE, PagedCase
from oracle import attention_fp64 as ora
from parity import check_bf16, check_lse

pytestmark = pytest.mark.gpu

NAMES = ("q", "k_cache", "v_cache", "block_table", "ctx_lens")


def run(inp):
    o, lse = fa.paged_decode(*(inp[n].cuda() for n in NAMES))
    torch.cuda.synchronize()
    return o, lse


def oracle(inp, bs=16):
    d = inp["q"].shape[-1]
    return ora.paged_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["block_table"], inp["ctx_lens"], bs,
                            1.0 / np.sqrt(d))


def test_paged_decode_full_config():
    """64 requests, Hq=12, Hkv=2, d=128, 16-token blocks, ctx ~ U[512, 8192], permuted pool."""
    inp = PAGED_DECODE.make(poison_unused=True)
    o, lse = run(inp)
    assert fa.device_status() == 0
    O, L = oracle(inp)
    check_bf16(o, O, "O")
    check_lse(lse, L, "lse")


@pytest.mark.parametrize(
    "Hq,Hkv,ctx",
    [
        (12, 2, (1, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1000, 4096)),
        (8, 8, (1, 2, 100, 700)),
        (16, 1, (5, 16, 600, 2000)),
        (4, 2, (8192, 1, 8191, 300)),
    ],
)
def test_paged_decode_edges(Hq, Hkv, ctx):
    pc = PagedCase("edge", len(ctx), Hq, Hkv, 128, 16, 1, 8192, 512, 40 + Hq, ctx_lens_override=ctx)
    inp = pc.make(poison_unused=True)
    o, lse = run(inp)
    assert fa.device_status() == 0
    O, L = oracle(inp)
    check_bf16(o, O, "O")
    check_lse(lse, L, "lse")


def test_shared_physical_blocks_read_only():
    """Two requests pointing at the same physical blocks (prefix sharing) read the same keys."""
    pc = PagedCase("share", 2, 12, 2, 128, 16, 1, 8192, 64, 50, ctx_lens_override=(700, 700))
    inp = pc.make()
    inp["block_table"][1] = inp["block_table"][0]
    inp["q"][1] = inp["q"][0]
    o, lse = run(inp)
    assert torch.equal(o[0], o[1]) and torch.equal(lse[0], lse[1])
    O, L = oracle(inp)
    check_bf16(o, O, "O")


def test_out_of_range_block_id_is_flagged_not_read():
    pc = PagedCase("bad", 2, 12, 2, 128, 16, 1, 8192, 64, 51, ctx_lens_override=(40, 40))
    inp = pc.make()
    inp["block_table"][1, 1] = inp["num_blocks"] + 5  # outside the pool
    fa.device_status(reset=True)
    o, lse = run(inp)
    assert fa.device_status(reset=True) == fa.FA_ERR_INVALID_ARG
    O, L = oracle({**inp, "block_table": inp["block_table"][:1], "ctx_lens": inp["ctx_lens"][:1],
                   "q": inp["q"][:1]})
    check_bf16(o[:1], O, "untouched request")


@pytest.mark.parametrize("split", [32, 64, 128])
def test_split_size_does_not_change_the_result(split):
    """The blocks of a request are cut into splits of `split` blocks and the splits' partial
    results merged by their lse weights ("No basta con promediar los resultados de los
    bloques"): a different cut of the same keys must give the same attention.  Config 5
    at each split size against the oracle, and against the default split within the bf16
    bar (128-block splits: 1-4 per request; 32-block splits: up to 16)."""
    inp = PAGED_DECODE.make(poison_unused=True)
    ref_o, ref_lse = run(inp)
    old = fa.set_decode_split(split)
    try:
        o, lse = run(inp)
    finally:
        fa.set_decode_split(old)
    assert fa.device_status() == 0
    O, L = oracle(inp)
    check_bf16(o, O, f"O split {split}")
    check_lse(lse, L, f"lse split {split}")
    check_bf16(o, ref_o.double().cpu().numpy(), f"O split {split} vs default split")
    check_lse(lse, ref_lse.double().cpu().numpy(), f"lse split {split} vs default split")
