"""fa_paged_decode_noalloc: the decode step for callers that cannot allocate device memory.

Such callers (plugins inside a framework that owns all device allocations, serving
loops that must not call cudaMalloc after start-up) get the split-KV scratch from a
fixed array inside the library instead of a workspace argument.  This file is
collected last so that a run stopping at the first failure has run everything else.
"""
import ctypes

import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import PAGED_DECODE, PagedCase
from oracle import attention_fp64 as ora
from parity import check_bf16, check_lse, to_np

pytestmark = pytest.mark.gpu

NAMES = ("q", "k_cache", "v_cache", "block_table", "ctx_lens")


def _noalloc(inp):
    L = fa.lib()
    t = {n: inp[n].cuda() for n in NAMES}
    R, Hq, d = t["q"].shape
    nb, Hkv, bs, _ = t["k_cache"].shape
    o = torch.empty_like(t["q"])
    lse = torch.empty(R, Hq, device="cuda", dtype=torch.float32)
    st = L.fa_paged_decode_noalloc(*(ctypes.c_void_p(t[n].data_ptr()) for n in NAMES), ctypes.c_void_p(o.data_ptr()),
                                   ctypes.c_void_p(lse.data_ptr()), R, Hq, Hkv, d, bs, t["block_table"].shape[1],
                                   nb, ctypes.c_float(d ** -0.5), fa.FA_DTYPE_BF16,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == fa.FA_OK, st
    torch.cuda.synchronize()
    return o, lse


def _with_workspace(inp):
    o, lse = fa.paged_decode(*(inp[n].cuda() for n in NAMES))
    torch.cuda.synchronize()
    return o, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [
        PAGED_DECODE.make(poison_unused=True),  # 64 requests, ctx up to 8192: needs most of the scratch
        PagedCase("second", 5, 12, 2, 128, 16, 1, 4096, 256, 61, ctx_lens_override=(1, 17, 513, 4000, 2048)).make(),
    ]
    fa.device_status(reset=True)
    for inp in cases:
        ref_o, ref_lse = _with_workspace(inp)
        o, lse = _noalloc(inp)
        check_bf16(o, to_np(ref_o), "noalloc O")
        check_lse(lse, ref_lse.cpu().numpy(), "noalloc lse")
        # and against the fp64 oracle on the same inputs
        d = inp["q"].shape[-1]
        O, L = ora.paged_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["block_table"], inp["ctx_lens"], 16,
                                d ** -0.5)
        check_bf16(o, O, "noalloc O vs oracle")
        check_lse(lse, L, "noalloc lse vs oracle")
    assert fa.device_status(reset=True) == fa.FA_OK


def test_noalloc_rejects_requests_beyond_its_scratch():
    L = fa.lib()
    fake = ctypes.c_void_p(1 << 20)  # rejected on the host before any use
    need = L.fa_paged_decode_workspace_size(64, 12, 128, 8192, 16)
    assert need > 8 * 1024 * 1024
    st = L.fa_paged_decode_noalloc(fake, fake, fake, fake, fake, fake, None, 64, 12, 2, 128, 16, 8192, 40000,
                                   ctypes.c_float(0.088), fa.FA_DTYPE_BF16, None)
    assert st == fa.FA_ERR_WORKSPACE
