"""CUDA-graph capture of a decode step ("Fusión y CUDA Graphs con torch.compile": a graph
records a sequence of GPU work and replays it with one submission; it needs stable
addresses and shapes, and its results are checked with tolerances that suit the dtype).
The append + decode C-ABI calls are captured once and replayed on new inputs written in
place; each replay's cache must equal the oracle's append bit for bit, its output and lse
must match the oracle's decode on that cache, and it must equal the eager calls."""
import numpy as np
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import PagedCase, randn
from oracle import attention_fp64 as ora
from parity import check_bf16, check_lse

pytestmark = pytest.mark.gpu


def test_append_and_decode_replay_in_a_cuda_graph():
    pc = PagedCase("graph", 8, 12, 2, 128, 16, 1, 2000, 128, 70, ctx_lens_override=(1, 15, 16, 17, 300, 999, 1500, 2000))
    inp = pc.make()
    dev = torch.device("cuda")
    kc, vc = inp["k_cache"].to(dev), inp["v_cache"].to(dev)
    table = inp["block_table"].to(dev)
    # static buffers the graph reads and writes
    q = torch.empty(pc.R, pc.Hq, pc.d, device=dev, dtype=torch.bfloat16)
    k_new = torch.empty(pc.R, pc.Hkv, pc.d, device=dev, dtype=torch.bfloat16)
    v_new = torch.empty_like(k_new)
    pos = torch.empty(pc.R, device=dev, dtype=torch.int32)
    ctx = torch.empty(pc.R, device=dev, dtype=torch.int32)
    o = torch.empty_like(q)
    lse = torch.empty(pc.R, pc.Hq, device=dev, dtype=torch.float32)
    ws = torch.empty(fa.paged_decode_workspace_size(pc.R, pc.Hq, pc.d, pc.max_blocks_per_seq, pc.block_size),
                     device=dev, dtype=torch.uint8)
    L = fa.lib()

    def step():
        fa.paged_kv_append(k_new, v_new, kc, vc, table, pos)
        # the C entry point directly, so the graph also writes lse into a fixed buffer
        st = L.fa_paged_decode(*(fa._ptr(t) for t in (q, kc, vc, table, ctx, o, lse)), pc.R, pc.Hq, pc.Hkv,
                               pc.d, pc.block_size, pc.max_blocks_per_seq, inp["num_blocks"],
                               float(pc.scale), fa.FA_DTYPE_BF16, fa._ptr(ws), ws.numel(), fa._stream())
        assert st == fa.FA_OK

    def load(t):
        base = inp["ctx_lens"].to(torch.int32)
        q.copy_(randn((pc.R, pc.Hq, pc.d), 700 + t, torch.bfloat16))
        k_new.copy_(randn((pc.R, pc.Hkv, pc.d), 710 + t, torch.bfloat16))
        v_new.copy_(randn((pc.R, pc.Hkv, pc.d), 720 + t, torch.bfloat16))
        # overwrite each request's last cached slot (a slot its table maps)
        pos.copy_(base - 1)
        ctx.copy_(base)

    load(0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm-up outside the capture (first-call set-up)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in (1, 2, 3):
        load(t)
        kc_before, vc_before = kc.clone(), vc.clone()
        g.replay()
        torch.cuda.synchronize()
        got_o, got_lse = o.clone(), lse.clone()
        # oracle: the append on the cache as it was before the replay, then the decode step
        ek, ev = ora.paged_append(ora.to_f64(kc_before), ora.to_f64(vc_before), table.cpu().numpy(),
                                  pos.cpu().numpy(), ora.to_f64(k_new), ora.to_f64(v_new), pc.block_size)
        assert np.array_equal(ora.to_f64(kc), ek) and np.array_equal(ora.to_f64(vc), ev), f"replay {t}: cache"
        O, LSE = ora.paged_decode(ora.to_f64(q), ek, ev, table.cpu().numpy(), ctx.cpu().numpy(), pc.block_size,
                                  pc.scale)
        check_bf16(got_o, O, f"replay {t} O")
        check_lse(got_lse, LSE, f"replay {t} lse")
        # and the eager calls on the same inputs give the same bits
        kc.copy_(kc_before)
        vc.copy_(vc_before)
        step()
        torch.cuda.synchronize()
        assert torch.equal(got_o, o) and torch.equal(got_lse, lse), f"replay {t} differs from the eager calls"
    assert fa.device_status() == 0
