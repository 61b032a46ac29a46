"""CUDA-graph capture of a decode step ("Fusión y CUDA Graphs con torch.compile": a graph
records a sequence of GPU work and replays it with one submission; it needs stable
addresses and shapes).  The append + decode C-ABI calls are captured once and replayed on
new inputs written in place; each replay must equal the eager calls."""
import pytest
import torch

import exact_attention_128_b200 as fa
from exact_attention_128_b200.workloads import PagedCase, randn

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
    ws = torch.empty(fa.paged_decode_workspace_size(pc.R, pc.Hq, pc.d, pc.max_blocks_per_seq, pc.block_size),
                     device=dev, dtype=torch.uint8)

    def step():
        fa.paged_kv_append(k_new, v_new, kc, vc, table, pos)
        fa.paged_decode(q, kc, vc, table, ctx, with_lse=False, workspace=ws, out=o)

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
        kc_ref, vc_ref = kc.clone(), vc.clone()
        g.replay()
        torch.cuda.synchronize()
        got = o.clone()
        kc.copy_(kc_ref)
        vc.copy_(vc_ref)
        step()
        torch.cuda.synchronize()
        assert torch.equal(got, o), f"replay {t} differs from the eager calls"
    assert fa.device_status() == 0
