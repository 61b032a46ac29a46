#!/usr/bin/env python
"""Throughput of the exact-attention kernels on B200, one JSON line per run.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-secondary] [--no-cpu-baseline]

A step is one call of the library over one batch of the workload with inputs
resident in device memory; K steps run back to back on rotating input sets whose
total size exceeds twice the L2 cache, bracketed by a barrier and a device
synchronisation, timed with CUDA events on the launching stream.  Under torchrun
each rank runs its own replica (weak scaling) and the slowest rank's time counts.

The headline workload is the largest single-GPU forward: the non-causal GQA prefill at
N=16384 (B=2, Hq=32, Hkv=8, d=128, bf16; 8.8 TFLOP per call), the end point of the
sweep over N at B*N = 32768.  With secondary measurements on (the default at one GPU)
the line ends with a compact record of every other workload: the other sweep points,
the long causal GQA prefill, the causal training step (forward + backward), the paged
decode step, the batched ViT-B/16 layer, the paged prefill, head dimensions 96 and 256,
the fp32 ViT layer (forward; forward + backward), the KV-cache append and the CUDA-graph
decode step.  Their full records go to stderr.

`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload (the only other implementation of this method here).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s & % of B200 BF16 tensor peak; paged-decode HBM GB/s"
L2_BYTES = 126 * 2**20
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
EX2_PER_CLK_SM = 16  # SFU ex2.approx.f32 throughput per SM per clock (microbenchmark on B200)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return FALLBACK, "fallback"


def kernel_sources_sha(files) -> str:
    """Hash of the code (comments and layout stripped) of the kernel source files a
    profile was taken on (csrc-relative names): any change to the code voids the stored
    traffic figure, a comment edit does not."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_128_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(f.encode() + " ".join(text.split()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str):
    """Per-launch DRAM bytes (read + write) from a committed ncu summary.

    None unless the summary was taken on the current sources of that kernel.
    """
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(kernel)
    if not e or e.get("src_sha") != kernel_sources_sha(e.get("files", [])):
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"fa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return parse_clock_lines(lines)


def parse_clock_lines(lines):
    """Summarise `nvidia-smi --query-gpu=<ClockSampler.FIELDS> --format=csv,noheader,nounits`
    samples: median SM clock, maximum SM clock, and every throttle reason seen Active."""
    sm, mx, reasons = [], [], set()
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx.append(float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers
def dist_setup():
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step_per_rank: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job rate: every rank processes its own replica; the slowest rank's time counts."""
    return world * units_per_step_per_rank * steps / (max_ms * 1e-3)


def n_rotations(bytes_per_set: int) -> int:
    return max(2, math.ceil(2 * L2_BYTES / max(bytes_per_set, 1)) + 1)


def timed_loop(fns, steps, warmup, world):
    """Run fns[i % len(fns)]() for warmup then `steps` iterations; device-timed ms."""
    import torch

    for i in range(warmup):
        fns[i % len(fns)]()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(steps):
        fns[i % len(fns)]()
    e1.record(st)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), world)


# ----------------------------------------------------------------------------- workloads
def dense_fwd_step_fns(case, dev, rot=None):
    """Device-resident rotating input sets and one C-ABI fa_fwd call per step."""
    import ctypes

    import torch

    import exact_attention_128_b200 as fa

    q, k, v = case.make()
    set_bytes = 2 * q.numel() * q.element_size() + k.numel() * k.element_size() * 2
    rot = rot or n_rotations(set_bytes)
    L = fa.lib()
    sets, fns = [], []
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    for i in range(rot):
        qq, kk, vv = (qd, kd, vd) if i == 0 else (qd.clone(), kd.clone(), vd.clone())
        o = torch.empty_like(qq)
        lse = torch.empty(case.B, case.Hq, case.Nq, device=dev, dtype=torch.float32)
        sets.append((qq, kk, vv, o, lse))
        args = [ctypes.c_void_p(t.data_ptr()) for t in (qq, kk, vv, o, lse)] + [
            case.B, case.Hq, case.Hkv, case.Nq, case.Nkv, case.d, ctypes.c_float(case.scale), int(case.causal),
            fa.FA_DTYPE_F32 if case.dtype == "f32" else fa.FA_DTYPE_BF16,
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)]

        def fn(args=args):
            s = L.fa_fwd(*args)
            if s != 0:
                raise fa.FAError("fa_fwd", s)

        fns.append(fn)
    return fns, sets, (q, k, v), rot * set_bytes


def e2e_fwd(case, dev, steps, warmup, world, pipelined=True):
    """Same metric through the public API with pinned host buffers: every step copies its
    q, k, v host -> device, runs the forward, and reads o and lse back device -> host.

    pipelined: the copies in, the forward and the read-back run on three streams with two
    device buffer sets, so step i+1's inputs cross PCIe while step i computes and returns
    its result (each step still moves all of its bytes).  Otherwise every step is serial
    on one stream.
    """
    import torch

    import exact_attention_128_b200 as fa

    q, k, v = (t.pin_memory() for t in case.make())
    nb = 2 if pipelined else 1
    dev_in = [tuple(torch.empty_like(t, device=dev) for t in (q, k, v)) for _ in range(nb)]
    dev_out = [(torch.empty_like(dev_in[0][0]),
                torch.empty(case.B, case.Hq, case.Nq, device=dev, dtype=torch.float32)) for _ in range(nb)]
    host_out = [(torch.empty_like(q).pin_memory(), torch.empty(case.B, case.Hq, case.Nq, dtype=torch.float32).pin_memory())
                for _ in range(nb)]
    main = torch.cuda.current_stream()
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3)) if pipelined else (main, main, main)
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_comp = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]
    used = [False] * nb
    i_step = [0]

    def step():
        b = i_step[0] % nb
        i_step[0] += 1
        qd, kd, vd = dev_in[b]
        od, ld = dev_out[b]
        oh, lh = host_out[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_comp[b])  # the forward that read these inputs is done
            qd.copy_(q, non_blocking=True)
            kd.copy_(k, non_blocking=True)
            vd.copy_(v, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if used[b]:
                s_comp.wait_event(ev_out[b])  # the previous read-back of these outputs is done
            fa.fwd(qd, kd, vd, causal=case.causal, scale=case.scale, out=od, lse=ld)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            oh.copy_(od, non_blocking=True)
            lh.copy_(ld, non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    def join():  # the timed region ends when every stream's work has finished
        if pipelined:
            for st in (s_in, s_comp, s_out):
                main.wait_stream(st)

    for _ in range(warmup):
        step()
    join()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    if pipelined:
        for st in (s_in, s_comp, s_out):
            st.wait_stream(main)
    for _ in range(steps):
        step()
    join()
    e1.record(main)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = host_out[0][0].numel() * host_out[0][0].element_size() + host_out[0][1].numel() * 4
    return ms, h2d, d2h


def measure_dense_fwd(case, dev, steps, warmup, world, peaks, peak_key="bf16_tflops"):
    """Forward kernel throughput; the roofline is whichever of tensor or HBM binds.

    Algorithmic work per launch: 4*d FLOP per allowed (query, key) pair and head; bytes
    = q, k, v read once + o written once + lse (fp32).  The bound is the larger of
    flops / tensor peak and bytes / HBM peak (fp32 inputs: the CUDA cores' FFMA peak).
    """
    fns, sets, host, rot_bytes = dense_fwd_step_fns(case, dev)
    ms = timed_loop(fns, steps, warmup, world)
    flops = case.fwd_flops()
    q, k, v = host
    esz = q.element_size()
    nbytes = 2 * q.numel() * esz + 2 * k.numel() * esz + case.B * case.Hq * case.Nq * 4
    per_step_ms = ms / steps
    sec = per_step_ms * 1e-3
    tflops = flops / sec / 1e12
    gbs = nbytes / sec / 1e9
    if case.dtype == "f32":
        # up to 256 keys the library runs its one-pass fp32 kernel, above that the tiled one
        kname = "fa_fwd_f32_small_kernel" if case.Nkv <= 256 else "fa_fwd_f32_kernel"
        peak = fp32_alu_peak_tflops(peaks)
        roof = {"bound": "alu", "achieved": round(tflops, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(tflops / peak, 4), "peak_kind": "fp32 FFMA, 148 SMs x 128 lanes x 2 x max clock",
                "traffic": None, "kernel": kname, "algorithmic_flops_per_launch": flops,
                "algorithmic_bytes_per_launch": nbytes, "gbs": round(gbs, 1)}
        return {"ms": ms, "per_step_ms": per_step_ms, "tflops": tflops, "roofline": roof, "rot_bytes": rot_bytes,
                "launches_per_step": 1}
    if case.d == 256:
        kname = f"fa_fwd_d256_kernel<{str(case.causal).lower()}>"
    elif case.d == 96:  # the d = 128 kernel on 96-wide rows
        kname = f"fa_fwd_bf16_kernel<128,{str(case.causal).lower()}>(d=96)"
    else:
        kname = f"fa_fwd_bf16_kernel<{case.d},{str(case.causal).lower()}>"
    t_tensor = flops / (peaks[peak_key] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    if t_hbm > t_tensor:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "peak_kind": "hbm_gbs",
                "frac_of_nominal_8000": round(gbs / NOMINAL_HBM_GBS, 4)}
    else:
        roof = {"bound": "tensor", "achieved": round(tflops, 2), "peak": peaks[peak_key], "unit": "TFLOP/s",
                "frac": round(tflops / peaks[peak_key], 4), "peak_kind": peak_key,
                "frac_of_nominal_2250": round(tflops / NOMINAL_BF16_TFLOPS, 4)}
    roof.update({"traffic": traffic_for(kname), "kernel": kname, "algorithmic_flops_per_launch": flops,
                 "algorithmic_bytes_per_launch": nbytes, "tflops": round(tflops, 2), "gbs": round(gbs, 1),
                 "tensor_frac": round(tflops / peaks[peak_key], 4),
                 "hbm_frac": round(gbs / peaks["hbm_gbs"], 4)})
    # secondary ceiling: one exponential per allowed (query, key) pair and head on the SFU,
    # at 16 ex2 per clock per SM (measured on this GPU) and the maximum SM clock
    exps = case.B * case.Hq * case.allowed_pairs()
    exp_s = exps / (EX2_PER_CLK_SM * 148 * peaks.get("sm_max_mhz", 1965.0) * 1e6)
    roof["exp_bound"] = {"tflops": round(flops / exp_s / 1e12, 1), "frac": round(exp_s / sec, 4),
                         "ex2_per_launch": exps}
    return {"ms": ms, "per_step_ms": per_step_ms, "tflops": tflops, "roofline": roof, "rot_bytes": rot_bytes,
            "launches_per_step": 1}


def fp32_alu_peak_tflops(peaks):
    """FP32 FFMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP x max SM clock."""
    return 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12


def measure_train(case, dev, steps, warmup, world, peaks):
    """Forward + backward (recompute) per step."""
    import torch

    import exact_attention_128_b200 as fa

    q, k, v, do = case.make(with_grad_output=True)
    set_bytes = sum(t.numel() * t.element_size() for t in (q, k, v, do)) * 2
    rot = n_rotations(set_bytes)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    sets = []
    ws = torch.empty(fa.bwd_workspace_size(case.B, case.Hq, case.Nq, case.d), device=dev, dtype=torch.uint8)
    for i in range(rot):
        s = (qd, kd, vd, dod) if i == 0 else tuple(t.clone() for t in (qd, kd, vd, dod))
        sets.append(s)

    def mk(s):
        def step():
            o, lse = fa.fwd(s[0], s[1], s[2], causal=case.causal, scale=case.scale)
            fa.bwd(s[0], s[1], s[2], o, lse, s[3], causal=case.causal, scale=case.scale, workspace=ws)
        return step

    fns = [mk(s) for s in sets]
    ms = timed_loop(fns, steps, warmup, world)
    fwd = case.fwd_flops()
    flops = fwd * 3.5  # forward 2 contractions + backward 5 (score recompute included)
    per = ms / steps
    tflops = flops / (per * 1e-3) / 1e12
    if case.dtype == "f32":  # CUDA-core FFMA kernels
        peak = fp32_alu_peak_tflops(peaks)
        return {"per_step_ms": per, "tflops": tflops,
                "roofline": {"bound": "alu", "achieved": round(tflops, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
                             "frac": round(tflops / peak, 4), "peak_kind": "fp32 FFMA, 148 SMs x 128 lanes x 2 x max clock",
                             "algorithmic_flops_per_step": flops}}
    peak = peaks["bf16_tflops"]
    # the backward dominates the step; its algorithmic bytes: q, k, v, o, dO (bf16) and lse
    # read, dq, dk, dv (fp32) written
    n_q, n_kv = case.B * case.Hq * case.Nq * case.d, case.B * case.Hkv * case.Nkv * case.d
    bwd_bytes = 2 * (2 * n_q + 2 * n_kv + n_q) + 4 * case.B * case.Hq * case.Nq + 4 * (n_q + 2 * n_kv)
    kname = f"fa_bwd_d256_kernel<{str(case.causal).lower()}>" if case.d == 256 else \
        f"fa_bwd_bf16_kernel<{64 if case.d == 64 else 128},{str(case.causal).lower()}>"
    return {"per_step_ms": per, "tflops": tflops,
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tflops / peak, 4), "frac_of_nominal_2250": round(tflops / NOMINAL_BF16_TFLOPS, 4),
                         "algorithmic_flops_per_step": flops, "kernel": kname, "traffic": traffic_for(kname),
                         "algorithmic_bytes_per_launch": bwd_bytes}}


def measure_decode(pc, dev, steps, warmup, world, peaks):
    import ctypes

    import torch

    import exact_attention_128_b200 as fa
    from exact_attention_128_b200.workloads import PagedCase

    inp = pc.make()
    kvb = PagedCase.kv_bytes(inp["ctx_lens"].tolist(), pc.Hkv, pc.d)
    set_bytes = inp["k_cache"].numel() * 4
    rot = n_rotations(set_bytes)
    L = fa.lib()
    base = {n: inp[n].to(dev) for n in ("q", "k_cache", "v_cache", "block_table", "ctx_lens")}
    need = fa.paged_decode_workspace_size(pc.R, pc.Hq, pc.d, pc.max_blocks_per_seq, pc.block_size)
    fns, keep = [], []
    for i in range(rot):
        s = base if i == 0 else {n: t.clone() for n, t in base.items()}
        o = torch.empty_like(s["q"])
        lse = torch.empty(pc.R, pc.Hq, device=dev, dtype=torch.float32)
        ws = torch.empty(need, device=dev, dtype=torch.uint8)
        keep.append((s, o, lse, ws))
        args = [ctypes.c_void_p(s[n].data_ptr()) for n in ("q", "k_cache", "v_cache", "block_table", "ctx_lens")]
        args += [ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), pc.R, pc.Hq, pc.Hkv, pc.d,
                 pc.block_size, pc.max_blocks_per_seq, inp["num_blocks"], ctypes.c_float(pc.scale),
                 fa.FA_DTYPE_BF16, ctypes.c_void_p(ws.data_ptr()), need,
                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)]

        def fn(args=args):
            st = L.fa_paged_decode(*args)
            if st != 0:
                raise fa.FAError("fa_paged_decode", st)

        fns.append(fn)
    ms = timed_loop(fns, steps, warmup, world)
    per = ms / steps
    gbs = kvb / (per * 1e-3) / 1e9
    peak = peaks["hbm_gbs"]
    return {"per_step_ms": per, "gbs": gbs, "kv_bytes": kvb,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "frac_of_nominal_8000": round(gbs / NOMINAL_HBM_GBS, 4),
                         "algorithmic_bytes_per_step": kvb, "algorithmic_bytes_per_launch": kvb,
                         "kernel": "fa_paged_decode_kernel", "traffic": traffic_for("fa_paged_decode_kernel"),
                         "kernels": ["fa_paged_decode_kernel", "fa_paged_decode_combine_kernel"]}}


def measure_paged_prefill(pc, dev, steps, warmup, world, peaks, peak_key="bf16_tflops"):
    """Prefill over the paged cache: 4*d FLOP per computed (query, key) pair and head;
    bytes = every cached K/V row once per KV head + q and o rows (bf16)."""
    import ctypes

    import torch

    import exact_attention_128_b200 as fa

    inp = pc.make()
    names = ("q", "k_cache", "v_cache", "block_table", "ctx_lens", "q_lens")
    set_bytes = (inp["k_cache"].numel() * 2 + inp["q"].numel() * 2) * 2
    rot = n_rotations(set_bytes)
    L = fa.lib()
    base = {n: inp[n].to(dev) for n in names}
    R, Hq, nq_max, d = inp["q"].shape
    fns, keep = [], []
    for i in range(rot):
        s = base if i == 0 else {n: t.clone() for n, t in base.items()}
        o = torch.empty_like(s["q"])
        lse = torch.empty(R, Hq, nq_max, device=dev, dtype=torch.float32)
        keep.append((s, o, lse))
        args = [ctypes.c_void_p(s[n].data_ptr()) for n in names]
        args += [ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), R, Hq, pc.Hkv, nq_max, d,
                 pc.block_size, pc.max_blocks_per_seq, inp["num_blocks"], ctypes.c_float(pc.scale), int(pc.causal),
                 fa.FA_DTYPE_BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)]

        def fn(args=args):
            st = L.fa_paged_prefill(*args)
            if st != 0:
                raise fa.FAError("fa_paged_prefill", st)

        fns.append(fn)
    ms = timed_loop(fns, steps, warmup, world)
    per = ms / steps
    flops = pc.fwd_flops()
    tflops = flops / (per * 1e-3) / 1e12
    peak = peaks[peak_key]
    kname = f"fa_fwd_bf16_kernel<{pc.d},{str(pc.causal).lower()},paged>"
    return {"per_step_ms": per, "tflops": tflops,
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tflops / peak, 4), "peak_kind": peak_key,
                         "frac_of_nominal_2250": round(tflops / NOMINAL_BF16_TFLOPS, 4),
                         "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": pc.io_bytes(),
                         "kernel": kname, "traffic": traffic_for(kname)}}


def measure_append(pc, dev, steps, warmup, world, peaks):
    """One new token per request written into the paged cache (KV-cache append)."""
    import ctypes

    import torch

    import exact_attention_128_b200 as fa

    inp = pc.make()
    L = fa.lib()
    kc, vc, table = inp["k_cache"].to(dev), inp["v_cache"].to(dev), inp["block_table"].to(dev)
    # append at each request's last cached position (a slot its table already maps)
    pos = (inp["ctx_lens"] - 1).to(torch.int32).to(dev)
    k_new = torch.randn(pc.R, pc.Hkv, pc.d, device=dev).to(torch.bfloat16)
    v_new = torch.randn(pc.R, pc.Hkv, pc.d, device=dev).to(torch.bfloat16)
    args = [ctypes.c_void_p(t.data_ptr()) for t in (k_new, v_new, kc, vc, table, pos)]
    args += [pc.R, pc.Hkv, pc.d, pc.block_size, pc.max_blocks_per_seq, inp["num_blocks"], fa.FA_DTYPE_BF16,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)]

    def fn():
        st = L.fa_paged_kv_append(*args)
        if st != 0:
            raise fa.FAError("fa_paged_kv_append", st)

    ms = timed_loop([fn], steps, warmup, world)
    per = ms / steps
    nbytes = 2 * 2 * pc.R * pc.Hkv * pc.d * 2  # read the new K, V rows and write them
    gbs = nbytes / (per * 1e-3) / 1e9
    return {"per_step_ms": per, "gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 5), "algorithmic_bytes_per_step": nbytes,
                         "note": "131 KB per call: launch-latency bound, not bandwidth bound"}}


def measure_graph_decode(dev, steps, warmup, world):
    """A small, launch-bound decode step (8 requests, append + decode) issued eagerly
    through the C ABI vs replayed from a CUDA graph; per-step device time of each."""
    import torch

    import exact_attention_128_b200 as fa
    from exact_attention_128_b200.workloads import PagedCase

    pc = PagedCase("graph_decode_r8", 8, 12, 2, 128, 16, 512, 1024, 64, 71)
    inp = pc.make()
    kc, vc, table = inp["k_cache"].to(dev), inp["v_cache"].to(dev), inp["block_table"].to(dev)
    q = inp["q"].to(dev)
    ctx = inp["ctx_lens"].to(dev)
    pos = (inp["ctx_lens"] - 1).to(dev)
    k_new = torch.randn(pc.R, pc.Hkv, pc.d, device=dev).to(torch.bfloat16)
    v_new = torch.randn_like(k_new)
    o = torch.empty_like(q)
    ws = torch.empty(fa.paged_decode_workspace_size(pc.R, pc.Hq, pc.d, pc.max_blocks_per_seq, pc.block_size),
                     device=dev, dtype=torch.uint8)

    def step():
        fa.paged_kv_append(k_new, v_new, kc, vc, table, pos)
        fa.paged_decode(q, kc, vc, table, ctx, with_lse=False, workspace=ws, out=o)

    eager = timed_loop([step], steps, warmup, world) / steps
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    graph = timed_loop([g.replay], steps, warmup, world) / steps
    del g
    return {"eager_ms_per_step": round(eager, 5), "graph_ms_per_step": round(graph, 5),
            "speedup": round(eager / graph, 3), "kernels_per_step": 3}


# ----------------------------------------------------------------------------- CPU oracle
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


class OracleRows:
    """The fp64 oracle over a dense workload in units of up to `rows` query rows of one
    (b, h) head (whole heads when N <= rows), each unit one call of its exact per-row
    forward function on that head's stored values (so no N x N fp64 matrix larger than
    rows x Nkv is ever held).  Counts the algorithmic FLOPs of the rows done."""

    def __init__(self, case, rows=2048):
        self.case = case
        self.q, self.k, self.v = case.make()
        self.rows = min(rows, case.Nq)
        self.per_head = (case.Nq + self.rows - 1) // self.rows
        self.units = case.B * case.Hq * self.per_head
        self.G = case.Hq // case.Hkv
        self.done = 0
        self.flops = 0.0
        self.rows_done = 0

    def step(self):
        from oracle import attention_fp64 as ora

        c = self.case
        u = self.done % self.units
        bh, part = divmod(u, self.per_head)
        b, h = divmod(bh, c.Hq)
        r0 = part * self.rows
        rows = list(range(r0, min(c.Nq, r0 + self.rows)))
        g = h // self.G
        ora.attention_fwd_rows(self.q[b:b + 1, h:h + 1], self.k[b:b + 1, g:g + 1], self.v[b:b + 1, g:g + 1],
                               c.scale, c.causal, 0, 0, rows)
        off = c.Nkv - c.Nq
        keys = sum(min(c.Nkv, i + off + 1) for i in rows) if c.causal else len(rows) * c.Nkv
        self.flops += 4.0 * c.d * keys
        self.rows_done += len(rows)
        self.done += 1

    def describe(self):
        return (f"{self.done} unit(s) of <= {self.rows} query rows of one (b,h) head of {self.case.name} "
                f"({self.rows_done} rows, {self.rows_done / (self.case.B * self.case.Hq * self.case.Nq):.4f} of "
                f"the workload), NumPy fp64 materialising each unit's score rows")


def cpu_oracle_dense(case, budget_s=12.0):
    """Time the fp64 oracle on units of the workload until ~budget_s of CPU work."""
    orc = OracleRows(case)
    t0 = time.perf_counter()
    while orc.done == 0 or time.perf_counter() - t0 < budget_s:
        orc.step()
    dt = time.perf_counter() - t0
    return {"value": orc.flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": orc.describe() + f", {dt:.1f} s"}


def cpu_oracle_extrapolated(case, train=False, budget_s=2.0):
    """The fp64 oracle on a bounded sample of a long workload, reported as a rate (which
    is what a linear extrapolation to the whole workload gives): forward row units, or
    one whole (b, h) head forward + backward for a training step."""
    from oracle import attention_fp64 as ora

    if not train:
        r = cpu_oracle_dense(case, budget_s)
        r["sample"] += ", extrapolated to the whole workload"
        return r
    t = case.make(with_grad_output=True)
    q, k, v, do = (ora.to_f64(x[0, 0]) for x in t)
    t0 = time.perf_counter()
    ora.attention_head(q, k, v, case.scale, case.causal)
    ora.attention_bwd_head(q, k, v, do, case.scale, case.causal)
    dt = time.perf_counter() - t0
    heads = case.B * case.Hq
    return {"value": case.fwd_flops() * 3.5 / (dt * heads) / 1e12, "unit": "TFLOP/s", "cores": oracle_threads(),
            "kind": "oracle", "sample": f"1 whole (b,h) head of {case.name} forward + backward in {dt:.2f} s, "
                                        f"extrapolated to {heads} heads"}


def reference_line(case, args):
    """The oracle as the reference arm: W + K steps, each step the same number of row units
    of the workload, sized from one probe unit so the whole run stays within
    ``args.reference_seconds`` (90 s by default)."""
    orc = OracleRows(case)
    t0 = time.perf_counter()
    orc.step()
    t_unit = max(time.perf_counter() - t0, 1e-4)
    per_step = max(1, min(orc.units, int(args.reference_seconds / ((args.steps + args.warmup) * t_unit))))

    def step():
        for _ in range(per_step):
            orc.step()

    for _ in range(args.warmup):
        step()
    f0, r0 = orc.flops, orc.rows_done
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = (orc.flops - f0) / dt / 1e12
    rows = orc.rows_done - r0
    cb = {"value": value, "unit": "TFLOP/s", "cores": oracle_threads(), "kind": "oracle",
          "sample": f"{per_step} unit(s) of <= {orc.rows} query rows of one (b,h) head of {case.name} per step "
                    f"({rows} rows over {args.steps} steps), {dt:.1f} s"}
    # under torchrun with N ranks the job is N-wide, but rank 0 alone times the oracle
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": case.name, "B": case.B, "Hq": case.Hq, "Hkv": case.Hkv, "N": case.Nq,
                       "d": case.d, "causal": case.causal, "sample_units_per_step": per_step,
                       "parallelism": "rank 0 on its host cores" + (f" (of {args.gpus} ranks)" if args.gpus > 1 else "")},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def compact(r, value_key, digits=2):
    """[value, unit, ms per step, roofline frac, DRAM traffic / algorithmic bytes or None]."""
    roof = r.get("roofline", {})
    tr = roof.get("traffic")
    alg = roof.get("algorithmic_bytes_per_launch")
    ratio = round(tr / alg, 2) if tr and alg else None
    unit = "GB/s" if value_key == "gbs" else "TFLOP/s"
    return [round(r[value_key], digits), unit, round(r["per_step_ms"], 4), roof.get("frac"), ratio]


# ----------------------------------------------------------------------------- main
HEADLINE = "gqa_prefill_noncausal_n16384"


def run_secondaries(W, case, dev, world, peaks, no_cpu):
    """Every other workload, each timed over >= 50 steps (300 for the microsecond ones).

    Returns (compact, detail): compact[name] = [value, unit, ms per step, roofline frac,
    DRAM traffic / algorithmic bytes]; detail[name] = the full measurement."""
    import torch

    import exact_attention_128_b200 as fa

    compact_out, detail = {}, {}

    def put(name, r, key, digits=2, oracle=None):
        compact_out[name] = compact(r, key, digits)
        r = {k: v for k, v in r.items() if k != "rot_bytes"}
        if oracle is not None:
            r["cpu_oracle_extrapolated"] = oracle
            compact_out[name].append(round(oracle["value"], 4))
        detail[name] = r
        torch.cuda.empty_cache()

    for c in (*W.prefill_sweep(), W.GQA_PREFILL_CAUSAL):
        if c.name == case.name:
            continue
        r = measure_dense_fwd(c, dev, 50, 5, world, peaks)
        put(c.name, r, "tflops", oracle=None if no_cpu else cpu_oracle_extrapolated(c))
    try:
        r = measure_train(W.TRAIN_CAUSAL, dev, 50, 5, world, peaks)
        put(W.TRAIN_CAUSAL.name, r, "tflops",
            oracle=None if no_cpu else cpu_oracle_extrapolated(W.TRAIN_CAUSAL, train=True))
    except fa.FAError as e:
        compact_out[W.TRAIN_CAUSAL.name] = detail[W.TRAIN_CAUSAL.name] = {"unavailable": str(e)}
    put(W.D256_TRAIN.name, measure_train(W.D256_TRAIN, dev, 50, 5, world, peaks), "tflops")
    r = measure_decode(W.PAGED_DECODE, dev, 300, 10, world, peaks)
    put(W.PAGED_DECODE.name, r, "gbs", 1)
    if case.name != W.VIT_BATCHED_BF16.name:
        put(W.VIT_BATCHED_BF16.name, measure_dense_fwd(W.VIT_BATCHED_BF16, dev, 300, 10, world, peaks), "tflops")
    put(W.PAGED_PREFILL.name, measure_paged_prefill(W.PAGED_PREFILL, dev, 50, 5, world, peaks), "tflops")
    for c in (W.D96_PREFILL, W.D256_PREFILL):
        put(c.name, measure_dense_fwd(c, dev, 50, 5, world, peaks), "tflops")
    put(W.VIT_LAYER_F32.name, measure_dense_fwd(W.VIT_LAYER_F32, dev, 300, 10, world, peaks), "tflops", 3)
    put("vit_b16_layer_f32_fwd_bwd", measure_train(W.VIT_LAYER_F32, dev, 300, 10, world, peaks), "tflops", 3)
    put("paged_kv_append_r64_hkv2_d128", measure_append(W.PAGED_DECODE, dev, 300, 10, world, peaks), "gbs", 2)
    g = measure_graph_decode(dev, 300, 10, world)
    compact_out["graph_decode_r8_append_plus_decode"] = [g["eager_ms_per_step"], g["graph_ms_per_step"]]
    detail["graph_decode_r8_append_plus_decode"] = g
    return compact_out, detail


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--reference-seconds", type=float, default=90.0,
                    help="--impl reference: host-time budget of the whole oracle run")
    ap.add_argument("--only", choices=["prefill_causal", "prefill_noncausal", "train", "decode", "append", "graph",
                                       "paged_prefill", "d96", "d256", "d256_train", "f32_train", "vit"],
                    help="measure just this one secondary workload (for profiling runs) and print it")
    ap.add_argument("--decode-split", type=int, default=0,
                    help="cache blocks per decode split (0: the library's default)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from exact_attention_128_b200 import workloads as W

    dense = {c.name: c for c in [W.VIT_BATCHED_BF16, W.GQA_PREFILL_CAUSAL, *W.prefill_sweep()]}
    if args.workload not in dense:
        ap.error(f"unknown workload {args.workload}; choose from {sorted(dense)}")
    case = dense[args.workload]
    peaks, peaks_kind = load_peaks()

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return  # rank 0 alone times the CPU oracle
        print(json.dumps(reference_line(case, args)))
        return

    import torch

    import exact_attention_128_b200 as fa

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    fa.lib()
    fa.device_status(reset=True)
    if args.decode_split:
        fa.set_decode_split(args.decode_split)

    if args.only:
        if args.only == "train":
            r = measure_train(W.TRAIN_CAUSAL, dev, args.steps, args.warmup, world, peaks)
        elif args.only == "d256_train":
            r = measure_train(W.D256_TRAIN, dev, args.steps, args.warmup, world, peaks)
        elif args.only == "decode":
            r = measure_decode(W.PAGED_DECODE, dev, args.steps, args.warmup, world, peaks)
        elif args.only == "append":
            r = measure_append(W.PAGED_DECODE, dev, args.steps, args.warmup, world, peaks)
        elif args.only == "graph":
            r = measure_graph_decode(dev, args.steps, args.warmup, world)
        elif args.only == "paged_prefill":
            r = measure_paged_prefill(W.PAGED_PREFILL, dev, args.steps, args.warmup, world, peaks)
        elif args.only in ("d96", "d256"):
            r = measure_dense_fwd(W.D96_PREFILL if args.only == "d96" else W.D256_PREFILL, dev, args.steps,
                                  args.warmup, world, peaks)
        elif args.only == "f32_train":
            r = measure_train(W.VIT_LAYER_F32, dev, args.steps, args.warmup, world, peaks)
        elif args.only == "vit":
            r = measure_dense_fwd(W.VIT_BATCHED_BF16, dev, args.steps, args.warmup, world, peaks)
        elif args.only == "prefill_causal":
            r = measure_dense_fwd(W.GQA_PREFILL_CAUSAL, dev, args.steps, args.warmup, world, peaks)
        else:
            r = measure_dense_fwd(case, dev, args.steps, args.warmup, world, peaks)
        r.pop("rot_bytes", None)
        if rank == 0:
            print(json.dumps({"only": args.only, "steps": args.steps, **r}))
        if fa.device_status(reset=True) != 0:
            raise SystemExit("device status set after the run")
        return

    sampler = ClockSampler(local)
    sampler.start()
    head = measure_dense_fwd(case, dev, args.steps, args.warmup, world, peaks)
    clocks = sampler.stop()

    e2e = None
    if not args.no_e2e:
        e_steps = max(3, min(args.steps, 50))
        ms, h2d, d2h = e2e_fwd(case, dev, e_steps, args.warmup, world, pipelined=True)
        ms_serial, _, _ = e2e_fwd(case, dev, e_steps, args.warmup, world, pipelined=False)
        e2e = {"value": round(world * case.fwd_flops() * e_steps / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "ms_per_step": round(ms / e_steps, 4),
               "schedule": "copy-in, forward and read-back of consecutive steps overlap on three streams",
               "serial_ms_per_step": round(ms_serial / e_steps, 4)}
    torch.cuda.empty_cache()

    secondary, sec_clocks = {}, None
    if not args.no_secondary and world == 1:
        sampler2 = ClockSampler(local)
        sampler2.start()
        secondary, detail = run_secondaries(W, case, dev, world, peaks, args.no_cpu_baseline)
        sec_clocks = sampler2.stop()
        # the full secondary records go to stderr; stdout keeps the one JSON line
        print("secondary detail: " + json.dumps(detail), file=sys.stderr)

    status = fa.device_status(reset=True)
    if status != 0:
        raise SystemExit(f"device status {status} after the run")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_dense(case, budget_s=12.0)

    value = job_throughput(case.fwd_flops(), args.steps, head["ms"], world) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(head["per_step_ms"], 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": case.name, "B": case.B, "Hq": case.Hq, "Hkv": case.Hkv, "N": case.Nq, "d": case.d,
                   "causal": case.causal, "parallelism": f"replicas{world}",
                   "l2": f"rotating input sets, {head['rot_bytes'] / 2**20:.0f} MiB > 2x L2"},
        "roofline": head["roofline"],
        "peaks": peaks_kind,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": clocks,
    }
    if secondary:
        # last, so that a reader keeping only the end of the line still sees every workload:
        # name: [value, unit, ms/step, roofline frac, DRAM traffic / algorithmic bytes (null:
        # no profile of the current code), fp64 oracle TFLOP/s where timed]
        line["secondary_clocks"] = {k: sec_clocks[k] for k in ("sm_mhz", "reasons")} if sec_clocks else None
        line["secondary"] = secondary
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
