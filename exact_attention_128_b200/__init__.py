"""Exact attention for B200 (sm_100a): Python binding of the C ABI in ``include/fa.h``.

Every step of the computation runs in the CUDA kernels of ``libfa_b200.so``; this
module only checks tensors, allocates outputs with torch, and passes raw pointers and
the current CUDA stream.  There is no fallback: if the library is missing or a
call is rejected, an exception is raised.

    o, lse = fwd(q, k, v, causal=False)             # q [B,Hq,N,d], k/v [B,Hkv,N,d]
    dq, dk, dv = bwd(q, k, v, o, lse, do, causal=False)
    paged_kv_append(k_new, v_new, k_cache, v_cache, block_table, positions)
    o, lse = paged_decode(q, k_cache, v_cache, block_table, ctx_lens)
    o, lse = paged_prefill(q, k_cache, v_cache, block_table, ctx_lens, q_lens, causal=True)

bf16 inputs run on the tensor cores (d in {64, 96, 128, 256} forward, {64, 96, 128}
backward); fp32 inputs (d = 64) on the CUDA cores.  Paged caches are
[num_blocks, Hkv, 16, d].
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = [
    "FAError",
    "lib",
    "fwd",
    "bwd",
    "bwd_workspace_size",
    "paged_decode",
    "paged_decode_workspace_size",
    "paged_kv_append",
    "paged_prefill",
    "device_status",
    "set_decode_split",
    "set_wait_limit_ns",
    "selftest_wait_timeout",
    "EXPORTED",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_b200.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_WORKSPACE, FA_ERR_DEVICE_TIMEOUT = range(6)
FA_DTYPE_F32, FA_DTYPE_BF16 = 0, 1
_DT = {torch.float32: FA_DTYPE_F32, torch.bfloat16: FA_DTYPE_BF16}

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

# name -> (restype, argtypes); the same names as the C entry points
EXPORTED = {
    "fa_status_string": (ctypes.c_char_p, [_i]),
    "fa_version": (_i, []),
    "fa_fwd": (_i, [_vp] * 5 + [_i] * 6 + [_f, _i, _i, _vp]),
    "fa_bwd_workspace_size": (_sz, [_i] * 4),
    "fa_bwd": (_i, [_vp] * 9 + [_i] + [_i] * 6 + [_f, _i, _i, _vp, _sz, _vp]),
    "fa_paged_decode_workspace_size": (_sz, [_i] * 5),
    "fa_paged_decode": (_i, [_vp] * 7 + [_i] * 7 + [_f, _i, _vp, _sz, _vp]),
    "fa_paged_decode_noalloc": (_i, [_vp] * 7 + [_i] * 7 + [_f, _i, _vp]),
    "fa_paged_kv_append": (_i, [_vp] * 6 + [_i] * 6 + [_i, _vp]),
    "fa_paged_prefill": (_i, [_vp] * 6 + [_vp, _vp] + [_i] * 8 + [_f, _i, _i, _vp]),
    "fa_device_status": (_i, [_i]),
    "fa_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "fa_selftest_wait_timeout": (_i, [_vp]),
    "fa_set_decode_split": (_i, [_i]),
}


class FAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {_status_string(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libfa_b200.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m exact_attention_128_b200.build` "
                "(there is no non-CUDA implementation of this library)"
            )
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTED.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _status_string(s: int) -> str:
    return lib().fa_status_string(int(s)).decode()


def _check(fn: str, status: int):
    if status != FA_OK:
        raise FAError(fn, status)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _cuda4(name, t, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None):
    """Forward pass: returns (o [B,Hq,Nq,d] of q's dtype, lse [B,Hq,Nq] fp32)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda4(n, t, q.dtype)
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("expected q [B,Hq,Nq,d] and k, v [B,Hkv,Nkv,d]")
    B, Hq, Nq, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    if k.shape[0] != B or k.shape[3] != d:
        raise ValueError("q and k disagree on batch or head dim")
    if q.dtype not in _DT:
        raise ValueError(f"unsupported dtype {q.dtype}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = out if out is not None else torch.empty_like(q)
    lse = lse if lse is not None else torch.empty((B, Hq, Nq), device=q.device, dtype=torch.float32)
    st = lib().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nkv, d,
                      float(scale), int(bool(causal)), _DT[q.dtype], _stream())
    _check("fa_fwd", st)
    return o, lse


def bwd_workspace_size(B, Hq, Nq, d) -> int:
    return int(lib().fa_bwd_workspace_size(B, Hq, Nq, d))


def bwd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
        grad_dtype: torch.dtype = torch.float32, workspace=None):
    """Backward pass of fwd: returns (dq, dk, dv) of dtype grad_dtype."""
    for n, t in (("q", q), ("k", k), ("v", v), ("o", o), ("do", do)):
        _cuda4(n, t, q.dtype)
    _cuda4("lse", lse, torch.float32)
    B, Hq, Nq, d = q.shape
    Hkv, Nkv = k.shape[1], k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if grad_dtype not in _DT:
        raise ValueError(f"unsupported grad dtype {grad_dtype}")
    dq = torch.empty(q.shape, device=q.device, dtype=grad_dtype)
    dk = torch.empty(k.shape, device=q.device, dtype=grad_dtype)
    dv = torch.empty(v.shape, device=q.device, dtype=grad_dtype)
    need = bwd_workspace_size(B, Hq, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    st = lib().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                      _DT[grad_dtype], B, Hq, Hkv, Nq, Nkv, d, float(scale), int(bool(causal)), _DT[q.dtype],
                      _ptr(workspace), workspace.numel() * workspace.element_size(), _stream())
    _check("fa_bwd", st)
    return dq, dk, dv


def paged_decode_workspace_size(R, Hq, d, max_blocks_per_seq, block_size) -> int:
    return int(lib().fa_paged_decode_workspace_size(R, Hq, d, max_blocks_per_seq, block_size))


def paged_decode(q, k_cache, v_cache, block_table, ctx_lens, scale: float | None = None,
                 with_lse: bool = True, workspace=None, out=None):
    """One decode step: q [R,Hq,d], caches [num_blocks,Hkv,block_size,d] -> (o [R,Hq,d], lse [R,Hq])."""
    _cuda4("q", q, torch.bfloat16)
    _cuda4("k_cache", k_cache, torch.bfloat16)
    _cuda4("v_cache", v_cache, torch.bfloat16)
    _cuda4("block_table", block_table, torch.int32)
    _cuda4("ctx_lens", ctx_lens, torch.int32)
    if v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must have the same shape")
    R, Hq, d = q.shape
    num_blocks, Hkv, bs, _ = k_cache.shape
    maxb = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty((R, Hq), device=q.device, dtype=torch.float32) if with_lse else None
    need = paged_decode_workspace_size(R, Hq, d, maxb, bs)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    st = lib().fa_paged_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(ctx_lens),
                               _ptr(o), _ptr(lse), R, Hq, Hkv, d, bs, maxb, num_blocks, float(scale),
                               FA_DTYPE_BF16, _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream())
    _check("fa_paged_decode", st)
    return o, lse


def paged_kv_append(k_new, v_new, k_cache, v_cache, block_table, positions):
    """Write one new token per request into the paged caches in place (slot positions[r])."""
    _cuda4("k_new", k_new, torch.bfloat16)
    _cuda4("v_new", v_new, torch.bfloat16)
    _cuda4("k_cache", k_cache, torch.bfloat16)
    _cuda4("v_cache", v_cache, torch.bfloat16)
    _cuda4("block_table", block_table, torch.int32)
    _cuda4("positions", positions, torch.int32)
    if k_new.shape != v_new.shape or k_cache.shape != v_cache.shape:
        raise ValueError("k/v shapes disagree")
    R, Hkv, d = k_new.shape
    num_blocks, _, bs, _ = k_cache.shape
    st = lib().fa_paged_kv_append(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                  _ptr(positions), R, Hkv, d, bs, block_table.shape[1], num_blocks, FA_DTYPE_BF16,
                                  _stream())
    _check("fa_paged_kv_append", st)


def paged_prefill(q, k_cache, v_cache, block_table, ctx_lens, q_lens, causal: bool = True,
                  scale: float | None = None, out=None, lse=None):
    """Prefill over a paged KV cache: q [R,Hq,Nq_max,d] (request r's rows < q_lens[r] are its
    last q_lens[r] positions), caches [num_blocks,Hkv,block_size,d] -> (o, lse [R,Hq,Nq_max]).
    Rows >= q_lens[r] of o and lse are undefined."""
    _cuda4("q", q, torch.bfloat16)
    _cuda4("k_cache", k_cache, torch.bfloat16)
    _cuda4("v_cache", v_cache, torch.bfloat16)
    _cuda4("block_table", block_table, torch.int32)
    _cuda4("ctx_lens", ctx_lens, torch.int32)
    _cuda4("q_lens", q_lens, torch.int32)
    if q.dim() != 4 or k_cache.dim() != 4 or v_cache.shape != k_cache.shape:
        raise ValueError("expected q [R,Hq,Nq_max,d] and caches [num_blocks,Hkv,block_size,d]")
    R, Hq, Nq, d = q.shape
    num_blocks, Hkv, bs, _ = k_cache.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = out if out is not None else torch.empty_like(q)
    if lse is None:
        lse = torch.empty((R, Hq, Nq), device=q.device, dtype=torch.float32)
    st = lib().fa_paged_prefill(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(ctx_lens),
                                _ptr(q_lens), _ptr(o), _ptr(lse), R, Hq, Hkv, Nq, d, bs, block_table.shape[1],
                                num_blocks, float(scale), int(bool(causal)), FA_DTYPE_BF16, _stream())
    _check("fa_paged_prefill", st)
    return o, lse


def device_status(reset: bool = True) -> int:
    return int(lib().fa_device_status(int(bool(reset))))


def set_decode_split(blocks: int) -> int:
    """Cache blocks per decode split (multiple of 4 in [32, 128]; 0 = default); returns the old value."""
    old = int(lib().fa_set_decode_split(int(blocks)))
    if old < 0:
        raise ValueError(f"decode split of {blocks} blocks is out of range")
    return old


def set_wait_limit_ns(ns: int):
    lib().fa_set_wait_limit_ns(int(ns))


def selftest_wait_timeout():
    _check("fa_selftest_wait_timeout", lib().fa_selftest_wait_timeout(_stream()))
