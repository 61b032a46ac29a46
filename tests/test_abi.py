"""The C-ABI library: loads, exports every declared entry point, rejects bad input
on the host before touching the device.  Runs without a GPU."""
import ctypes
import os
import re

import pytest

import exact_attention_128_b200 as fa
from exact_attention_128_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    fabuild.build()
    return fa.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(fa.EXPORTED), "Python binding and header disagree"


def test_status_strings_and_version(L):
    assert L.fa_status_string(0) == b"ok"
    for s in range(1, 6):
        assert len(L.fa_status_string(s)) > 3
    assert L.fa_version() >= 10000


def test_workspace_sizes(L):
    n = L.fa_bwd_workspace_size(8, 16, 4096, 64)
    assert n >= 8 * 16 * 4096 * (64 + 1) * 4 and n % 256 == 0
    assert L.fa_bwd_workspace_size(0, 16, 4096, 64) == 0
    m = L.fa_paged_decode_workspace_size(64, 12, 128, 512, 16)
    assert m >= 64 * 12 * 129 * 4 and m % 256 == 0
    assert L.fa_paged_decode_workspace_size(64, 12, 128, 0, 16) == 0


def test_decode_split_setting_sizes_the_workspace(L):
    """Splits of 32 blocks need four times the partial results of 128-block splits; values
    outside [32, 128] or not a multiple of 4 are refused and change nothing."""
    old = L.fa_set_decode_split(128)
    try:
        big = L.fa_paged_decode_workspace_size(64, 12, 128, 512, 16)
        assert L.fa_set_decode_split(32) == 128
        small = L.fa_paged_decode_workspace_size(64, 12, 128, 512, 16)
        assert small >= 4 * (big - 512) and small == 64 * 12 * 16 * 128 * 4 + 64 * 12 * 16 * 4
        for bad in (31, 16, 130, 256, -4, 34):
            assert L.fa_set_decode_split(bad) == -1
        assert L.fa_set_decode_split(0) == 32
        assert L.fa_paged_decode_workspace_size(64, 12, 128, 512, 16) == big
    finally:
        L.fa_set_decode_split(old)


FAKE = 1 << 20  # 16-byte aligned, never dereferenced: every call below is rejected on the host


def fwd_args(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, Nq=128, Nkv=128, d=64, scale=0.125,
             causal=0, dtype=fa.FA_DTYPE_BF16, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize(
    "kw,code",
    [
        (dict(q=None), fa.FA_ERR_INVALID_ARG),
        (dict(lse=None), fa.FA_ERR_INVALID_ARG),
        (dict(B=0), fa.FA_ERR_INVALID_ARG),
        (dict(Nkv=-1), fa.FA_ERR_INVALID_ARG),
        (dict(Hq=5, Hkv=2), fa.FA_ERR_INVALID_ARG),
        (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
        (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
        (dict(causal=2), fa.FA_ERR_INVALID_ARG),
        (dict(causal=1, Nq=200, Nkv=100), fa.FA_ERR_INVALID_ARG),
        (dict(q=FAKE + 8), fa.FA_ERR_INVALID_ARG),
        (dict(lse=FAKE + 2), fa.FA_ERR_INVALID_ARG),
        (dict(d=80), fa.FA_ERR_UNSUPPORTED),
        (dict(d=128, dtype=fa.FA_DTYPE_F32), fa.FA_ERR_UNSUPPORTED),
        (dict(dtype=7), fa.FA_ERR_UNSUPPORTED),
        (dict(B=70000, Hq=2, Hkv=2), fa.FA_ERR_UNSUPPORTED),
    ],
)
def test_fwd_rejects_on_host(L, kw, code):
    assert L.fa_fwd(*fwd_args(**kw)) == code


def bwd_args(**kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, do=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
             grad_dtype=fa.FA_DTYPE_F32, B=1, Hq=4, Hkv=2, Nq=128, Nkv=128, d=64, scale=0.125, causal=1,
             dtype=fa.FA_DTYPE_BF16, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize(
    "kw,code",
    [
        (dict(do=None), fa.FA_ERR_INVALID_ARG),
        (dict(dk=FAKE + 4), fa.FA_ERR_INVALID_ARG),
        (dict(Hq=3), fa.FA_ERR_INVALID_ARG),
        (dict(causal=1, Nq=256), fa.FA_ERR_INVALID_ARG),
        (dict(dtype=fa.FA_DTYPE_F32, d=128), fa.FA_ERR_UNSUPPORTED),
        (dict(dtype=fa.FA_DTYPE_F32, grad_dtype=fa.FA_DTYPE_BF16), fa.FA_ERR_UNSUPPORTED),
        (dict(grad_dtype=9), fa.FA_ERR_UNSUPPORTED),
        (dict(d=192), fa.FA_ERR_UNSUPPORTED),
        (dict(d=256, dtype=fa.FA_DTYPE_F32), fa.FA_ERR_UNSUPPORTED),
        (dict(d=256, ws=None), fa.FA_ERR_WORKSPACE),
        (dict(ws=None), fa.FA_ERR_WORKSPACE),
        (dict(ws_bytes=1000), fa.FA_ERR_WORKSPACE),
        (dict(ws=FAKE + 16), fa.FA_ERR_WORKSPACE),
    ],
)
def test_bwd_rejects_on_host(L, kw, code):
    assert L.fa_bwd(*bwd_args(**kw)) == code


def dec_args(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, ctx=FAKE, o=FAKE, lse=None, R=4, Hq=12, Hkv=2, d=128, bs=16,
             maxb=64, nblocks=100, scale=0.088, dtype=fa.FA_DTYPE_BF16, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize(
    "kw,code",
    [
        (dict(bt=None), fa.FA_ERR_INVALID_ARG),
        (dict(ctx=None), fa.FA_ERR_INVALID_ARG),
        (dict(nblocks=0), fa.FA_ERR_INVALID_ARG),
        (dict(Hq=13), fa.FA_ERR_INVALID_ARG),
        (dict(bt=FAKE + 2), fa.FA_ERR_INVALID_ARG),
        (dict(o=FAKE + 4), fa.FA_ERR_INVALID_ARG),
        (dict(d=64), fa.FA_ERR_UNSUPPORTED),
        (dict(bs=32), fa.FA_ERR_UNSUPPORTED),
        (dict(dtype=fa.FA_DTYPE_F32), fa.FA_ERR_UNSUPPORTED),
        (dict(Hq=34, Hkv=2), fa.FA_ERR_UNSUPPORTED),
        (dict(ws=None), fa.FA_ERR_WORKSPACE),
        (dict(ws_bytes=16), fa.FA_ERR_WORKSPACE),
    ],
)
def test_decode_rejects_on_host(L, kw, code):
    assert L.fa_paged_decode(*dec_args(**kw)) == code


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(fa, "_lib", None)
    monkeypatch.setattr(fa, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fa.lib()


def test_binding_rejects_cpu_tensors():
    import torch

    x = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        fa.fwd(x, x, x)


def pre_args(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, ctx=FAKE, ql=FAKE, o=FAKE, lse=FAKE, R=4, Hq=8, Hkv=2, Nq=512,
             d=128, bs=16, maxb=64, nblocks=100, scale=0.088, causal=1, dtype=fa.FA_DTYPE_BF16, stream=None)
    a.update(kw)
    return list(a.values())


@pytest.mark.parametrize(
    "kw,code",
    [
        (dict(ql=None), fa.FA_ERR_INVALID_ARG),
        (dict(lse=None), fa.FA_ERR_INVALID_ARG),
        (dict(Nq=0), fa.FA_ERR_INVALID_ARG),
        (dict(Hq=6, Hkv=4), fa.FA_ERR_INVALID_ARG),
        (dict(causal=3), fa.FA_ERR_INVALID_ARG),
        (dict(kc=FAKE + 8), fa.FA_ERR_INVALID_ARG),
        (dict(ctx=FAKE + 2), fa.FA_ERR_INVALID_ARG),
        (dict(d=80), fa.FA_ERR_UNSUPPORTED),
        (dict(bs=32), fa.FA_ERR_UNSUPPORTED),
        (dict(dtype=fa.FA_DTYPE_F32), fa.FA_ERR_UNSUPPORTED),
        (dict(R=70000), fa.FA_ERR_UNSUPPORTED),
    ],
)
def test_paged_prefill_rejects_on_host(L, kw, code):
    assert L.fa_paged_prefill(*pre_args(**kw)) == code
