"""The C-ABI library builds, loads and exports every symbol its header
declares; argument validation rejects bad calls on the host, with nothing
launched (these calls never reach a GPU)."""
import ctypes
import os
import re

import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "fa.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = fa.load_library()
    syms = declared_symbols()
    assert "fa_fwd" in syms and "fa_bwd" in syms
    for s in syms:
        assert hasattr(lib, s), s
    # the binding wraps every declared entry point under the same name
    for s in syms:
        assert s in binding.SIGNATURES, s
        assert hasattr(fa, s), s


def test_status_strings():
    for code in binding.STATUS:
        assert fa.fa_status_string(code)
    assert fa.fa_status_string(12345) == "unknown status"


# Fake, 16-byte aligned "device" addresses: validation fails before any use.
P = 0x10000


def fwd(**kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=128, d=128, scale=0.1, causal=0,
                window=0, cu_seqlens=None, stream=0)
    args.update(kw)
    return fa.fa_fwd(**args)


def bwd(**kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=1, H=1, N=128, d=128,
                scale=0.1, causal=0, window=0, cu_seqlens=None, workspace=P,
                workspace_bytes=1 << 20, stream=0)
    args.update(kw)
    return fa.fa_bwd(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(lse=None), -1),
    (dict(d=96), -2), (dict(d=256), -2),
    (dict(H=0), -3), (dict(B=-1), -3), (dict(N=-5), -3),
    (dict(q=P + 8), -4), (dict(o=P + 2), -4),
    (dict(window=16), -5),
    (dict(scale=0.0), -9), (dict(scale=-1.0), -9), (dict(scale=float("inf")), -9),
    (dict(cu_seqlens=P, B=5000, N=100), -3),
    (dict(cu_seqlens=P + 2, B=2, N=100), -4),
])
def test_fwd_validation(kw, code):
    assert fwd(**kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dout=None), -1), (dict(dv=None), -1),
    (dict(d=32), -2),
    (dict(dq=P + 4), -4),
    (dict(window=3), -5),
    (dict(workspace=None), -6), (dict(workspace_bytes=16), -6),
    (dict(workspace=P + 8), -4),
])
def test_bwd_validation(kw, code):
    assert bwd(**kw) == code


def fwd_kv(**kw):
    args = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Nq=128, Nk=512, d=128, scale=0.1,
                causal=1, window=0, cu_seqlens_q=None, cu_seqlens_k=None, stream=0)
    args.update(kw)
    return fa.fa_fwd_kv(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(k=None), -1), (dict(lse=None), -1),
    (dict(d=80), -2),
    (dict(Nk=-1), -3), (dict(Nq=-1), -3),
    (dict(cu_seqlens_q=P), -3), (dict(cu_seqlens_k=P), -3),
    (dict(cu_seqlens_q=P, cu_seqlens_k=P + 2), -4),
    (dict(v=P + 4), -4),
    (dict(causal=0, window=8), -5),
    (dict(scale=float("nan")), -9),
])
def test_fwd_kv_validation(kw, code):
    assert fwd_kv(**kw) == code


def kvcache(**kw):
    args = dict(q=P, k_cache=P, v_cache=P, o=P, lse=P, B=2, H=2, Nq=1, Nk=512, d=128, scale=0.1,
                causal=1, window=0, seqlens_k=None, num_splits=1, workspace=None,
                workspace_bytes=0, stream=0)
    args.update(kw)
    return fa.fa_fwd_kvcache(**args)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(v_cache=None), -1),
    (dict(d=96), -2),
    (dict(Nk=-1), -3), (dict(num_splits=33), -3), (dict(num_splits=-1), -3),
    (dict(seqlens_k=P + 2), -4), (dict(o=P + 8), -4),
    (dict(causal=0, window=4), -5),
    (dict(scale=0.0), -9),
    (dict(num_splits=4), -6), (dict(num_splits=4, workspace=P, workspace_bytes=64), -6),
    (dict(num_splits=4, workspace=P + 4, workspace_bytes=1 << 20), -4),
])
def test_kvcache_validation(kw, code):
    assert kvcache(**kw) == code


def test_kvcache_workspace_size_and_splits():
    # num_splits * B * Nq * H * (d + 1) * 4, rounded to 256; none for one split
    assert fa.fa_fwd_kvcache_workspace_size(2, 2, 1, 128, 4) == 8448      # 8256 rounded up
    assert fa.fa_fwd_kvcache_workspace_size(16, 16, 1, 128, 8) == 8 * 16 * 16 * 129 * 4
    assert fa.fa_fwd_kvcache_workspace_size(2, 2, 1, 128, 1) == 0
    assert fa.fa_fwd_kvcache_workspace_size(0, 2, 1, 128, 4) == 0
    assert fa.fa_fwd_kvcache_num_splits(0, 1, 1, 128, 128) == 1
    ns = fa.fa_fwd_kvcache_num_splits(16, 16, 1, 8192, 128)
    assert 1 <= ns <= 32
    # at least 4 key tiles of 64 per split
    assert fa.fa_fwd_kvcache_num_splits(1, 1, 1, 300, 128) == 1


def test_fp8_validation_on_host():
    def quant(**kw):
        a = dict(x=P, out=P, scales=P, B=1, N=128, H=1, d=128, transpose=0, signs=None, stream=0)
        a.update(kw)
        return fa.fa_quantize_fp8(**a)

    def fwd8(**kw):
        a = dict(q8=P, k8=P, vt8=P, sq=P, sk=P, sv=P, o=P, lse=P, B=1, H=1, N=128, d=128,
                 scale=0.1, causal=0, window=0, stream=0)
        a.update(kw)
        return fa.fa_fwd_fp8(**a)

    assert quant(x=None) == -1 and quant(d=64) == -2 and quant(N=-1) == -3
    assert quant(transpose=1, signs=P) == -3          # no rotation for V
    assert quant(out=P + 8) == -4 and quant(scales=P + 2) == -4
    assert quant(N=0) == 0
    assert fwd8(sv=None) == -1 and fwd8(d=64) == -2 and fwd8(window=5) == -5
    assert fwd8(k8=P + 4) == -4 and fwd8(scale=-1.0) == -9 and fwd8(B=0) == 0
    # V codes transposed to [B, H, 128, N rounded up to 16]
    assert fa.fa_fp8_vt_bytes(2, 3, 200, 128) == 2 * 3 * 128 * 208
    assert fa.fa_fp8_vt_bytes(2, 3, 200, 64) == 0


def test_empty_problems_are_noops():
    assert kvcache(Nq=0) == 0
    assert kvcache(B=0) == 0
    assert fwd_kv(B=0) == 0
    assert fwd_kv(Nq=0) == 0
    assert fwd(B=0) == 0
    assert fwd(N=0) == 0
    assert bwd(B=0, workspace=None, workspace_bytes=0) == 0


def test_workspace_size():
    # 8 bytes per (head, row), each sequence padded to 128 rows
    assert fa.fa_bwd_workspace_size(2, 16, 4096, 128, 0) == 2 * 16 * 4096 * 8
    assert fa.fa_bwd_workspace_size(2, 16, 4000, 128, 0) == 2 * 16 * 4096 * 8
    # packed: H * roundup(T + 127 B, 128) * 8
    assert fa.fa_bwd_workspace_size(16, 32, 0, 128, 1000) == 32 * 3072 * 8
    assert fa.fa_bwd_workspace_size(1, 1, 1, 64, 0) == 128 * 8
    assert fa.fa_bwd_workspace_size(0, 1, 1, 64, 0) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_reports_cuda_error():
    assert fwd() == -7
    assert fwd_kv() == -7
    assert fwd_kv(Nk=0) == -7
    assert fwd_kv(Nk=0, k=None, v=None) == -7      # no key rows: k, v may be NULL


def test_noalloc_validation_on_host():
    base = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=1, H=1, N=128, d=128,
                scale=0.1, causal=0, window=0, cu_seqlens=None, stream=0)

    def call(**kw):
        a = dict(base)
        a.update(kw)
        return fa.fa_bwd_noalloc(**a)

    assert call(dq=None) == -1
    assert call(d=80) == -2
    assert call(window=4) == -5
    assert call(dv=P + 8) == -4
    # a workspace above the built-in scratch (8 * FA_NOALLOC_MAX_ROWS bytes) is rejected
    assert call(H=16, N=binding.NOALLOC_MAX_ROWS // 16 + 1) == -10
    assert call(H=16, N=binding.NOALLOC_MAX_ROWS // 16) == -7 or torch.cuda.is_available()
    assert call(B=0) == 0
    header = open(HEADER).read()
    assert "#define FA_NOALLOC_MAX_ROWS (1 << 20)" in header
    assert binding.NOALLOC_MAX_ROWS == 1 << 20
