"""The torch-level wrappers derive the library's size arguments from the
tensors and refuse tensors that do not match them, on the CPU: the library
calls are replaced by recorders (and the CUDA-device requirement lifted), so
that the accepted argument patterns -- those the GPU tests and bench.py use --
and the refusals are checked without a GPU."""
import pytest
import torch

from io_aware_exact_21_b200 import binding as bd
from io_aware_exact_21_b200.inputs import (fixed_inputs, fp8_signs, kv_inputs, kvcache_inputs,
                                           varlen_inputs, varlen_kv_inputs)


@pytest.fixture
def calls(monkeypatch):
    rec = []
    monkeypatch.setattr(bd, "_require_cuda", lambda t, name: None)

    def recorder(name):
        def f(*args):
            rec.append((name, args))
            return 0
        return f

    for name in ("fa_fwd", "fa_fwd_kv", "fa_fwd_kvcache", "fa_bwd", "fa_quantize_fp8",
                 "fa_fwd_fp8"):
        monkeypatch.setattr(bd, name, recorder(name))
    monkeypatch.setattr(bd, "fa_bwd_workspace_size", lambda B, H, N, d, t=0: 4096)
    monkeypatch.setattr(bd, "fa_fwd_kvcache_num_splits", lambda B, H, Nq, Nk, d: 3)
    monkeypatch.setattr(bd, "fa_fwd_kvcache_workspace_size", lambda B, H, Nq, d, ns: 1024)
    monkeypatch.setattr(bd, "fa_fp8_vt_bytes", lambda B, H, N, d: B * H * d * ((N + 15) // 16 * 16))
    return rec


def sizes(call, n):
    return call[1][n:n + 4]


def test_forward_and_backward_fixed(calls):
    x = fixed_inputs(2, 130, 3, 64, seed=1, with_dout=True)
    o, lse = bd.forward(x["q"], x["k"], x["v"], causal=True)
    assert o.shape == x["q"].shape and lse.shape == (2, 3, 130)
    assert calls[-1][0] == "fa_fwd" and sizes(calls[-1], 5) == (2, 3, 130, 64)
    grads = bd.backward(x["q"], x["k"], x["v"], o, lse, x["dout"], causal=True)
    assert [g.shape for g in grads] == [x["q"].shape] * 3
    assert calls[-1][0] == "fa_bwd" and sizes(calls[-1], 9) == (2, 3, 130, 64)


def test_forward_and_backward_packed(calls):
    x = varlen_inputs(4, 1, 50, 2, 128, seed=2, with_dout=True)
    cu = x["cu_seqlens"]
    T = x["q"].shape[0]
    o, lse = bd.forward(x["q"], x["k"], x["v"], cu_seqlens=cu)
    assert lse.shape == (2, T)
    assert sizes(calls[-1], 5) == (4, 2, T, 128)
    bd.backward(x["q"], x["k"], x["v"], o, lse, x["dout"], cu_seqlens=cu)
    assert sizes(calls[-1], 9) == (4, 2, T, 128)


def test_cached_kv_fixed_and_packed(calls):
    x = kv_inputs(2, 40, 300, 2, 128, seed=3)
    o, lse = bd.forward_kv(x["q"], x["k"], x["v"], causal=True)
    assert lse.shape == (2, 2, 40)
    assert calls[-1][1][5:10] == (2, 2, 40, 300, 128)
    y = varlen_kv_inputs([3, 5], [10, 20], 2, 64, seed=4)
    bd.forward_kv(y["q"], y["k"], y["v"], cu_seqlens_q=y["cu_seqlens_q"],
                  cu_seqlens_k=y["cu_seqlens_k"])
    assert calls[-1][1][5:10] == (2, 2, 8, 30, 64)


def test_cache_interface(calls):
    x = kvcache_inputs(3, 2, 500, 2, 128, seed=5, lens=(0, 500))
    o, lse = bd.forward_kvcache(x["q"], x["k"], x["v"], seqlens_k=x["seqlens_k"], causal=True)
    assert lse.shape == (3, 2, 2)
    args = calls[-1][1]
    assert args[5:10] == (3, 2, 2, 500, 128) and args[14] == 3 and args[16] == 1024
    ws = torch.empty(1024, dtype=torch.uint8)
    bd.forward_kvcache(x["q"], x["k"], x["v"], workspace=ws)


def test_fp8(calls):
    x = fixed_inputs(1, 200, 2, 128, seed=6)
    qz = bd.quantize_fp8(x["q"], x["k"], x["v"], fp8_signs(1))
    assert [c[0] for c in calls[-3:]] == ["fa_quantize_fp8"] * 3
    o, lse = bd.forward_fp8(qz, 1, 200, 2)
    assert o.shape == (1, 200, 2, 128) and lse.shape == (1, 2, 200)


def test_refusals(calls):
    x = fixed_inputs(2, 64, 2, 64, seed=7, with_dout=True)
    q, k, v = x["q"], x["k"], x["v"]
    with pytest.raises(TypeError):
        bd.forward(q, k.float(), v)                            # dtype
    with pytest.raises(ValueError):
        bd.forward(q, k[:, :32].contiguous(), v)               # fewer keys than queries
    with pytest.raises(ValueError):
        bd.forward(q.transpose(1, 2).contiguous().transpose(1, 2), k, v)   # strided view
    with pytest.raises(ValueError):
        bd.forward(q, k, v, lse=torch.empty(2, 2, 63))         # output too small
    with pytest.raises(ValueError):
        bd.backward(q, k, v, q, torch.empty(2, 2, 64), x["dout"],
                    workspace=torch.empty(100, dtype=torch.uint8))   # workspace too small
    y = varlen_inputs(3, 1, 20, 2, 64, seed=8)
    with pytest.raises(TypeError):
        bd.forward(y["q"], y["k"], y["v"], cu_seqlens=y["cu_seqlens"].long())
    z = kvcache_inputs(2, 1, 100, 2, 64, seed=9, lens=(0, 100))
    with pytest.raises(ValueError):
        bd.forward_kvcache(z["q"], z["k"], z["v"], seqlens_k=z["seqlens_k"][:1])
    w = varlen_kv_inputs([3, 5], [10, 20], 2, 64, seed=10)
    with pytest.raises(ValueError):
        bd.forward_kv(w["q"], w["k"], w["v"], cu_seqlens_q=w["cu_seqlens_q"])
    assert not calls                                           # nothing reached the library
