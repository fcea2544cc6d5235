"""The softmax scale as an argument: every other GPU test runs at the default
1/sqrt(d), so a kernel that ignored the argument and used 1/sqrt(d) itself
would pass them.  Here the forward (fixed and packed), the backward, the
cached-KV forward and decode run at scales far from the default (sharper and
flatter softmaxes), element by element against the float64 oracle called
with the same scale: the forwards within the usual tolerances, the backward
within element-wise bounds derived from its bf16 roundings (they grow with
the scale; see backward_bounds)."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import fixed_inputs, kv_inputs, varlen_inputs
from oracle import oracle as orc

from helpers import assert_close_bf16, assert_close_lse, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
SCALES = [0.05, 0.37]


def _check_default_differs(d, scale):
    # the cases mean something only if the scale is not the default one
    assert abs(scale - 1 / math.sqrt(d)) > 0.02


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("B,H,N,d,causal,window", [(2, 2, 300, 128, False, 0),
                                                    (2, 2, 300, 128, True, 0),
                                                    (1, 3, 257, 64, True, 100)])
def test_forward_scale(scale, B, H, N, d, causal, window):
    _check_default_differs(d, scale)
    x = fixed_inputs(B, N, H, d, seed=700 + N)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, causal=causal, window=window, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    O, L = orc.fwd(x["q"], x["k"], x["v"], scale, causal=causal, window=window)
    assert_close_bf16(o, O, "O")
    assert_close_lse(lse, L)


@pytest.mark.parametrize("scale", SCALES)
def test_forward_packed_scale(scale):
    x = varlen_inputs(3, 1, 400, 2, 128, seed=711)
    cu = x["cu_seqlens"]
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = fa.forward(q, k, v, causal=True, cu_seqlens=cu.to(DEV), scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    O, L = orc.fwd(x["q"], x["k"], x["v"], scale, causal=True, cu_seqlens=cu)
    assert_close_bf16(o, O, "O")
    assert_close_lse(lse, L)


def backward_bounds(x, o_bf16, scale, causal, window):
    """Element-wise error bounds of the gradients, from the arithmetic the
    kernels use, evaluated in float64 per (sequence, head):
      dS = P (dP - D) is rounded to bf16 before the dQ and dK GEMMs (relative
      2^-9 per element), P to bf16 before the dV GEMM, and D is taken from the
      bf16 output O (relative 2^-9 per term of dO . O); products of bf16
      operands are exact and the float32 sums add nothing of this size; each
      output is rounded to bf16 (2^-9 of its value).  So, with
      dD_i = 2^-9 sum_c |dO_ic O_ic|,
      dq: scale (2^-9 |dS| |K| + |P| diag(dD) |K|) + 2^-9 |dq|
      dk: scale (2^-9 |dS|^T |Q| + |P|^T diag(dD) |Q|) + 2^-9 |dk|
      dv: 2^-9 |P|^T |dO| + 2^-9 |dv|
    With scales far above 1/sqrt(d) the softmax is sharp, dS has large terms
    that cancel, and these bounds grow past the fixed absolute tolerance of
    the other tests, so this test uses them (times 2) instead."""
    u = 2.0 ** -9
    q, k, v, do = (x[n].double().numpy() for n in ("q", "k", "v", "dout"))
    o = o_bf16.detach().cpu().double().numpy()
    B, N, H, d = q.shape
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    allowed = np.ones((N, N), dtype=bool)
    if causal:
        allowed &= j <= i
    if window > 0:
        allowed &= j > i - window
    out = {n: np.zeros((B, N, H, d)) for n in ("dq", "dk", "dv")}
    for b in range(B):
        for h in range(H):
            Q, K, V, dO, O = q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], o[b, :, h]
            S = np.where(allowed, scale * Q @ K.T, -np.inf)
            P = np.exp(S - S.max(1, keepdims=True))
            P /= P.sum(1, keepdims=True)
            dP = dO @ V.T
            D = (P * dP).sum(1, keepdims=True)
            dS = P * (dP - D)
            dD = u * np.abs(dO * O).sum(1, keepdims=True)
            out["dq"][b, :, h] = scale * (u * np.abs(dS) @ np.abs(K) + (P * dD) @ np.abs(K))
            out["dk"][b, :, h] = scale * (u * np.abs(dS).T @ np.abs(Q) + (P * dD).T @ np.abs(Q))
            out["dv"][b, :, h] = u * P.T @ np.abs(dO)
    return out


@pytest.mark.parametrize("scale", SCALES + [1 / math.sqrt(128)])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 64)])
def test_backward_scale(scale, causal, window):
    B, H, N, d = 1, 2, 300, 128
    x = fixed_inputs(B, N, H, d, seed=720, with_dout=True)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v, causal=causal, window=window, scale=scale)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=causal, window=window, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], scale, causal=causal, window=window)
    bound = backward_bounds(x, o, scale, causal, window)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        g = to64(t)
        err = np.abs(g - ref[name])
        tol = 2.0 * (bound[name] + 2.0 ** -9 * np.abs(ref[name])) + 1e-3
        worst = np.unravel_index(np.argmax(err / tol), err.shape)
        assert (err <= tol).all(), "%s: err %.3e > tol %.3e at %s (ref %.3f)" % (
            name, err[worst], tol[worst], worst, ref[name][worst])


@pytest.mark.parametrize("scale", SCALES)
def test_forward_kv_scale(scale):
    x = kv_inputs(2, 100, 300, 2, 128, seed=730)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = fa.forward_kv(q, k, v, causal=True, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    O, L = orc.fwd_kv(x["q"], x["k"], x["v"], scale, causal=True)
    assert_close_bf16(o, O, "O")
    assert_close_lse(lse, L)


@pytest.mark.parametrize("scale", SCALES)
@pytest.mark.parametrize("num_splits", [1, 4])
def test_decode_scale(scale, num_splits):
    x = kv_inputs(3, 1, 700, 2, 128, seed=740)
    lens = torch.tensor([700, 513, 129], dtype=torch.int32)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o, lse = fa.forward_kvcache(q, k, v, seqlens_k=lens.to(DEV), causal=True, scale=scale,
                                num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    O, L = orc.fwd_kvcache(x["q"], x["k"], x["v"], scale, seqlens_k=lens, causal=True)
    assert_close_bf16(o, O, "O")
    g = to64(lse)
    assert np.isfinite(g).all()
    assert np.abs(g - L).max() <= 1e-3
