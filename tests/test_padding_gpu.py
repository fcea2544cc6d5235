"""Packed buffers larger than their batch: the rows past cu_seqlens[B] belong
to no sequence and may hold anything.  Here they hold NaN.  The forward, the
backward (two-kernel, no-alloc and fused) and the cached-KV forward must give,
on the batch's rows, exactly what they give with zeros there, and match the
float64 oracle, which never sees those rows.  The last sequence ends inside
a 128-row tile in every case but one, so the tile loaded past it reaches
into the padding."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import varlen_inputs, varlen_kv_inputs
from oracle import oracle as orc

from helpers import TOL_LSE, assert_close_bf16, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAD = 77


def padded(t, rows, value):
    """t with `rows` more rows of `value` after it (first dimension)."""
    extra = torch.full((rows,) + tuple(t.shape[1:]), value, dtype=t.dtype)
    return torch.cat([t, extra], 0)


def run_self(x, causal, window, mode, value):
    T = int(x["cu_seqlens"][-1])
    q, k, v, do = (padded(x[n], PAD, value).to(DEV) for n in ("q", "k", "v", "dout"))
    cu = x["cu_seqlens"].to(DEV)
    o, lse = fa.forward(q, k, v, causal=causal, window=window, cu_seqlens=cu)
    if mode == "noalloc":
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        rc = fa.fa_bwd_noalloc(q, k, v, o, lse, do, *grads, cu.numel() - 1, q.shape[1],
                               q.shape[0], q.shape[2], 1 / math.sqrt(q.shape[2]), int(causal),
                               window, cu, None)
        assert rc == 0, fa.fa_status_string(rc)
    else:
        grads = fa.backward(q, k, v, o, lse, do, causal=causal, window=window, cu_seqlens=cu,
                            fused=(mode == "fused"))
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return [o[:T].clone(), lse[:, :T].clone()] + [g[:T].clone() for g in grads]


@pytest.mark.parametrize("lens", [[100, 300, 77], [129, 5], [1000, 64], [300], [128, 256]])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 33)])
@pytest.mark.parametrize("mode", ["two_kernel", "noalloc", "fused"])
def test_nan_rows_past_the_batch(lens, causal, window, mode):
    x = varlen_inputs(len(lens), 0, 0, 2, 128, seed=len(lens) + sum(lens), with_dout=True,
                      lengths=lens)
    got = run_self(x, causal, window, mode, float("nan"))
    ref = run_self(x, causal, window, mode, 0.0)
    for name, a, b in zip(("o", "lse", "dq", "dk", "dv"), got, ref):
        if mode == "fused" and name == "dq":
            # its dQ parts are added by fp32 reductions in no fixed order, so two
            # runs need not agree bit for bit: finite, and within the oracle's
            # tolerance below
            assert torch.isfinite(a).all(), "dq has non-finite values with NaN padding"
            continue
        assert torch.equal(a, b), "%s differs with NaN padding" % name
    cu = x["cu_seqlens"]
    O, L = orc.fwd(x["q"], x["k"], x["v"], 1 / math.sqrt(128), causal=causal, window=window,
                   cu_seqlens=cu)
    assert_close_bf16(got[0], O, "O")
    assert np.abs(to64(got[1]) - L).max() <= TOL_LSE
    r = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(128), causal=causal,
                window=window, cu_seqlens=cu)
    for name, t in zip(("dq", "dk", "dv"), got[2:]):
        assert_close_bf16(t, r[name], name)


@pytest.mark.parametrize("lens,causal,window", [([100, 300, 77], True, 0), ([129, 5], False, 0),
                                                ([1000, 64], True, 33)])
@pytest.mark.parametrize("mode", ["two_kernel", "noalloc"])
def test_nan_rows_past_the_batch_d64(lens, causal, window, mode):
    x = varlen_inputs(len(lens), 0, 0, 3, 64, seed=7 + sum(lens), with_dout=True, lengths=lens)
    got = run_self(x, causal, window, mode, float("nan"))
    ref = run_self(x, causal, window, mode, 0.0)
    for name, a, b in zip(("o", "lse", "dq", "dk", "dv"), got, ref):
        assert torch.equal(a, b), "%s differs with NaN padding" % name
    cu = x["cu_seqlens"]
    r = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(64), causal=causal,
                window=window, cu_seqlens=cu)
    assert_close_bf16(got[0], r["o"], "O")
    for name, t in zip(("dq", "dk", "dv"), got[2:]):
        assert_close_bf16(t, r[name], name)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lq,lk,causal", [([50, 200], [300, 700], True), ([17, 129], [129, 255], False),
                                          ([40], [1000], True)])
def test_nan_rows_past_the_batch_cached_kv(lq, lk, causal, d):
    x = varlen_kv_inputs(lq, lk, 2, d, seed=3 + sum(lk))
    Tq = int(x["cu_seqlens_q"][-1])
    outs = []
    for value in (float("nan"), 0.0):
        q = padded(x["q"], 33, value).to(DEV)
        k, v = (padded(x[n], PAD, value).to(DEV) for n in ("k", "v"))
        o, lse = fa.forward_kv(q, k, v, causal=causal, cu_seqlens_q=x["cu_seqlens_q"].to(DEV),
                               cu_seqlens_k=x["cu_seqlens_k"].to(DEV))
        torch.cuda.synchronize()
        assert fa.fa_get_device_error() == 0
        outs.append((o[:Tq].clone(), lse[:, :Tq].clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    O, L = orc.fwd_kv(x["q"], x["k"], x["v"], 1 / math.sqrt(d), causal=causal,
                      cu_seqlens_q=x["cu_seqlens_q"], cu_seqlens_k=x["cu_seqlens_k"])
    assert_close_bf16(outs[0][0], O, "O")
    g = to64(outs[0][1])
    fin = np.isfinite(L)
    assert np.array_equal(np.isneginf(g), np.isneginf(L))
    if fin.any():
        assert np.abs(g[fin] - L[fin]).max() <= TOL_LSE
