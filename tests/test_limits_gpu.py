"""Size limits on the GPU: a packed batch at the 2048-sequence limit, one
65536-token sequence, and 2048 short heads, each against the float64 oracle
-- element by element where the oracle finishes quickly, else on sampled rows
and through identities that hold at any size."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import fixed_inputs, varlen_inputs
from oracle import oracle as orc

from helpers import (assert_close_bf16, assert_close_bf16_scaled, assert_close_lse, gather_rows,
                     sample_rows, to64)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 3)])
def test_packed_batch_at_the_sequence_limit(causal, window):
    # 2048 sequences (the packed-batch limit) of 1..40 tokens, H2 d64
    x = varlen_inputs(2048, 1, 40, 2, 64, seed=17, with_dout=True)
    cu = x["cu_seqlens"]
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    cu_d = cu.to(DEV)
    o, lse = fa.forward(q, k, v, causal=causal, window=window, cu_seqlens=cu_d)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=causal, window=window, cu_seqlens=cu_d)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    scale = 1 / math.sqrt(64)
    O, L = orc.fwd(x["q"], x["k"], x["v"], scale, causal=causal, window=window, cu_seqlens=cu)
    assert_close_bf16(o, O, "O")
    assert_close_lse(lse, L)
    r = orc.bwd(x["q"], x["k"], x["v"], x["dout"], scale, causal=causal, window=window,
                cu_seqlens=cu)
    # sequences of a few tokens give gradients of several units (a query that
    # sees two keys gets dS of the size of dO.v); their bf16 rounding alone
    # exceeds the absolute bound, so the bound scales with |ref| beyond 1
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_close_bf16_scaled(t, r[name], name)


@pytest.mark.parametrize("causal", [False, True])
def test_one_sequence_of_65536_tokens(causal):
    N, d = 65536, 128
    x = fixed_inputs(1, N, 1, d, seed=23, with_dout=True)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v, causal=causal)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=causal)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    scale = 1 / math.sqrt(d)
    # forward: sampled rows (tile edges and random rows) against the oracle
    rows = sample_rows([N], 1, 48, seed=5)
    Or, Lr = orc.fwd_rows(x["q"], x["k"], x["v"], rows, scale, causal=causal)
    og, lg = gather_rows(o, lse, rows)
    assert_close_bf16(og, Or, "O rows")
    assert_close_lse(lg, Lr)
    # backward, element by element: dQ of the same sampled rows (each from its
    # own row's statistics); with the causal mask also dK and dV of key rows
    # in the last 1024 positions (only the queries after a key attend it, so
    # the oracle needs the statistics of those rows alone)
    qrows = rows
    krows = np.zeros((0, 3), dtype=np.int32)
    if causal:
        rng = np.random.default_rng(7)
        tail = {N - 1, N - 2, N - 128, N - 129, N - 256}
        tail |= {int(j) for j in rng.integers(N - 1024, N, 16)}
        krows = np.array([[0, 0, j] for j in sorted(tail)], dtype=np.int32)
    dq_r, dk_r, dv_r = orc.bwd_rows(x["q"], x["k"], x["v"], x["dout"], scale, qrows, krows,
                                    causal=causal)
    g = {n: to64(t)[0, :, 0] for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    assert_close_bf16(np.stack([g["dq"][i] for _, _, i in qrows]), dq_r, "dq rows")
    if len(krows):
        assert_close_bf16(np.stack([g["dk"][j] for _, _, j in krows]), dk_r, "dk rows")
        assert_close_bf16(np.stack([g["dv"][j] for _, _, j in krows]), dv_r, "dv rows")
    # and over all rows: sum_j dV_j = sum_i dO_i (each row of P sums to one)
    # and sum_j dK_j = 0 (each row of dS sums to zero), both up to the bf16
    # rounding of the 65536 summed rows
    dv64, dk64 = to64(dv)[0, :, 0], to64(dk)[0, :, 0]
    do64 = x["dout"].double().numpy()[0, :, 0]
    err_v = np.abs(dv64.sum(0) - do64.sum(0)).max()
    assert err_v <= 1e-2 * np.abs(dv64).sum(0).max(), err_v
    err_k = np.abs(dk64.sum(0)).max()
    assert err_k <= 1e-2 * np.abs(dk64).sum(0).max(), err_k
    assert torch.isfinite(dq).all()


def test_many_short_heads():
    # 64 sequences x 32 heads of 128 tokens: 2048 one-block work units
    B, H, N, d = 64, 32, 128, 64
    x = fixed_inputs(B, N, H, d, seed=29, with_dout=True)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v, causal=True)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    scale = 1 / math.sqrt(d)
    O, L = orc.fwd(x["q"], x["k"], x["v"], scale, causal=True)
    assert_close_bf16(o, O, "O")
    assert_close_lse(lse, L)
    r = orc.bwd(x["q"], x["k"], x["v"], x["dout"], scale, causal=True)
    # under a causal mask the first keys' gradients are dominated by rows that
    # see a handful of keys (dV_0 holds dO_0 with weight 1): several units, so
    # the bound scales with |ref| beyond 1 as for the tiny packed sequences
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert_close_bf16_scaled(t, r[name], name)
