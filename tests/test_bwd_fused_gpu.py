"""The single-kernel backward (fa_bwd_fused, d = 128) on the GPU: gradients
against the float64 oracle element by element on small and ragged shapes,
masks and packed batches, one whole head of the B4 H16 N8192 workload, and
against fa_bwd (dK and dV bit for bit: the same arithmetic in the same order;
dQ within the parity tolerance, its fp32 additions land in any order)."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import WORKLOADS, fixed_inputs, varlen_inputs
from oracle import oracle as orc

from helpers import assert_close_bf16, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run(x, causal, window, cu=None, fused=True):
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    cu_d = None if cu is None else cu.to(DEV)
    o, lse = fa.forward(q, k, v, causal=causal, window=window, cu_seqlens=cu_d)
    g = fa.backward(q, k, v, o, lse, do, causal=causal, window=window, cu_seqlens=cu_d, fused=fused)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return g


SMALL = [(1, 1, 128), (1, 2, 17), (2, 2, 129), (1, 2, 300), (2, 1, 513), (1, 1, 1), (1, 3, 1000)]
MASKS = [(False, 0), (True, 0), (True, 1), (True, 100)]


@pytest.mark.parametrize("B,H,N", SMALL)
@pytest.mark.parametrize("causal,window", MASKS)
def test_fused_bwd_small_elementwise(B, H, N, causal, window):
    x = fixed_inputs(B, N, H, 128, seed=500 + N, with_dout=True)
    grads = run(x, causal, window)
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(128), causal=causal,
                  window=window)
    for name, t in zip(("dq", "dk", "dv"), grads):
        assert_close_bf16(t, ref[name], name)


@pytest.mark.parametrize("lens", [[1, 127, 128, 129, 200], [5, 300, 64]])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 33)])
def test_fused_bwd_packed_elementwise(lens, causal, window):
    x = varlen_inputs(len(lens), 0, 0, 2, 128, seed=51, with_dout=True, lengths=lens)
    cu = x["cu_seqlens"]
    grads = run(x, causal, window, cu)
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(128), causal=causal,
                  window=window, cu_seqlens=cu)
    for name, t in zip(("dq", "dk", "dv"), grads):
        assert_close_bf16(t, ref[name], name)


def test_fused_bwd_matches_two_kernel_backward():
    x = fixed_inputs(2, 700, 3, 128, seed=52, with_dout=True)
    gf = run(x, True, 0)
    g2 = run(x, True, 0, fused=False)
    assert torch.equal(gf[1], g2[1]) and torch.equal(gf[2], g2[2])
    assert_close_bf16(gf[0], to64(g2[0]), "dq vs fa_bwd")


def test_fused_bwd_bench_configuration_one_head():
    """B4 H16 N8192 d128 non-causal (the bench's workload): one head in full."""
    wl = WORKLOADS["prefill_b4"]
    x = fixed_inputs(wl.B, wl.N, wl.H, wl.d, seed=wl.seed, with_dout=True)
    dq, dk, dv = run(x, False, 0)
    heads = [(1, 5)]
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], wl.scale, causal=False, heads=heads)
    for s, h in heads:
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_close_bf16(t[s, :, h], ref[name][s, :, h], "%s[%d,:,%d]" % (name, s, h))
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()


def test_fused_bwd_rejects_d64():
    x = fixed_inputs(1, 64, 1, 64, seed=53, with_dout=True)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v)
    assert fa.fa_bwd_fused_workspace_size(1, 1, 64, 64, 0) == 0
    rc = fa.fa_bwd_fused(q, k, v, o, lse, do, q, k, v, 1, 1, 64, 64, 0.125, 0, 0, None, q, 1 << 20,
                         None)
    assert rc == -2
