"""Backward parity on the GPU: fa_bwd (through the C ABI, after fa_fwd)
against the float64 oracle's gradients on the same seeded inputs, plus
gradient invariants, determinism and guard bands."""
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


def run(x, causal, window, cu=None):
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    cu_d = None if cu is None else cu.to(DEV)
    o, lse = fa.forward(q, k, v, causal=causal, window=window, cu_seqlens=cu_d)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, causal=causal, window=window, cu_seqlens=cu_d)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return o, lse, dq, dk, dv


def check(grads, ref):
    for name, t in zip(("dq", "dk", "dv"), grads):
        assert_close_bf16(t, ref[name], name)


SMALL = [(1, 1, 128, 64), (1, 2, 17, 128), (2, 2, 129, 64), (1, 2, 300, 128), (2, 1, 513, 64),
         (1, 1, 1, 128)]
MASKS = [(False, 0), (True, 0), (True, 1), (True, 100)]


@pytest.mark.parametrize("B,H,N,d", SMALL)
@pytest.mark.parametrize("causal,window", MASKS)
def test_bwd_small_elementwise(B, H, N, d, causal, window):
    x = fixed_inputs(B, N, H, d, seed=200 + N, with_dout=True)
    o, lse, dq, dk, dv = run(x, causal, window)
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(d), causal=causal,
                  window=window)
    check((dq, dk, dv), ref)


@pytest.mark.parametrize("lens", [[1, 127, 128, 129, 200], [5, 300, 64], [0, 129, 0, 300, 0]])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 33)])
def test_bwd_varlen_elementwise(lens, causal, window):
    x = varlen_inputs(len(lens), 0, 0, 2, 128, seed=21, with_dout=True, lengths=lens)
    cu = x["cu_seqlens"]
    o, lse, dq, dk, dv = run(x, causal, window, cu)
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(128), causal=causal,
                  window=window, cu_seqlens=cu)
    check((dq, dk, dv), ref)


def test_bwd_workload_parity_all_heads():
    """B=2, H=16, N=4096, d=128, causal: the gradients of all 32 (sequence,
    head) slices, element by element.  Under a causal mask the backward kernels
    deal the heads of the last round block by block (the snake tail), so this
    covers both kinds of schedule."""
    wl = WORKLOADS["bwd_causal"]
    x = wl.make()
    o, lse, dq, dk, dv = run(x, wl.causal, wl.window)
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], wl.scale, causal=True)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.isfinite(t).all(), name
        for s in range(wl.B):
            for h in range(wl.H):
                assert_close_bf16(t[s, :, h], ref[name][s, :, h], "%s[%d,:,%d]" % (name, s, h))


def test_bwd_invariants_and_determinism():
    B, N, H, d = 2, 700, 2, 128
    x = fixed_inputs(B, N, H, d, seed=22, with_dout=True)
    r1 = run(x, True, 0)
    r2 = run(x, True, 0)
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)
    dq, dk, dv = (to64(t) for t in r1[2:])
    # sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per (sequence, head), up to bf16 rounding
    assert np.abs(dk.sum(1)).max() < 0.5
    assert np.abs(dv.sum(1) - x["dout"].double().sum(1).numpy()).max() < 0.5


def test_bwd_uniform_varlen_equals_fixed():
    B, N, H, d = 2, 300, 2, 64
    x = fixed_inputs(B, N, H, d, seed=23, with_dout=True)
    r = run(x, True, 0)
    xp = {n: x[n].reshape(B * N, H, d) for n in ("q", "k", "v", "dout")}
    cu = torch.tensor([0, N, 2 * N], dtype=torch.int32)
    rp = run(xp, True, 0, cu)
    for a, b in zip(r[2:], rp[2:]):
        assert torch.equal(a.reshape(B * N, H, d), b)


def test_bwd_guard_bands():
    B, N, H, d = 1, 200, 2, 128
    x = fixed_inputs(B, N, H, d, seed=24, with_dout=True)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v, causal=True)
    guard = 2048
    sentinel = 777.0
    bufs = [torch.full((B * N * H * d + 2 * guard,), sentinel, dtype=torch.bfloat16, device=DEV)
            for _ in range(3)]
    views = [b[guard:guard + B * N * H * d].view(B, N, H, d) for b in bufs]
    ws_bytes = fa.fa_bwd_workspace_size(B, H, N, d, 0)
    ws = torch.full((ws_bytes // 4 + 2 * guard,), sentinel, dtype=torch.float32, device=DEV)
    rc = fa.fa_bwd(q, k, v, o, lse, do, views[0], views[1], views[2], B, H, N, d, d ** -0.5, 1, 0,
                   None, ws[guard:], ws_bytes, None)
    assert rc == 0
    torch.cuda.synchronize()
    for b in bufs:
        assert (b[:guard] == sentinel).all() and (b[-guard:] == sentinel).all()
    assert (ws[:guard] == sentinel).all() and (ws[guard + ws_bytes // 4:] == sentinel).all()
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], d ** -0.5, causal=True)
    check(views, ref)


def test_bwd_training_shape_causal_sampled_heads():
    """B=4, H=16, N=2048, d=128, causal (the training-shape inputs plus dO)."""
    wl = WORKLOADS["train_causal"]
    x = fixed_inputs(wl.B, wl.N, wl.H, wl.d, seed=wl.seed, with_dout=True)
    o, lse, dq, dk, dv = run(x, True, 0)
    # heads 37..63 in (sequence, head) order, e.g. (2, 7), (3, 12) and (3, 15),
    # are dealt block by block by the snake tail of the last round
    heads = [(0, 3), (2, 7), (3, 12), (3, 15)]
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], wl.scale, causal=True, heads=heads)
    for s, h in heads:
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_close_bf16(t[s, :, h], ref[name][s, :, h], "%s[%d,:,%d]" % (name, s, h))


@pytest.mark.parametrize("window", [0, 1024])
def test_bwd_packed_batch_sampled_sequences(window):
    """16 packed sequences, lengths U[128, 4096], H=32, d=128, causal (and a
    1024-key window): gradients of two (sequence, head) pairs checked in full,
    every output checked finite."""
    wl = WORKLOADS["varlen_window" if window else "varlen_causal"]
    nseq, lo, hi = wl.varlen
    x = varlen_inputs(nseq, lo, hi, wl.H, wl.d, wl.seed, with_dout=True)
    cu = x["cu_seqlens"]
    o, lse, dq, dk, dv = run(x, True, window, cu)
    lens = np.diff(cu.numpy())
    order = np.argsort(lens)
    heads = [(int(order[0]), 0), (int(order[nseq // 2]), wl.H - 1), (int(order[-1]), 5),
             (nseq - 1, wl.H - 1)]
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], wl.scale, causal=True, window=window,
                  cu_seqlens=cu, heads=heads)
    for s, h in heads:
        a, b = int(cu[s]), int(cu[s + 1])
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_close_bf16(t[a:b, h], ref[name][a:b, h], "%s[seq %d, head %d]" % (name, s, h))
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()


def test_bwd_bench_configuration_sampled_head():
    """The launch configuration bench.py times: B=4, H=16, N=8192, d=128,
    non-causal (seed 2, the prefill inputs plus dO); one head in full."""
    wl = WORKLOADS["prefill_b4"]
    x = fixed_inputs(wl.B, wl.N, wl.H, wl.d, seed=wl.seed, with_dout=True)
    o, lse, dq, dk, dv = run(x, False, 0)
    heads = [(2, 9)]
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], wl.scale, causal=False, heads=heads)
    for s, h in heads:
        for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
            assert_close_bf16(t[s, :, h], ref[name][s, :, h], "%s[%d,:,%d]" % (name, s, h))
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all()


@pytest.mark.parametrize("name", ["prefill_b4", "prefill_b4_causal", "train_causal"])
def test_bwd_sampled_rows_every_head(name):
    """Full-size backward, every (sequence, head): dQ of ten rows each (tile
    edges, the middle, the last rows and two seeded random rows) against the
    oracle's row-wise gradients; under the causal mask also dK and dV of
    eight key rows in the last 256 positions of four heads (the first, the
    last, and two the backward's snake tail deals), for which the oracle
    needs only the queries after them."""
    wl = WORKLOADS[name]
    x = fixed_inputs(wl.B, wl.N, wl.H, wl.d, seed=wl.seed, with_dout=True)
    o, lse, dq, dk, dv = run(x, wl.causal, 0)
    N = wl.N
    rng = np.random.default_rng(wl.seed + 100)
    qrows = []
    for s in range(wl.B):
        for h in range(wl.H):
            picks = {0, 1, 127, 128, 129, N // 2, N - 2, N - 1}
            picks |= {int(i) for i in rng.integers(0, N, 2)}
            qrows += [(s, h, i) for i in sorted(picks)]
    krows = []
    if wl.causal:
        for s, h in ((0, 0), (2, 7), (3, 12), (wl.B - 1, wl.H - 1)):
            picks = {N - 1, N - 2, N - 128, N - 129, N - 256}
            picks |= {int(j) for j in rng.integers(N - 256, N, 3)}
            krows += [(s, h, j) for j in sorted(picks)]
    qrows = np.array(qrows, dtype=np.int32)
    krows = np.array(krows, dtype=np.int32).reshape(-1, 3)
    dq_r, dk_r, dv_r = orc.bwd_rows(x["q"], x["k"], x["v"], x["dout"], wl.scale, qrows, krows,
                                    causal=wl.causal)
    g = {n: to64(t) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    assert_close_bf16(np.stack([g["dq"][s, i, h] for s, h, i in qrows]), dq_r, "dq rows")
    if len(krows):
        assert_close_bf16(np.stack([g["dk"][s, j, h] for s, h, j in krows]), dk_r, "dk rows")
        assert_close_bf16(np.stack([g["dv"][s, j, h] for s, h, j in krows]), dv_r, "dv rows")
