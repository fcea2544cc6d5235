"""Seeded random shapes and masks, forward and backward against the float64
oracle: fixed-length and packed batches (empty sequences included), d in
{64, 128}, causal masks with windows from 1 to 300 keys, and softmax scales
other than 1/sqrt(d).  The forward is held to the usual tolerances; the
backward to the element-wise bounds derived from its bf16 roundings
(test_scale_gpu.backward_bounds), since short windows give gradients of
several units where bf16's own spacing exceeds the fixed absolute bound."""
import math
import random

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import fixed_inputs, varlen_inputs
from oracle import oracle as orc

from helpers import TOL_LSE, TOL_MAX, TOL_MEAN, to64
from test_scale_gpu import backward_bounds

pytestmark = pytest.mark.gpu

DEV = "cuda"
CASES = 48


def draw(case):
    """The configuration of one case, from its own seeded stream."""
    rng = random.Random(9000 + case)
    d = rng.choice([64, 128])
    H = rng.choice([1, 2, 3])
    causal = rng.random() < 0.7
    window = rng.choice([0, 0, 1, 2, 17, 64, 127, 128, 129, 255, 300]) if causal else 0
    scale = rng.choice([1 / math.sqrt(d), 0.05, 0.1])
    if rng.random() < 0.4:
        lens = [rng.choice([0, 1, 2, 63, 64, 65, 127, 128, 129, 200, 255, 256, 257, 384, 511])
                for _ in range(rng.randint(1, 5))]
        if sum(lens) == 0:
            lens[0] = 5
        return dict(d=d, H=H, causal=causal, window=window, scale=scale, lens=lens)
    return dict(d=d, H=H, causal=causal, window=window, scale=scale, B=rng.randint(1, 3),
                N=rng.choice([1, 3, 64, 127, 128, 129, 200, 256, 257, 383, 512, 600]))


def slices(x, c):
    """The case's (sequence) problems as fixed-length [1, n, H, d] inputs."""
    if "lens" not in c:
        yield None, x
        return
    cu = x["cu_seqlens"]
    for s in range(len(c["lens"])):
        a, b = int(cu[s]), int(cu[s + 1])
        if b > a:
            yield (a, b), {n: x[n][a:b].unsqueeze(0) for n in ("q", "k", "v", "dout")}


@pytest.mark.parametrize("case", range(CASES))
def test_random_forward_backward(case):
    c = draw(case)
    if "lens" in c:
        x = varlen_inputs(len(c["lens"]), 0, 0, c["H"], c["d"], seed=case, with_dout=True,
                          lengths=c["lens"])
        cu = x["cu_seqlens"]
    else:
        x = fixed_inputs(c["B"], c["N"], c["H"], c["d"], seed=case, with_dout=True)
        cu = None
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    cu_d = None if cu is None else cu.to(DEV)
    kw = dict(causal=c["causal"], window=c["window"], cu_seqlens=cu_d, scale=c["scale"])
    o, lse = fa.forward(q, k, v, **kw)
    dq, dk, dv = fa.backward(q, k, v, o, lse, do, **kw)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    # forward: the usual tolerances
    O, L = orc.fwd(x["q"], x["k"], x["v"], c["scale"], causal=c["causal"], window=c["window"],
                   cu_seqlens=cu)
    err = np.abs(to64(o) - O)
    assert err.max() <= TOL_MAX and err.mean() <= TOL_MEAN, (c, err.max(), err.mean())
    lg = to64(lse)
    assert np.array_equal(np.isneginf(lg), np.isneginf(L)), c
    fin = np.isfinite(L)
    if fin.any():
        assert np.abs(lg[fin] - L[fin]).max() <= TOL_LSE, c
    # backward: derived element-wise bounds, sequence by sequence
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], c["scale"], causal=c["causal"],
                  window=c["window"], cu_seqlens=cu)
    for rows, xs in slices(x, c):
        if rows is None:
            o_s, got = o, {"dq": dq, "dk": dk, "dv": dv}
            want = ref
        else:
            a, b = rows
            o_s = o[a:b].unsqueeze(0)
            got = {n: t[a:b].unsqueeze(0) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
            want = {n: ref[n][a:b][None] for n in ("dq", "dk", "dv")}
        bound = backward_bounds(xs, o_s, c["scale"], c["causal"], c["window"])
        for n in ("dq", "dk", "dv"):
            e = np.abs(to64(got[n]) - want[n])
            tol = 2.0 * (bound[n] + 2.0 ** -9 * np.abs(want[n])) + 1e-3
            assert (e <= tol).all(), (c, rows, n, float((e / tol).max()))
