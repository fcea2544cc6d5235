"""fa_bwd_noalloc serves callers that cannot allocate device memory -- a plugin
inside a framework that owns every device allocation and offers no workspace,
or a serving loop that must not allocate once it runs.  It takes no workspace
argument and keeps its scratch (the D = rowsum(dO * O) values) in a fixed array
inside the library.  Its gradients must equal those of fa_bwd, which gets a
caller-provided workspace, on consecutive calls that reuse that array."""
import math

import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import fixed_inputs, varlen_inputs
from oracle import oracle as orc

from helpers import assert_close_bf16, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"

# Two different problems back to back: a value left in the shared scratch by
# the first call must not leak into the second.
CASES = [
    dict(B=2, N=700, H=3, d=128, causal=True, window=0, seed=41),
    dict(B=1, N=300, H=2, d=64, causal=True, window=37, seed=42),
]


def _problem(c):
    x = fixed_inputs(c["B"], c["N"], c["H"], c["d"], seed=c["seed"], with_dout=True)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v, causal=c["causal"], window=c["window"])
    return q, k, v, do, o, lse


def test_noalloc_backward_matches_fa_bwd_on_two_calls_in_a_row():
    probs = [_problem(c) for c in CASES]
    refs = []
    for c, (q, k, v, do, o, lse) in zip(CASES, probs):
        refs.append(fa.backward(q, k, v, o, lse, do, causal=c["causal"], window=c["window"]))
    torch.cuda.synchronize()
    for c, (q, k, v, do, o, lse), ref in zip(CASES, probs, refs):
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        rc = fa.fa_bwd_noalloc(q, k, v, o, lse, do, *grads, c["B"], c["H"], c["N"], c["d"],
                               1 / math.sqrt(c["d"]), int(c["causal"]), c["window"], None, None)
        assert rc == 0, fa.fa_status_string(rc)
        torch.cuda.synchronize()
        assert fa.fa_get_device_error() == 0
        for name, got, want in zip(("dq", "dk", "dv"), grads, ref):
            assert_close_bf16(got, to64(want), name)


def test_noalloc_packed_batch_after_a_larger_call():
    """A packed batch (its statistics sit at per-sequence offsets rounded up to
    128 rows in the scratch) right after a larger fixed-length call that left
    other values there; checked against fa_bwd and the float64 oracle."""
    big = dict(B=2, N=1500, H=4, d=128, causal=False, window=0, seed=43)
    q, k, v, do, o, lse = _problem(big)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    rc = fa.fa_bwd_noalloc(q, k, v, o, lse, do, *grads, big["B"], big["H"], big["N"], big["d"],
                           1 / math.sqrt(big["d"]), 0, 0, None, None)
    assert rc == 0, fa.fa_status_string(rc)
    lens = [130, 1, 517]
    H, d, window = 3, 128, 200
    x = varlen_inputs(len(lens), 0, 0, H, d, seed=44, with_dout=True, lengths=lens)
    cu = x["cu_seqlens"].to(DEV)
    q, k, v, do = (x[n].to(DEV) for n in ("q", "k", "v", "dout"))
    o, lse = fa.forward(q, k, v, causal=True, window=window, cu_seqlens=cu)
    want = fa.backward(q, k, v, o, lse, do, causal=True, window=window, cu_seqlens=cu)
    T = sum(lens)
    ref = orc.bwd(x["q"], x["k"], x["v"], x["dout"], 1 / math.sqrt(d), causal=True,
                  window=window, cu_seqlens=x["cu_seqlens"])
    for _ in range(2):
        got = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
        rc = fa.fa_bwd_noalloc(q, k, v, o, lse, do, *got, len(lens), H, T, d, 1 / math.sqrt(d), 1,
                               window, cu, None)
        assert rc == 0, fa.fa_status_string(rc)
        torch.cuda.synchronize()
        assert fa.fa_get_device_error() == 0
        for name, g, w in zip(("dq", "dk", "dv"), got, want):
            assert_close_bf16(g, to64(w), name + " vs fa_bwd")
            assert_close_bf16(g, ref[name], name + " vs oracle")


def test_noalloc_rejects_problems_beyond_its_scratch():
    # H * rows above the built-in maximum: rejected on the host, nothing launched
    H, d = 16, 128
    N = fa.binding.NOALLOC_MAX_ROWS // H + 1
    p = 0x10000
    rc = fa.fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, H, N, d, 0.1, 0, 0, None, None)
    assert rc == -10
