"""Cached-KV prefill on the GPU: fa_fwd_kv (queries that are the last
positions of a longer key/value sequence; causal and window masks aligned
bottom-right) through the C ABI against the float64 oracle's fwd_kv, plus
the identities that tie it to self-attention."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import WORKLOADS, fixed_inputs, kv_inputs, varlen_kv_inputs
from oracle import oracle as orc

from helpers import TOL_LSE, assert_close_bf16, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run_kv(x, causal, window):
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    cq = x.get("cu_seqlens_q")
    ck = x.get("cu_seqlens_k")
    o, lse = fa.forward_kv(q, k, v, causal=causal, window=window,
                           cu_seqlens_q=None if cq is None else cq.to(DEV),
                           cu_seqlens_k=None if ck is None else ck.to(DEV))
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return o, lse


def oracle_kv(x, causal, window, scale):
    return orc.fwd_kv(x["q"], x["k"], x["v"], scale, causal=causal, window=window,
                      cu_seqlens_q=x.get("cu_seqlens_q"), cu_seqlens_k=x.get("cu_seqlens_k"))


def assert_lse_with_empty_rows(got, ref):
    """LSE within tolerance; rows without any allowed key must be -inf on
    both sides."""
    g = to64(got)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), empty), "rows without keys differ"
    if (~empty).any():
        err = np.abs(g[~empty] - ref[~empty]).max()
        assert err <= TOL_LSE, "lse: max %.3e" % err


FIXED = [(1, 1, 1, 1, 64), (2, 17, 300, 2, 128), (1, 128, 1024, 2, 64), (2, 200, 700, 3, 128),
         (1, 300, 100, 2, 128), (2, 257, 257, 2, 128), (1, 1, 4000, 2, 128),
         (1, 513, 1000, 1, 64)]
MASKS = [(False, 0), (True, 0), (True, 1), (True, 64), (True, 300)]


@pytest.mark.parametrize("B,Nq,Nk,H,d", FIXED)
@pytest.mark.parametrize("causal,window", MASKS)
def test_fwd_kv_fixed_elementwise(B, Nq, Nk, H, d, causal, window):
    x = kv_inputs(B, Nq, Nk, H, d, seed=Nq * 7 + Nk)
    o, lse = run_kv(x, causal, window)
    O, L = oracle_kv(x, causal, window, 1 / math.sqrt(d))
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


def test_fwd_kv_without_keys():
    # Nk = 0: every query sees no key
    x = kv_inputs(2, 130, 0, 2, 128, seed=3)
    for causal in (False, True):
        o, lse = run_kv(x, causal, 0)
        assert torch.count_nonzero(o) == 0
        assert torch.isneginf(lse).all()


PACKED = [[(100, 500), (0, 300), (257, 257), (64, 0), (300, 100), (1, 1000), (129, 130)],
          [(2048, 2048)],
          [(5, 9), (128, 128), (127, 1130), (0, 0), (700, 701)]]


@pytest.mark.parametrize("pairs", PACKED)
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 64), (True, 1)])
def test_fwd_kv_packed_elementwise(pairs, causal, window):
    x = varlen_kv_inputs([a for a, _ in pairs], [b for _, b in pairs], 3, 128, seed=11)
    o, lse = run_kv(x, causal, window)
    O, L = oracle_kv(x, causal, window, 1 / math.sqrt(128))
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 50)])
def test_fwd_kv_packed_many_sequences_long_caches(causal, window):
    # 300 sequences (more than are ranked by length), keys at least twice the
    # queries in total, so the single-block walk runs in index order
    rng = np.random.default_rng(17)
    nq = [int(x) for x in rng.integers(0, 40, 300)]
    nk = [int(x) + 2 * q for x, q in zip(rng.integers(0, 300, 300), nq)]
    x = varlen_kv_inputs(nq, nk, 1, 64, seed=18)
    o, lse = run_kv(x, causal, window)
    O, L = oracle_kv(x, causal, window, 1 / math.sqrt(64))
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


@pytest.mark.parametrize("Nq", [1, 200, 1000])
@pytest.mark.parametrize("window", [0, 100])
def test_fwd_kv_is_suffix_of_self_attention(Nq, window):
    # The last Nq rows of causal self-attention over Nk tokens are the
    # Nq-query prefill against those Nk keys.  Below Nk = 2 Nq the prefill runs
    # the self-attention kernel: same keys, same tiles, same order of the
    # online softmax, so the results agree bit for bit.  From Nk = 2 Nq on it
    # runs the padded-cache kernel, whose last key tile is read right-aligned
    # (keys Nk - 128 .. Nk - 1, the overlap masked), so the sums group
    # differently: equal to fa_fwd_kvcache without lengths bit for bit (more
    # than 16 queries), and to the self-attention rows within the bf16 tolerance.
    Nk = 1000
    x = fixed_inputs(2, Nk, 2, 128, seed=21)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o_full, lse_full = fa.forward(q, k, v, causal=True, window=window)
    qs = q[:, Nk - Nq:].contiguous()
    o, lse = fa.forward_kv(qs, k, v, causal=True, window=window)
    torch.cuda.synchronize()
    if Nk < 2 * Nq:
        assert torch.equal(o, o_full[:, Nk - Nq:])
        assert torch.equal(lse, lse_full[:, :, Nk - Nq:])
    else:
        if Nq > 16:      # (up to 16 queries the cache call runs the decode kernel)
            oc, lc = fa.forward_kvcache(qs, k, v, causal=True, window=window, num_splits=1)
            torch.cuda.synchronize()
            assert torch.equal(o, oc) and torch.equal(lse, lc)
        assert_close_bf16(o, to64(o_full[:, Nk - Nq:]), "O")
        assert np.abs(to64(lse) - to64(lse_full[:, :, Nk - Nq:])).max() <= TOL_LSE


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 33)])
def test_fwd_kv_equal_lengths_is_fwd(causal, window):
    x = fixed_inputs(2, 777, 2, 128, seed=5)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o1, l1 = fa.forward(q, k, v, causal=causal, window=window)
    o2, l2 = fa.forward_kv(q, k, v, causal=causal, window=window)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_kv_workload_parity():
    # 2048 new tokens after 6144 cached ones, B4 H16 d128, causal; three
    # whole (sequence, head) slices are checked against the oracle.
    wl = WORKLOADS["prefill_kv_causal"]
    x = wl.make()
    o, lse = run_kv(x, wl.causal, wl.window)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    for s, h in ((0, 0), (1, 7), (3, 15)):
        sl = {n: x[n][s:s + 1, :, h:h + 1] for n in ("q", "k", "v")}
        O, L = oracle_kv(sl, wl.causal, wl.window, wl.scale)
        assert_close_bf16(o[s:s + 1, :, h:h + 1], O, "O seq %d head %d" % (s, h))
        assert_lse_with_empty_rows(lse[s:s + 1, h:h + 1], L)
