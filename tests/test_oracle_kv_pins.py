"""Pins for the oracle's cached-key/value forward (queries = the last Nq
positions of an Nk-long key sequence; causal masks bottom-right aligned)."""
import math

import numpy as np
import pytest

from oracle import oracle as orc


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _brute_kv(q, k, v, scale, causal, window):
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    off = Nk - Nq
    i = np.arange(Nq)[:, None] + off
    j = np.arange(Nk)[None, :]
    allowed = np.ones((Nq, Nk), bool)
    if causal:
        allowed &= j <= i
    if window > 0:
        allowed &= j > i - window
    O = np.zeros_like(q)
    L = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        for h in range(H):
            S = scale * q[b, :, h] @ k[b, :, h].T
            S = np.where(allowed, S, -np.inf)
            rows = allowed.any(1)
            m = np.where(rows, S.max(1), 0.0)[:, None]
            E = np.where(allowed, np.exp(S - m), 0.0)
            den = E.sum(1, keepdims=True)
            O[b, rows, h] = (E[rows] / den[rows]) @ v[b, :, h]
            L[b, h, rows] = m[rows, 0] + np.log(den[rows, 0])
    return O, L


def test_hand_worked_single_query_sees_the_whole_prefix():
    # keys [0, ln2], values [3, 6]; one query q = 1 at the last position: under
    # the causal mask it sees both keys, P = [1/3, 2/3], O = 5, LSE = ln 3
    q = np.array([1.0]).reshape(1, 1, 1, 1)
    k = np.array([0.0, math.log(2)]).reshape(1, 2, 1, 1)
    v = np.array([3.0, 6.0]).reshape(1, 2, 1, 1)
    O, L = orc.fwd_kv(q, k, v, 1.0, causal=True)
    assert abs(O.ravel()[0] - 5.0) < 1e-14
    assert abs(L.ravel()[0] - math.log(3)) < 1e-14


@pytest.mark.parametrize("Nq,Nk", [(1, 7), (3, 8), (8, 8), (5, 16)])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 1), (True, 3)])
def test_brute_force_bottom_right(Nq, Nk, causal, window):
    q = _rand((2, Nq, 2, 8), 1)
    k = _rand((2, Nk, 2, 8), 2)
    v = _rand((2, Nk, 2, 8), 3)
    O, L = orc.fwd_kv(q, k, v, 0.4, causal=causal, window=window)
    Ob, Lb = _brute_kv(q, k, v, 0.4, causal, window)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 5)])
def test_equal_lengths_reduce_to_self_attention(causal, window):
    q, k, v = (_rand((2, 19, 3, 8), s) for s in (4, 5, 6))
    O, L = orc.fwd_kv(q, k, v, 0.3, causal=causal, window=window)
    O2, L2 = orc.fwd(q, k, v, 0.3, causal=causal, window=window)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)


@pytest.mark.parametrize("window", [0, 4])
def test_suffix_of_full_causal_attention(window):
    """The last Nq queries against all Nk keys equal the last Nq rows of the
    full self-attention over the Nk-long sequence."""
    Nk, Nq = 23, 6
    qf, k, v = (_rand((2, Nk, 2, 8), s) for s in (7, 8, 9))
    Of, Lf = orc.fwd(qf, k, v, 0.5, causal=True, window=window)
    O, L = orc.fwd_kv(qf[:, -Nq:], k, v, 0.5, causal=True, window=window)
    np.testing.assert_array_equal(O, Of[:, -Nq:])
    np.testing.assert_array_equal(L, Lf[:, :, -Nq:])


def test_packed_equals_separate_and_empty_rows():
    H, d = 2, 8
    nq = [3, 1, 4, 2]
    nk = [7, 1, 4, 1]           # last sequence: 2 queries, 1 key -> first query sees nothing
    cq = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(nk)]).astype(np.int32)
    q = _rand((cq[-1], H, d), 10)
    k = _rand((ck[-1], H, d), 11)
    v = _rand((ck[-1], H, d), 12)
    O, L = orc.fwd_kv(q, k, v, 0.5, causal=True, cu_seqlens_q=cq, cu_seqlens_k=ck)
    for s in range(len(nq)):
        Os, Ls = orc.fwd_kv(q[None, cq[s]:cq[s + 1]], k[None, ck[s]:ck[s + 1]],
                            v[None, ck[s]:ck[s + 1]], 0.5, causal=True)
        np.testing.assert_array_equal(O[cq[s]:cq[s + 1]], Os[0])
        np.testing.assert_array_equal(L[:, cq[s]:cq[s + 1]], Ls[0])
    # query 0 of the last sequence sits at position -1: no key, O = 0, LSE = -inf
    assert (O[cq[3]] == 0).all() and np.isneginf(L[:, cq[3]]).all()
    np.testing.assert_allclose(O[cq[3] + 1], v[ck[3]], atol=1e-14)


# ------------------------------------------------ padded cache (decode) ---

@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 2)])
def test_kvcache_uses_only_the_first_seqlens_rows(causal, window):
    # Each sequence's result equals the fixed-length cached-KV forward of the
    # rows it uses; the unused rows (filled with NaN here) are never read.
    B, Nq, Nk, H, d = 3, 2, 9, 2, 4
    q = _rand((B, Nq, H, d), 11)
    k = _rand((B, Nk, H, d), 12)
    v = _rand((B, Nk, H, d), 13)
    lens = np.array([9, 4, 1], dtype=np.int32)
    for b in range(B):
        k[b, lens[b]:] = np.nan
        v[b, lens[b]:] = np.nan
    O, L = orc.fwd_kvcache(q, k, v, 0.5, seqlens_k=lens, causal=causal, window=window)
    for b in range(B):
        n = lens[b]
        Ob, Lb = _brute_kv(q[b:b + 1], k[b:b + 1, :n], v[b:b + 1, :n], 0.5, causal, window)
        np.testing.assert_allclose(O[b:b + 1], Ob, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(L[b:b + 1]), np.isneginf(Lb))
        fin = ~np.isneginf(Lb)
        np.testing.assert_allclose(L[b:b + 1][fin], Lb[fin], rtol=0, atol=1e-12)


def test_kvcache_without_seqlens_is_fwd_kv():
    q = _rand((2, 3, 2, 8), 21)
    k = _rand((2, 40, 2, 8), 22)
    v = _rand((2, 40, 2, 8), 23)
    O1, L1 = orc.fwd_kvcache(q, k, v, 0.3, causal=True)
    O2, L2 = orc.fwd_kv(q, k, v, 0.3, causal=True)
    assert np.array_equal(O1, O2) and np.array_equal(L1, L2)


def test_kvcache_empty_cache_rows():
    # nk = 0: no key at all; nk < Nq under causal: the first queries see none
    q = _rand((2, 3, 1, 4), 31)
    k = _rand((2, 5, 1, 4), 32)
    v = _rand((2, 5, 1, 4), 33)
    O, L = orc.fwd_kvcache(q, k, v, 1.0, seqlens_k=np.array([0, 2], np.int32), causal=True)
    assert np.all(O[0] == 0) and np.all(np.isneginf(L[0]))
    # sequence 1: positions -1, 0, 1 -> query 0 sees nothing, query 1 sees key 0
    assert np.all(O[1, 0] == 0) and np.isneginf(L[1, 0, 0])
    np.testing.assert_allclose(O[1, 1, 0], v[1, 0, 0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(L[1, 0, 1], 1.0 * q[1, 1, 0] @ k[1, 0, 0], rtol=0, atol=1e-14)
