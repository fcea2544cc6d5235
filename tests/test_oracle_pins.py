"""Pins for the float64 CPU oracle: checks against facts that do not come from
the oracle itself (hand-derived values, brute force with an explicit softmax
matrix, a library softmax with autograd, closed forms, invariants, the online
update of the pages, and finite differences).  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _num(x):
    """Parse the small symbolic numbers used in the golden file."""
    if isinstance(x, (int, float)):
        return float(x)
    table = {"ln2": math.log(2), "ln3": math.log(3), "ln5": math.log(5), "2ln2": 2 * math.log(2),
             "2/3*ln2": 2 / 3 * math.log(2), "-2/3": -2 / 3, "2/3": 2 / 3, "1/3": 1 / 3}
    return table[x]


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _brute(q, k, v, scale, causal=False, window=0):
    """Explicit N x N softmax matrix per head (numpy float64)."""
    B, N, H, d = q.shape
    O = np.zeros_like(q)
    L = np.zeros((B, H, N))
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    allowed = np.ones((N, N), bool)
    if causal:
        allowed &= j <= i
    if window > 0:
        allowed &= j > i - window
    for b in range(B):
        for h in range(H):
            S = scale * q[b, :, h, :] @ k[b, :, h, :].T
            S = np.where(allowed, S, -np.inf)
            m = S.max(1, keepdims=True)
            E = np.exp(S - m)
            P = E / E.sum(1, keepdims=True)
            O[b, :, h, :] = P @ v[b, :, h, :]
            L[b, h] = (m[:, 0] + np.log(E.sum(1)))
    return O, L


# ---------------------------------------------------------------- golden ---

def test_golden_hand_worked_forward():
    g = json.load(open(GOLDEN))
    q = np.array([_num(x) for x in g["inputs"]["q"]]).reshape(1, 2, 1, 1)
    k = np.array([_num(x) for x in g["inputs"]["k"]]).reshape(1, 2, 1, 1)
    v = np.array([_num(x) for x in g["inputs"]["v"]]).reshape(1, 2, 1, 1)
    for case, causal, window in (("noncausal", False, 0), ("causal", True, 0),
                                 ("window1", True, 1)):
        O, L = orc.fwd(q, k, v, 1.0, causal=causal, window=window)
        np.testing.assert_allclose(O.ravel(), [_num(x) for x in g[case]["o"]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(L.ravel(), [_num(x) for x in g[case]["lse"]], rtol=0,
                                   atol=1e-14)
    # the online update with one key per block reaches the same row-0 output
    O1, _ = orc.fwd_online(q, k, v, 1.0, block=1)
    assert abs(O1[0, 0, 0, 0] - g["online_row0_block1"]["o"]) < 1e-14
    # after the first block alone (a one-key sequence) the output is u/l = 3/1
    O0, L0 = orc.fwd_online(q[:, :1], k[:, :1], v[:, :1], 1.0, block=1)
    st = g["online_row0_block1"]["steps"][0]
    assert abs(O0.ravel()[0] - st["u"] / st["l"]) < 1e-14
    assert abs(L0.ravel()[0] - (st["m"] + math.log(st["l"]))) < 1e-14


def test_golden_hand_worked_backward():
    g = json.load(open(GOLDEN))
    arr = lambda key: np.array([_num(x) for x in g["inputs"][key]]).reshape(1, 2, 1, 1)
    r = orc.bwd(arr("q"), arr("k"), arr("v"), arr("dout"), 1.0)
    exp = g["noncausal_grad"]
    for name in ("dq", "dk", "dv"):
        np.testing.assert_allclose(r[name].ravel(), [_num(x) for x in exp[name]], rtol=0,
                                   atol=1e-14)
    np.testing.assert_allclose(r["D"].ravel(), exp["D"], rtol=0, atol=1e-14)


# ------------------------------------------------------------ brute force ---

@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 1), (True, 2), (True, 3),
                                           (True, 8)])
@pytest.mark.parametrize("N,d", [(1, 4), (5, 3), (8, 16)])
def test_brute_force_small(N, d, causal, window):
    q, k, v = (_rand((2, N, 3, d), s) for s in (1, 2, 3))
    scale = 0.37
    O, L = orc.fwd(q, k, v, scale, causal=causal, window=window)
    Ob, Lb = _brute(q, k, v, scale, causal, window)
    np.testing.assert_allclose(O, Ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 3)])
def test_library_softmax_and_autograd(causal, window):
    """torch float64 softmax + autograd as an independent library routine."""
    B, N, H, d = 2, 13, 2, 8
    q, k, v, do = (torch.from_numpy(_rand((B, N, H, d), s)) for s in (4, 5, 6, 7))
    scale = 1 / math.sqrt(d)
    qt, kt, vt = (x.clone().requires_grad_(True) for x in (q, k, v))
    S = torch.einsum("bihc,bjhc->bhij", qt, kt) * scale
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    allowed = torch.ones(N, N, dtype=torch.bool)
    if causal:
        allowed &= j <= i
    if window > 0:
        allowed &= j > i - window
    S = S.masked_fill(~allowed, float("-inf"))
    P = torch.softmax(S, dim=-1)
    O = torch.einsum("bhij,bjhc->bihc", P, vt)
    lse = torch.logsumexp(S, dim=-1)
    (O * do).sum().backward()
    r = orc.bwd(q, k, v, do, scale, causal=causal, window=window)
    np.testing.assert_allclose(r["o"], O.detach().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], lse.detach().numpy(), rtol=0, atol=1e-12)
    for name, t in (("dq", qt), ("dk", kt), ("dv", vt)):
        np.testing.assert_allclose(r[name], t.grad.numpy(), rtol=0, atol=1e-12)


# ------------------------------------------------------------ closed forms ---

def test_zero_keys_give_column_mean():
    B, N, H, d = 1, 37, 2, 8
    q, v = _rand((B, N, H, d), 8), _rand((B, N, H, d), 9)
    k = np.zeros_like(q)
    O, L = orc.fwd(q, k, v, 0.3)
    np.testing.assert_allclose(O, np.broadcast_to(v.mean(1, keepdims=True), O.shape), atol=1e-13)
    np.testing.assert_allclose(L, math.log(N), atol=1e-13)
    # causal: running mean of v_0..v_i and LSE = ln(i+1)
    Oc, Lc = orc.fwd(q, k, v, 0.3, causal=True)
    run = np.cumsum(v, axis=1) / np.arange(1, N + 1)[None, :, None, None]
    np.testing.assert_allclose(Oc, run, atol=1e-13)
    np.testing.assert_allclose(Lc, np.broadcast_to(np.log(np.arange(1, N + 1)), Lc.shape),
                               atol=1e-13)


def test_causal_row0_and_window1():
    B, N, H, d = 2, 19, 3, 16
    q, k, v = (_rand((B, N, H, d), s) for s in (10, 11, 12))
    scale = 0.25
    O, L = orc.fwd(q, k, v, scale, causal=True)
    np.testing.assert_allclose(O[:, 0], v[:, 0], atol=1e-14)
    np.testing.assert_allclose(L[:, :, 0], scale * np.einsum("bhc,bhc->bh", q[:, 0], k[:, 0]),
                               atol=1e-13)
    O1, L1 = orc.fwd(q, k, v, scale, causal=True, window=1)
    np.testing.assert_allclose(O1, v, atol=1e-14)
    np.testing.assert_allclose(L1, scale * np.einsum("bnhc,bnhc->bhn", q, k), atol=1e-13)


def test_one_hot_dominant_score_selects_row():
    N, d = 16, 16
    k = np.eye(N, d)[None, :, None, :]          # orthonormal keys
    v = _rand((1, N, 1, d), 13)
    perm = np.random.default_rng(14).permutation(N)
    q = 60.0 * k[:, perm]                       # row i is a large multiple of key perm[i]
    O, _ = orc.fwd(q, k, v, 1.0)
    np.testing.assert_allclose(O[0, :, 0], v[0, perm, 0], atol=1e-20 + 1e-12)


def test_window_at_least_n_equals_causal():
    q, k, v = (_rand((1, 23, 2, 8), s) for s in (15, 16, 17))
    Oc, Lc = orc.fwd(q, k, v, 0.5, causal=True)
    Ow, Lw = orc.fwd(q, k, v, 0.5, causal=True, window=23)
    np.testing.assert_array_equal(Oc, Ow)
    np.testing.assert_array_equal(Lc, Lw)


# --------------------------------------------------------------- invariants ---

def test_key_shift_invariance():
    B, N, H, d = 1, 21, 2, 8
    q, k, v = (_rand((B, N, H, d), s) for s in (18, 19, 20))
    c = _rand((d,), 21)
    scale = 0.4
    O, L = orc.fwd(q, k, v, scale)
    O2, L2 = orc.fwd(q, k + c, v, scale)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, L + scale * np.einsum("bnhc,c->bhn", q, c), atol=1e-12)


def test_joint_permutation_of_keys_and_values():
    B, N, H, d = 1, 29, 2, 8
    q, k, v = (_rand((B, N, H, d), s) for s in (22, 23, 24))
    p = np.random.default_rng(25).permutation(N)
    O, L = orc.fwd(q, k, v, 0.4)
    O2, L2 = orc.fwd(q, k[:, p], v[:, p], 0.4)
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, L, atol=1e-12)


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 5)])
def test_gradient_invariants(causal, window):
    B, N, H, d = 2, 17, 2, 8
    q, k, v, do = (_rand((B, N, H, d), s) for s in (26, 27, 28, 29))
    r = orc.bwd(q, k, v, do, 0.35, causal=causal, window=window)
    # sum_j dS_ij = 0 for every row, so the key gradients sum to zero
    np.testing.assert_allclose(r["dk"].sum(1), 0.0, atol=1e-12)
    # each row of P sums to one, so the value gradients sum to the sum of dO
    np.testing.assert_allclose(r["dv"].sum(1), do.sum(1), atol=1e-12)
    np.testing.assert_allclose(r["D"], np.einsum("bnhc,bnhc->bhn", do, r["o"]), atol=1e-12)


# ---------------------------------------------------- online vs three-pass ---

@pytest.mark.parametrize("block", [1, 3, 16, 40])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 7)])
def test_online_update_matches_three_pass(block, causal, window):
    B, N, H, d = 2, 40, 2, 16
    q, k, v = (_rand((B, N, H, d), s) for s in (30, 31, 32))
    q *= 3.0  # spread the scores so the running maximum moves
    O, L = orc.fwd(q, k, v, 0.5, causal=causal, window=window)
    O2, L2 = orc.fwd_online(q, k, v, 0.5, block=block, causal=causal, window=window)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L2, L, rtol=0, atol=1e-12)


# ------------------------------------------------------ finite differences ---

@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 4)])
def test_finite_difference_gradients(causal, window):
    B, N, H, d = 1, 9, 2, 5
    x = {n: _rand((B, N, H, d), s) for n, s in zip(("q", "k", "v", "dout"), (33, 34, 35, 36))}
    scale = 0.6
    r = orc.bwd(x["q"], x["k"], x["v"], x["dout"], scale, causal=causal, window=window)

    def f(qq, kk, vv):
        O, _ = orc.fwd(qq, kk, vv, scale, causal=causal, window=window)
        return float((O * x["dout"]).sum())

    rng = np.random.default_rng(37)
    h = 1e-5
    for name, grad in (("q", r["dq"]), ("k", r["dk"]), ("v", r["dv"])):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in (B, N, H, d))
            args = {n: x[n].copy() for n in ("q", "k", "v")}
            args[name][idx] += h
            fp = f(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * h
            fm = f(args["q"], args["k"], args["v"])
            fd = (fp - fm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx, fd,
                                                                            grad[idx])


# ----------------------------------------------------------- packing / API ---

def test_varlen_packing_equals_separate_sequences():
    lens = [1, 7, 16, 3]
    H, d = 2, 8
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v, do = (_rand((T, H, d), s) for s in (38, 39, 40, 41))
    for causal, window in ((False, 0), (True, 0), (True, 3)):
        O, L = orc.fwd(q, k, v, 0.5, causal=causal, window=window, cu_seqlens=cu)
        r = orc.bwd(q, k, v, do, 0.5, causal=causal, window=window, cu_seqlens=cu)
        for s, n in enumerate(lens):
            a, b = cu[s], cu[s + 1]
            Os, Ls = orc.fwd(q[None, a:b], k[None, a:b], v[None, a:b], 0.5, causal=causal,
                             window=window)
            np.testing.assert_array_equal(O[a:b], Os[0])
            np.testing.assert_array_equal(L[:, a:b], Ls[0])
            rs = orc.bwd(q[None, a:b], k[None, a:b], v[None, a:b], do[None, a:b], 0.5,
                         causal=causal, window=window)
            for name in ("dq", "dk", "dv"):
                np.testing.assert_array_equal(r[name][a:b], rs[name][0])


def test_rows_and_head_subsets_match_full():
    B, N, H, d = 2, 33, 3, 8
    q, k, v, do = (_rand((B, N, H, d), s) for s in (42, 43, 44, 45))
    O, L = orc.fwd(q, k, v, 0.5, causal=True)
    rows = np.array([[0, 0, 0], [1, 2, 32], [0, 1, 17], [1, 0, 5]])
    Or, Lr = orc.fwd_rows(q, k, v, rows, 0.5, causal=True)
    for r, (s, h, i) in enumerate(rows):
        np.testing.assert_array_equal(Or[r], O[s, i, h])
        assert Lr[r] == L[s, h, i]
    full = orc.bwd(q, k, v, do, 0.5, causal=True)
    part = orc.bwd(q, k, v, do, 0.5, causal=True, heads=[(1, 2), (0, 0)])
    for (s, h) in ((1, 2), (0, 0)):
        for name in ("dq", "dk", "dv", "o"):
            np.testing.assert_array_equal(part[name][s, :, h], full[name][s, :, h])
    assert np.isnan(part["dq"][0, :, 1]).all()


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 3), (True, 20)])
def test_backward_rows_match_full_and_autograd(causal, window):
    """bwd_rows (gradients of listed rows from the rows' own statistics) gives
    bit for bit the rows of the full bwd, and matches torch float64 autograd
    directly; key lists that start late in the sequence (where only later
    queries are computed) included."""
    B, N, H, d = 2, 41, 2, 8
    q, k, v, do = (_rand((B, N, H, d), s) for s in (61, 62, 63, 64))
    scale = 0.3
    qrows = np.array([[0, 0, 0], [1, 1, 40], [0, 1, 17], [1, 0, 5], [1, 0, 6]])
    krows = np.array([[0, 0, 0], [1, 1, 40], [1, 1, 30], [0, 1, 17], [1, 0, 39], [0, 0, 25]])
    dq, dk, dv = orc.bwd_rows(q, k, v, do, scale, qrows, krows, causal=causal, window=window)
    full = orc.bwd(q, k, v, do, scale, causal=causal, window=window)
    for r, (s_, h, i) in enumerate(qrows):
        np.testing.assert_array_equal(dq[r], full["dq"][s_, i, h])
    for r, (s_, h, j) in enumerate(krows):
        np.testing.assert_array_equal(dk[r], full["dk"][s_, j, h])
        np.testing.assert_array_equal(dv[r], full["dv"][s_, j, h])
    qt, kt, vt = (torch.from_numpy(x).clone().requires_grad_(True) for x in (q, k, v))
    S = torch.einsum("bihc,bjhc->bhij", qt, kt) * scale
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    allowed = torch.ones(N, N, dtype=torch.bool)
    if causal:
        allowed &= j <= i
    if window > 0:
        allowed &= j > i - window
    P = torch.softmax(S.masked_fill(~allowed, float("-inf")), dim=-1)
    (torch.einsum("bhij,bjhc->bihc", P, vt) * torch.from_numpy(do)).sum().backward()
    for r, (s_, h, i_) in enumerate(qrows):
        np.testing.assert_allclose(dq[r], qt.grad[s_, i_, h].numpy(), rtol=0, atol=1e-12)
    for r, (s_, h, j_) in enumerate(krows):
        np.testing.assert_allclose(dk[r], kt.grad[s_, j_, h].numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[r], vt.grad[s_, j_, h].numpy(), rtol=0, atol=1e-12)


def test_backward_rows_packed():
    """bwd_rows on a packed batch equals the full packed bwd at those rows."""
    lens = [5, 0, 37, 12]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, H, d = int(cu[-1]), 2, 8
    q, k, v, do = (_rand((T, H, d), s) for s in (65, 66, 67, 68))
    qrows = np.array([[0, 1, 4], [2, 0, 36], [3, 1, 0], [2, 1, 3]])
    krows = np.array([[2, 0, 36], [2, 0, 2], [0, 0, 0], [3, 1, 11]])
    dq, dk, dv = orc.bwd_rows(q, k, v, do, 0.4, qrows, krows, causal=True, window=9,
                              cu_seqlens=cu)
    full = orc.bwd(q, k, v, do, 0.4, causal=True, window=9, cu_seqlens=cu)
    for r, (s_, h, i) in enumerate(qrows):
        np.testing.assert_array_equal(dq[r], full["dq"][cu[s_] + i, h])
    for r, (s_, h, j) in enumerate(krows):
        np.testing.assert_array_equal(dk[r], full["dk"][cu[s_] + j, h])
        np.testing.assert_array_equal(dv[r], full["dv"][cu[s_] + j, h])


def test_window_without_causal_is_rejected():
    q = _rand((1, 4, 1, 2), 46)
    with pytest.raises(ValueError):
        orc.fwd(q, q, q, 1.0, causal=False, window=2)
