"""Pins for the FP8 oracle (fp8_oracle.c): e4m3 rounding against torch's
float8_e4m3fn conversion and hand values, the rotation against scipy's
Hadamard matrix, the block quantiser against a brute-force nearest-value
search over torch's table of all e4m3 values and the e4m3 error bound, and the
FP8 forward against hand-derived values (tests/golden/fp8_hand_worked.json),
the exact oracle where its quantisation steps are switched off, and closed
forms for rows that see one key or keys of equal score."""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from io_aware_exact_21_b200.inputs import fixed_inputs, fp8_signs
from oracle import oracle as orc


# ------------------------------------------------------------ e4m3 ---

def test_e4m3_hand_values():
    cases = {0.0: 0.0, 1.0: 1.0, 447.0: 448.0, 448.0: 448.0, 1000.0: 448.0, -1000.0: -448.0,
             2.0 ** -9: 2.0 ** -9,            # smallest subnormal
             2.0 ** -10: 0.0,                 # tie between 0 and 2^-9 -> even (0)
             3 * 2.0 ** -10: 2.0 ** -8,       # tie between 2^-9 and 2^-8 -> even (2^-8)
             1.0625: 1.0, 1.1875: 1.25,       # ties at spacing 1/8 -> even mantissa
             -0.3: -0.3125, 240.0: 240.0, 250.0: 256.0}
    for x, want in cases.items():
        assert orc.e4m3_round(np.array([x]))[0] == np.float32(want), x


def test_e4m3_matches_torch_float8():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(20000) * np.exp2(rng.uniform(-12, 8.7, 20000))).astype(np.float32)
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(orc.e4m3_round(x), ref)


# --------------------------------------------------------- rotation ---

def test_rotation_is_the_signed_hadamard_transform():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((40, 128)).astype(np.float32)
    s = fp8_signs(7).numpy()
    Hm = scipy.linalg.hadamard(128).astype(np.float64)
    want = (x.astype(np.float64) * s) @ Hm / math.sqrt(128)
    got = orc.rotate_rows(x, s)
    np.testing.assert_allclose(got, want, rtol=0, atol=2e-5)


def test_rotation_preserves_dot_products():
    rng = np.random.default_rng(2)
    a = rng.standard_normal((8, 128)).astype(np.float32)
    b = rng.standard_normal((8, 128)).astype(np.float32)
    s = fp8_signs(3).numpy()
    ra, rb = orc.rotate_rows(a, s), orc.rotate_rows(b, s)
    np.testing.assert_allclose(ra.astype(np.float64) @ rb.T.astype(np.float64),
                               a.astype(np.float64) @ b.T.astype(np.float64), rtol=0, atol=1e-4)


# -------------------------------------------------------- quantiser ---

def e4m3_table():
    """All finite e4m3 values (from torch's float8_e4m3fn bit patterns) and
    whether their last mantissa bit is 0 (the even ones)."""
    bits = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    vals = bits.view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    even = (bits.numpy() & 1) == 0
    ok = np.isfinite(vals)
    return vals[ok], even[ok]


def nearest_e4m3(y):
    """Nearest e4m3 value of each float64 y by brute force over the table;
    ties to the even code; |y| >= 448 saturates."""
    vals, even = e4m3_table()
    y = np.asarray(y, dtype=np.float64).ravel()
    out = np.empty_like(y)
    for n, t in enumerate(y):
        if abs(t) >= 448.0:
            out[n] = math.copysign(448.0, t)
            continue
        dist = np.abs(vals - t)
        best = dist.min()
        cand = np.nonzero(dist == best)[0]
        if len(cand) > 1:
            cand = [c for c in cand if even[c]] or list(cand)
        out[n] = vals[cand[0]]
    return out

@pytest.mark.parametrize("rotate", [False, True])
def test_quantiser_definition(rotate):
    x = fixed_inputs(2, 200, 3, 128, seed=4)["q"]          # ragged last block (72 rows)
    s = fp8_signs(5) if rotate else None
    codes, scales = orc.quantize_fp8(x, s)
    xf = x.float().numpy()
    y = orc.rotate_rows(xf, s.numpy()) if rotate else xf
    B, N, H, d = xf.shape
    for b in range(B):
        for h in range(H) if b == 0 else range(1):
            for blk in range(2):
                rows = slice(128 * blk, min(N, 128 * blk + 128))
                yb = y[b, rows, h]
                sc = np.float32(np.abs(yb).max()) / np.float32(448.0)
                assert scales[b, h, blk] == sc
                # the real quotient, rounded once to the nearest e4m3 value
                ref = nearest_e4m3(yb.astype(np.float64) / np.float64(sc)).reshape(yb.shape)
                assert np.array_equal(codes[b, rows, h], ref)
                # e4m3 error bound: half a spacing (2^-4 relative, 2^-10 absolute below 2^-6)
                err = np.abs(codes[b, rows, h].astype(np.float64) * sc - yb)
                assert np.all(err <= np.maximum(np.abs(yb) * 2.0 ** -4, 2.0 ** -10 * sc) * 1.0001)


def test_quantiser_rounds_the_real_quotient_not_a_reciprocal_product():
    # values whose float32 product x * fl(1/s) lands on the other side of an
    # e4m3 rounding boundary than the real quotient x / s: the codes follow
    # the quotient
    rng = np.random.default_rng(21)
    found = []
    while len(found) < 3:
        amax = np.float32(rng.uniform(1.0, 8.0))
        sc = amax / np.float32(448.0)
        inv = np.float32(1.0) / sc
        xs = rng.uniform(-amax, amax, 200000).astype(np.float32)
        prod = nearest_e4m3((xs * inv).astype(np.float32).astype(np.float64))
        quot = nearest_e4m3(xs.astype(np.float64) / np.float64(sc))
        for i in np.nonzero(prod != quot)[0][:1]:
            found.append((amax, xs[i], quot[i], prod[i]))
    for amax, xv, want, other in found:
        row = np.zeros((1, 1, 1, 128), np.float32)
        row[0, 0, 0, 0] = amax
        row[0, 0, 0, 1] = xv
        codes, scales = orc.quantize_fp8(row)
        assert codes[0, 0, 0, 1] == want and want != other
def test_quantiser_zero_block():
    x = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    codes, scales = orc.quantize_fp8(x)
    assert scales[0, 0, 0] == 1.0 and not codes.any()


# ---------------------------------------------------------- forward ---

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp8_hand_worked.json")


def _num(v):
    if isinstance(v, (int, float)):
        return float(v)
    if v.startswith("ln"):
        return math.log(float(v[2:]))
    a, b = v.split("/")
    return float(a) / float(b)


def test_fwd_fp8_golden_hand_worked():
    g = json.load(open(GOLDEN))
    inp = g["inputs"]
    arrays = {}
    for name in ("q_codes", "k_codes", "v_codes"):
        a = np.zeros((1, 2, 1, 128), np.float32)
        for r in (0, 1):
            for c, val in inp[name]["row%d" % r].items():
                a[0, r, 0, int(c)] = val
        arrays[name] = a
    one = np.ones((1, 1, 1), np.float32)
    sv = np.full((1, 1, 1), inp["sv"], np.float32)
    scale = -math.log(0.3) / 1.25
    args = (arrays["q_codes"], arrays["k_codes"], arrays["v_codes"], one * inp["sq"],
            one * inp["sk"], sv, scale)
    O, L, t = orc.fwd_fp8(*args, terms=True)
    np.testing.assert_allclose(O[0, 0, 0, :2], [_num(v) for v in g["o_row0"]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(O[0, 1, 0, :2], g["o_row1"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(L[0, 0], [_num(v) for v in g["lse"]], rtol=0, atol=1e-14)
    for name, v in g["terms_row0_ch0"].items():
        assert abs(t[name][0, 0, 0, 0] - _num(v)) < 1e-14, name
    Ou, _ = orc.fwd_fp8(*args, quantize_p=False)
    np.testing.assert_allclose(Ou[0, 0, 0, :2], [_num(v) for v in g["o_row0_unrounded"]],
                               rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 50)])
def test_fwd_fp8_without_quantisation_is_exact(causal, window):
    # exact values as "codes", unit Q/K scales, V block scales folded in
    # exactly (codes = V / s_b), p not rounded: the exact forward
    x = fixed_inputs(2, 300, 2, 128, seed=6)
    q, k, v = (x[n].float().numpy() for n in ("q", "k", "v"))
    nb = 3
    ones = np.ones((2, 2, nb), np.float32)
    sv = np.array([0.5, 2.0, 1.0], np.float32)[None, None, :].repeat(2, 0).repeat(2, 1)
    vc = v.copy()
    for blk in range(nb):
        vc[:, 128 * blk:128 * blk + 128] /= sv[0, 0, blk]
    O, L = orc.fwd_fp8(q, k, vc, ones, ones, sv, 0.1, causal, window, quantize_p=False)
    Oe, Le = orc.fwd(x["q"], x["k"], x["v"], 0.1, causal=causal, window=window)
    np.testing.assert_allclose(O, Oe, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Le, rtol=0, atol=1e-12)


def test_fwd_fp8_one_key_rows_and_equal_scores():
    # a row that sees one key has p = 1 = e4m3(1): O is that key's
    # dequantised V row exactly, and the bound sums are |v^|, |cv| and squares
    x = fixed_inputs(1, 300, 2, 128, seed=9)
    qc, sq = orc.quantize_fp8(x["q"])
    kc, sk = orc.quantize_fp8(x["k"])
    vc, sv = orc.quantize_fp8(x["v"])
    O, L, t = orc.fwd_fp8(qc, kc, vc, sq, sk, sv, 0.2, True, 1, terms=True)
    vh = vc.astype(np.float64) * np.repeat(sv, 128, axis=2)[:, :, :300].transpose(0, 2, 1)[..., None]
    np.testing.assert_array_equal(O, vh)
    np.testing.assert_array_equal(t["wa"], np.abs(vh))
    np.testing.assert_array_equal(t["wz"], np.abs(vc))
    np.testing.assert_allclose(t["wa2"], vh ** 2, rtol=1e-15)
    np.testing.assert_allclose(t["wz2"], vc.astype(np.float64) ** 2, rtol=1e-15)
    # all keys with equal scores (zero queries): the mean of the allowed V rows
    qz = np.zeros_like(qc)
    O2, L2 = orc.fwd_fp8(qz, kc, vc, sq, sk, sv, 0.2, True, 0)
    csum = np.cumsum(vh, axis=1) / np.arange(1, 301)[None, :, None, None]
    np.testing.assert_allclose(O2, csum, rtol=0, atol=1e-13)
    np.testing.assert_allclose(L2, np.log(np.arange(1, 301))[None, None, :].repeat(2, 1),
                               rtol=0, atol=1e-13)


def test_fwd_fp8_error_against_exact():
    # Size of the quantisation error on i.i.d. normal inputs: the mean absolute
    # error of O stays well under a tenth of the mean |O|.
    x = fixed_inputs(1, 2048, 2, 128, seed=8)
    scale = 1 / math.sqrt(128)
    Oe, Le = orc.fwd(x["q"], x["k"], x["v"], scale)
    qc, sq = orc.quantize_fp8(x["q"])
    kc, sk = orc.quantize_fp8(x["k"])
    vc, sv = orc.quantize_fp8(x["v"])
    O, L = orc.fwd_fp8(qc, kc, vc, sq, sk, sv, scale)
    assert np.abs(O - Oe).mean() < 0.1 * np.abs(Oe).mean()
    assert np.abs(L - Le).max() < 0.05


def test_rotation_rescues_values_below_the_e4m3_normal_range():
    # What the rotation is for: one element 1e5 times the others sets the
    # block scale so high that the rest of the block falls below e4m3's
    # smallest normal (2^-6 of the scale) and loses precision; rotating spreads
    # that element over its row first.  (With ordinary magnitudes e4m3's
    # floating-point codes keep 2^-4 relative precision and the rotation
    # brings nothing.)
    x = fixed_inputs(1, 128, 1, 128, seed=8)
    q = x["q"].float().clone()
    q[0, 3, 0, 17] = 1e5
    q = q.to(torch.bfloat16)
    k = x["k"]
    S = q[0, :, 0].double().numpy() @ k[0, :, 0].double().numpy().T
    rows = np.arange(128) != 3
    errs = []
    for signs in (None, fp8_signs(9)):
        qc, sq = orc.quantize_fp8(q, signs)
        kc, sk = orc.quantize_fp8(k, signs)
        Sq = (qc[0, :, 0].astype(np.float64) * sq[0, 0, 0]) @ \
             (kc[0, :, 0].astype(np.float64) * sk[0, 0, 0]).T
        errs.append(np.abs(Sq - S)[rows].mean() / np.abs(S)[rows].mean())
    assert errs[0] > 0.1 and errs[1] < 0.05
