"""Pins for the FP8 oracle (fp8_oracle.c): e4m3 rounding against torch's
float8_e4m3fn conversion and hand values, the rotation against scipy's
Hadamard matrix, the block quantiser against a numpy restatement of its
definition and the e4m3 error bound, and the FP8 forward against the exact
oracle where its quantisation steps are switched off."""
import math

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

@pytest.mark.parametrize("rotate", [False, True])
def test_quantiser_definition(rotate):
    x = fixed_inputs(2, 200, 3, 128, seed=4)["q"]          # ragged last block (72 rows)
    s = fp8_signs(5) if rotate else None
    codes, scales = orc.quantize_fp8(x, s)
    xf = x.float().numpy()
    y = orc.rotate_rows(xf, s.numpy()) if rotate else xf
    B, N, H, d = xf.shape
    for b in range(B):
        for h in range(H):
            for blk in range(2):
                rows = slice(128 * blk, min(N, 128 * blk + 128))
                yb = y[b, rows, h]
                sc = np.float32(np.abs(yb).max()) / np.float32(448.0)
                assert scales[b, h, blk] == sc
                inv = np.float32(1.0) / sc
                ref = torch.from_numpy((yb * inv).astype(np.float32)).to(torch.float8_e4m3fn).float()
                assert np.array_equal(codes[b, rows, h], ref.numpy())
                # e4m3 error bound: half a spacing (2^-4 relative, 2^-10 absolute below 2^-6)
                err = np.abs(codes[b, rows, h].astype(np.float64) * sc - yb)
                assert np.all(err <= np.maximum(np.abs(yb) * 2.0 ** -4, 2.0 ** -10 * sc) * 1.0001)


def test_quantiser_zero_block():
    x = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    codes, scales = orc.quantize_fp8(x)
    assert scales[0, 0, 0] == 1.0 and not codes.any()


# ---------------------------------------------------------- forward ---

@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 50)])
def test_fwd_fp8_without_quantisation_is_exact(causal, window):
    # exact values as "codes", unit Q/K scales, V block scales folded in
    # exactly (codes = V / s_b), P not rounded: the exact forward
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
