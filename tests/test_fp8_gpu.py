"""FP8 path on the GPU: fa_quantize_fp8 against the oracle's quantiser (bit
for bit: the codes are the real quotient x / s rounded once to e4m3 on both
sides), and fa_fwd_fp8 against the oracle's block-quantised forward and
against exact attention.

Tolerance of the forward against its oracle, derived from e4m3's spacing.
Both sides compute the scores from the same codes and scales; they differ in
how the probabilities are rounded to e4m3.  The oracle rounds p = exp(x - m)
against the row maximum m (p <= 1).  The kernel walks the keys in tiles with a
lagging reference (raised only when a tile's maximum exceeds it by more than
2^3 in base 2) and folds the V block scale into P, so it rounds p * kappa with
kappa = 2^(m - m_ref) * s_v(b) / max s_v >= s_v(b) / max s_v, then divides
kappa back out.  Rounding to nearest e4m3 moves a value y by at most
max(2^-4 y, 2^-10) (3 mantissa bits; spacing 2^-9 below 2^-6), so per key the
two sides' P differ by at most 2^-3 p + 2^-10 (1 + max s_v / s_v(b)), and per
output element (row i, channel c)
    |O_gpu - O_oracle| <= 2^-3 wa + 2^-9 max s_v wz + 2^-8 |O| + 1e-4 wa + 1e-6
with wa = sum_j p_j |v^_jc| / l and wz = sum_j |cv_jc| / l from the oracle
(v^ dequantised, cv the codes), 2^-8 |O| for the bf16 output, 1e-4 wa for the
float32 scores and exponentials.  The rounding errors of different keys are
independent and centred, so the mean error is held to the root mean square
of that sum, sqrt(2/3 (2^-8 wa2 + 2^-20 max s_v^2 wz2)) + 2^-9 |O| (wa2, wz2:
the oracle's sums of squares)."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import fixed_inputs, fp8_signs
from oracle import oracle as orc

from helpers import to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL_FP8_LSE = 1e-3


def e4m3_values(codes_u8):
    return codes_u8.cpu().view(torch.float8_e4m3fn).float().numpy()


def gpu_quantize(x, signs):
    qz = fa.quantize_fp8(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV),
                         None if signs is None else signs.to(DEV))
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return qz


def vt_to_tokens(vt8, B, N, H):
    Np = (N + 15) // 16 * 16
    a = vt8[:B * H * 128 * Np].view(B, H, 128, Np)
    return a, a[..., :N].permute(0, 3, 1, 2)          # [B, N, H, 128]


@pytest.mark.parametrize("B,N,H", [(1, 1, 1), (2, 200, 3), (1, 128, 2), (1, 300, 2), (2, 1000, 1)])
@pytest.mark.parametrize("rotate", [False, True])
def test_quantiser_bit_exact(B, N, H, rotate):
    x = fixed_inputs(B, N, H, 128, seed=N + 3)
    signs = fp8_signs(11) if rotate else None
    qz = gpu_quantize(x, signs)
    for name, src, sgn in (("q", x["q"], signs), ("k", x["k"], signs)):
        codes, scales = orc.quantize_fp8(src, sgn)
        assert np.array_equal(e4m3_values(qz[name + "8"]), codes), name
        assert np.array_equal(qz["s" + name].cpu().numpy(), scales), name
    codes, scales = orc.quantize_fp8(x["v"])
    full, tok = vt_to_tokens(qz["vt8"], B, N, H)
    assert np.array_equal(e4m3_values(tok.contiguous()), codes)
    assert np.array_equal(qz["sv"].cpu().numpy(), scales)
    assert torch.count_nonzero(full[..., N:]) == 0            # padding keys are zero


def oracle_fp8(x, signs, causal, window, scale=1 / math.sqrt(128)):
    qc, sq = orc.quantize_fp8(x["q"], signs)
    kc, sk = orc.quantize_fp8(x["k"], signs)
    vc, sv = orc.quantize_fp8(x["v"])
    O, L, t = orc.fwd_fp8(qc, kc, vc, sq, sk, sv, scale, causal, window, terms=True)
    return O, L, t, sv


def fp8_bounds(O, t, sv):
    """Per-element max bound and per-element RMS estimate (module docstring)."""
    svm = sv.max(axis=2)[:, None, :, None]          # [B, 1, H, 1]
    bmax = 2.0 ** -3 * t["wa"] + 2.0 ** -9 * svm * t["wz"] + 2.0 ** -8 * np.abs(O) \
        + 1e-4 * t["wa"] + 1e-6
    rms = np.sqrt((2.0 / 3.0) * (2.0 ** -8 * t["wa2"] + 2.0 ** -20 * svm ** 2 * t["wz2"])) \
        + 2.0 ** -9 * np.abs(O)
    return bmax, rms


def check_close(o, lse, ref):
    O, L, t, sv = ref
    g = to64(o)
    assert np.isfinite(g).all()
    err = np.abs(g - O)
    bmax, rms = fp8_bounds(O, t, sv)
    worst = np.unravel_index(np.argmax(err / bmax), err.shape)
    assert (err <= bmax).all(), "O: error %.3e above its bound %.3e at %s" % (
        err[worst], bmax[worst], worst)
    assert err.mean() <= rms.mean(), "O: mean error %.3e above %.3e" % (err.mean(), rms.mean())
    el = np.abs(to64(lse) - L)
    assert el.max() <= TOL_FP8_LSE, "lse: max %.3e" % el.max()


@pytest.mark.parametrize("B,N,H", [(1, 128, 1), (2, 300, 2), (1, 1000, 2), (2, 17, 1), (1, 2048, 1)])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 100)])
@pytest.mark.parametrize("rotate", [False, True])
def test_fwd_fp8_matches_its_oracle(B, N, H, causal, window, rotate):
    x = fixed_inputs(B, N, H, 128, seed=N + 17)
    signs = fp8_signs(12) if rotate else None
    qz = gpu_quantize(x, signs)
    o, lse = fa.forward_fp8(qz, B, N, H, causal=causal, window=window)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    check_close(o, lse, oracle_fp8(x, signs, causal, window))


@pytest.mark.parametrize("scale", [0.05, 0.15])
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_fp8_scale(scale, causal):
    """The softmax scale as an argument (the other cases run at 1/sqrt(128))."""
    B, N, H = 2, 300, 2
    x = fixed_inputs(B, N, H, 128, seed=760)
    signs = fp8_signs(12)
    qz = gpu_quantize(x, signs)
    o, lse = fa.forward_fp8(qz, B, N, H, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    check_close(o, lse, oracle_fp8(x, signs, causal, 0, scale))


def test_fwd_fp8_error_against_exact_attention():
    # the GPU's FP8 result is as far from exact attention as the FP8 oracle is
    x = fixed_inputs(1, 2048, 2, 128, seed=8)
    qz = gpu_quantize(x, None)
    o, lse = fa.forward_fp8(qz, 1, 2048, 2)
    torch.cuda.synchronize()
    Oe, Le = orc.fwd(x["q"], x["k"], x["v"], 1 / math.sqrt(128))
    g = to64(o)
    assert np.abs(g - Oe).mean() < 0.1 * np.abs(Oe).mean()
    assert np.abs(to64(lse) - Le).max() < 0.05


def test_fwd_fp8_workload_heads():
    # the measured configuration, B4 H16 N8192 d128 non-causal with the
    # rotation; two whole (sequence, head) slices against the oracle (the
    # quantisation is per (sequence, head), so a slice is self-contained)
    B, N, H = 4, 8192, 16
    x = fixed_inputs(B, N, H, 128, seed=2)
    signs = fp8_signs(1)
    qz = gpu_quantize(x, signs)
    o, lse = fa.forward_fp8(qz, B, N, H)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    for b, h in ((0, 0), (3, 9)):
        sl = {n: x[n][b:b + 1, :, h:h + 1] for n in ("q", "k", "v")}
        check_close(o[b:b + 1, :, h:h + 1], lse[b:b + 1, h:h + 1], oracle_fp8(sl, signs, False, 0))
