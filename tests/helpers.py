"""Shared test helpers: tolerance checks and seeded row sampling."""
import numpy as np
import torch

# Parity contract against the float64 oracle.
TOL_MAX = 2e-2      # bf16 outputs, max |err|
TOL_MEAN = 2e-3     # bf16 outputs, mean |err|
TOL_LSE = 1e-3      # fp32 LSE, max |err|


def to64(t) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close_bf16(got, ref, name=""):
    g = to64(got) if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), "%s has non-finite values" % name
    assert err.max() <= TOL_MAX and err.mean() <= TOL_MEAN, \
        "%s: max %.3e mean %.3e" % (name, err.max(), err.mean())


def assert_close_lse(got, ref, name="lse"):
    g = to64(got) if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    err = np.abs(g - ref)
    assert err.max() <= TOL_LSE, "%s: max %.3e" % (name, err.max())


def sample_rows(lens, H, count, seed):
    """Seeded (sequence, head, row) triples: tile edges of every sequence plus
    random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for s, n in enumerate(lens):
        for i in (0, 1, 127, 128, 129, 255, 256, n // 2, n - 2, n - 1):
            if 0 <= i < n:
                rows.add((s, int(rng.integers(0, H)), i))
    while len(rows) < count + len(lens) * 2:
        s = int(rng.integers(0, len(lens)))
        if lens[s] == 0:
            continue
        rows.add((s, int(rng.integers(0, H)), int(rng.integers(0, lens[s]))))
    return np.array(sorted(rows), dtype=np.int32)


def gather_rows(o, lse, rows, cu=None):
    """Rows of GPU outputs (fixed [B,N,H,d]/[B,H,N] or packed [T,H,d]/[H,T])."""
    O = o.detach().float().cpu().double().numpy()
    L = lse.detach().cpu().double().numpy()
    if cu is None:
        og = np.stack([O[s, i, h] for s, h, i in rows])
        lg = np.array([L[s, h, i] for s, h, i in rows])
    else:
        cu = np.asarray(cu)
        og = np.stack([O[cu[s] + i, h] for s, h, i in rows])
        lg = np.array([L[h, cu[s] + i] for s, h, i in rows])
    return og, lg


def assert_close_bf16_scaled(got, ref, name=""):
    """The bf16 bound for outputs that are not O(1): bf16 spaces values in
    [2^e, 2^(e+1)) by 2^(e-7), so rounding the output alone moves a value of
    magnitude 8 by up to 2^-5; the max-abs bound is TOL_MAX * max(1, |ref|)
    element by element, the mean-abs bound is unchanged."""
    g = to64(got) if hasattr(got, "detach") else np.asarray(got, dtype=np.float64)
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), "%s has non-finite values" % name
    ratio = err / np.maximum(1.0, np.abs(ref))
    assert ratio.max() <= TOL_MAX and err.mean() <= TOL_MEAN, \
        "%s: scaled max %.3e mean %.3e" % (name, ratio.max(), err.mean())
