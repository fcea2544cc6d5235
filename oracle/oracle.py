"""Python face of the float64 CPU oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke``
and by ``bench.py``'s CPU-baseline leg and its ``--impl reference`` arm (the
oracle timed on the host cores).  The CUDA library never imports it, and it
imports nothing from the CUDA package.

The oracle computes, in float64 from exact upcasts of the (bf16) inputs, the
definition of scaled-dot-product attention, ``O = softmax(scale * Q K^T) V``
row by row over the keys the mask allows (FlashAttention encyclopedia page,
section "attention and the memory bottleneck"), with the three-pass safe
softmax of the blog article "From Online Softmax to FlashAttention", sections
2.1-2.2, and the gradients that follow from that definition.  See the header
of ``attn_oracle.c`` for the formulas.

Layouts accepted here:
  * fixed length: q, k, v, dout are ``[B, N, H, d]``; returned LSE and D are
    ``[B, H, N]``;
  * packed variable length: ``[T, H, d]`` plus ``cu_seqlens`` (B+1 int
    offsets); returned LSE and D are ``[H, T]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_SRC_FP8 = os.path.join(_HERE, "fp8_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libattn_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``attn_oracle.c`` and ``fp8_oracle.c`` into
    ``oracle/_build/libattn_oracle.so``.  ``-ffp-contract=off``: the float32
    steps of the FP8 quantiser must stay single IEEE operations."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_FP8))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-ffp-contract=off", "-o", tmp, _SRC, _SRC_FP8, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        common = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ip, ip,
                  ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_fwd.argtypes = common + [dp, dp]
        lib.oracle_fwd_rows.argtypes = common + [ctypes.c_int, ip, dp, dp]
        lib.oracle_fwd_online.argtypes = common + [ctypes.c_int, dp, dp]
        lib.oracle_fwd_kv.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ip, ip, ip, ip, ctypes.c_double,
                                      ctypes.c_int, ctypes.c_int, dp, dp]
        lib.oracle_fwd_kv.restype = ctypes.c_int
        lib.oracle_bwd.argtypes = ([dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ip, ip, ctypes.c_double, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ip, dp, dp, dp, dp, dp, dp])
        lib.oracle_bwd_rows.argtypes = ([dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ip, ip, ctypes.c_double, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ip, dp, ctypes.c_int, ip, dp, dp])
        for f in (lib.oracle_fwd, lib.oracle_fwd_rows, lib.oracle_fwd_online, lib.oracle_bwd,
                  lib.oracle_bwd_rows):
            f.restype = ctypes.c_int
        lib.oracle_num_threads.restype = ctypes.c_int
        fp = ctypes.POINTER(ctypes.c_float)
        lib.oracle_e4m3_round.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_round.restype = ctypes.c_float
        lib.oracle_rotate_rows.argtypes = [fp, ctypes.c_int, ctypes.c_int, fp]
        lib.oracle_rotate_rows.restype = ctypes.c_int
        lib.oracle_quantize_fp8.argtypes = [fp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, fp, fp, fp]
        lib.oracle_quantize_fp8.restype = ctypes.c_int
        lib.oracle_fwd_fp8.argtypes = [fp, fp, fp, fp, fp, fp, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp]
        lib.oracle_fwd_fp8.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _f64(x) -> np.ndarray:
    """Exact upcast to a C-contiguous float64 array (bf16 -> f64 is exact)."""
    if hasattr(x, "detach"):  # torch tensor
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


class _Packed:
    """Token-major [T, H, d] view of the inputs plus sequence starts/lengths."""

    def __init__(self, q, cu_seqlens):
        if cu_seqlens is None:
            if q.ndim != 4:
                raise ValueError("fixed-length inputs must be [B, N, H, d]")
            self.B, self.N, self.H, self.d = q.shape
            self.T = self.B * self.N
            self.starts = np.arange(self.B, dtype=np.int32) * self.N
            self.lens = np.full(self.B, self.N, dtype=np.int32)
            self.fixed = True
        else:
            if q.ndim != 3:
                raise ValueError("packed inputs must be [T, H, d]")
            cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens,
                            dtype=np.int64)
            self.T, self.H, self.d = q.shape
            self.B = len(cu) - 1
            self.starts = np.ascontiguousarray(cu[:-1], dtype=np.int32)
            self.lens = np.ascontiguousarray(cu[1:] - cu[:-1], dtype=np.int32)
            self.fixed = False

    def tok(self, x) -> np.ndarray:
        return _f64(x).reshape(self.T, self.H, self.d)

    def out_shape(self):
        return (self.B, self.N, self.H, self.d) if self.fixed else (self.T, self.H, self.d)

    def rowstat(self, a_ht: np.ndarray) -> np.ndarray:
        """[H, T] -> [B, H, N] for fixed length; unchanged for packed."""
        if self.fixed:
            return a_ht.reshape(self.H, self.B, self.N).transpose(1, 0, 2).copy()
        return a_ht


def _check(rc: int):
    if rc != 0:
        raise ValueError("oracle rejected the arguments (code %d)" % rc)


def fwd(q, k, v, scale, causal=False, window=0, cu_seqlens=None):
    """Three-pass float64 forward.  Returns (O, LSE) as float64 arrays."""
    pk = _Packed(q, cu_seqlens)
    Q, K, V = pk.tok(q), pk.tok(k), pk.tok(v)
    O = np.zeros_like(Q)
    L = np.zeros((pk.H, pk.T), dtype=np.float64)
    _check(_load().oracle_fwd(_dp(Q), _dp(K), _dp(V), pk.T, pk.H, pk.d, pk.B, _ip(pk.starts),
                              _ip(pk.lens), float(scale), int(bool(causal)), int(window),
                              _dp(O), _dp(L)))
    return O.reshape(pk.out_shape()), pk.rowstat(L)


def fwd_online(q, k, v, scale, block, causal=False, window=0, cu_seqlens=None):
    """Blocked one-pass forward with the online update; (O, LSE)."""
    pk = _Packed(q, cu_seqlens)
    Q, K, V = pk.tok(q), pk.tok(k), pk.tok(v)
    O = np.zeros_like(Q)
    L = np.zeros((pk.H, pk.T), dtype=np.float64)
    _check(_load().oracle_fwd_online(_dp(Q), _dp(K), _dp(V), pk.T, pk.H, pk.d, pk.B,
                                     _ip(pk.starts), _ip(pk.lens), float(scale),
                                     int(bool(causal)), int(window), int(block), _dp(O), _dp(L)))
    return O.reshape(pk.out_shape()), pk.rowstat(L)


def fwd_rows(q, k, v, rows, scale, causal=False, window=0, cu_seqlens=None):
    """Forward for selected rows.  ``rows`` is an int array [R, 3] of
    (sequence, head, row-within-sequence).  Returns (O_rows [R, d], LSE [R])."""
    pk = _Packed(q, cu_seqlens)
    Q, K, V = pk.tok(q), pk.tok(k), pk.tok(v)
    R = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    O = np.zeros((len(R), pk.d), dtype=np.float64)
    L = np.zeros(len(R), dtype=np.float64)
    _check(_load().oracle_fwd_rows(_dp(Q), _dp(K), _dp(V), pk.T, pk.H, pk.d, pk.B,
                                   _ip(pk.starts), _ip(pk.lens), float(scale),
                                   int(bool(causal)), int(window), len(R), _ip(R), _dp(O), _dp(L)))
    return O, L


def bwd(q, k, v, dout, scale, causal=False, window=0, cu_seqlens=None, heads=None):
    """Float64 backward.  ``heads``: optional list of (sequence, head) pairs;
    entries of other heads are returned as NaN.  Returns a dict with the
    oracle's own ``o``, ``lse``, ``D`` and ``dq``, ``dk``, ``dv``."""
    pk = _Packed(q, cu_seqlens)
    Q, K, V, dO = pk.tok(q), pk.tok(k), pk.tok(v), pk.tok(dout)
    out = {name: np.full_like(Q, np.nan) for name in ("o", "dq", "dk", "dv")}
    L = np.full((pk.H, pk.T), np.nan)
    Dd = np.full((pk.H, pk.T), np.nan)
    if heads is None:
        npairs, P = 0, None
    else:
        P = np.ascontiguousarray(np.asarray(heads, dtype=np.int32).reshape(-1, 2))
        npairs = len(P)
    _check(_load().oracle_bwd(_dp(Q), _dp(K), _dp(V), _dp(dO), pk.T, pk.H, pk.d, pk.B,
                              _ip(pk.starts), _ip(pk.lens), float(scale), int(bool(causal)),
                              int(window), npairs, None if P is None else _ip(P),
                              _dp(out["dq"]), _dp(out["dk"]), _dp(out["dv"]), _dp(out["o"]),
                              _dp(L), _dp(Dd)))
    res = {name: a.reshape(pk.out_shape()) for name, a in out.items()}
    res["lse"] = pk.rowstat(L)
    res["D"] = pk.rowstat(Dd)
    return res


def bwd_rows(q, k, v, dout, scale, qrows, krows, causal=False, window=0, cu_seqlens=None):
    """Float64 gradients for listed rows: ``qrows`` and ``krows`` are int
    arrays [R, 3] of (sequence, head, row-within-sequence).  Returns (dQ of
    the query rows [Rq, d], dK and dV of the key rows [Rk, d]), equal to the
    corresponding rows of ``bwd`` (same formulas, computed from the rows'
    own statistics, so a long sequence costs only the rows asked for)."""
    pk = _Packed(q, cu_seqlens)
    Q, K, V, dO = pk.tok(q), pk.tok(k), pk.tok(v), pk.tok(dout)
    QR = np.ascontiguousarray(np.asarray(qrows, dtype=np.int32).reshape(-1, 3))
    KR = np.ascontiguousarray(np.asarray(krows, dtype=np.int32).reshape(-1, 3))
    dq = np.zeros((len(QR), pk.d), dtype=np.float64)
    dk = np.zeros((len(KR), pk.d), dtype=np.float64)
    dv = np.zeros((len(KR), pk.d), dtype=np.float64)
    _check(_load().oracle_bwd_rows(_dp(Q), _dp(K), _dp(V), _dp(dO), pk.T, pk.H, pk.d, pk.B,
                                   _ip(pk.starts), _ip(pk.lens), float(scale),
                                   int(bool(causal)), int(window), len(QR), _ip(QR), _dp(dq),
                                   len(KR), _ip(KR), _dp(dk), _dp(dv)))
    return dq, dk, dv


def fwd_kv(q, k, v, scale, causal=False, window=0, cu_seqlens_q=None, cu_seqlens_k=None):
    """Forward of queries against a key/value sequence that may be longer
    (prefill with cached keys and values; causal masks bottom-right aligned).
    Fixed length: q [B, Nq, H, d], k/v [B, Nk, H, d] -> O [B, Nq, H, d],
    LSE [B, H, Nq].  Packed: q [Tq, H, d], k/v [Tk, H, d] with cu_seqlens_q/_k
    -> O [Tq, H, d], LSE [H, Tq]."""
    if cu_seqlens_q is None:
        B, Nq, H, d = q.shape
        Nk = k.shape[1]
        Q, K, V = (_f64(x).reshape(-1, H, d) for x in (q, k, v))
        qs = np.ascontiguousarray(np.arange(B, dtype=np.int32) * Nq)
        ks = np.ascontiguousarray(np.arange(B, dtype=np.int32) * Nk)
        ql = np.full(B, Nq, dtype=np.int32)
        kl = np.full(B, Nk, dtype=np.int32)
    else:
        cq = np.asarray(cu_seqlens_q.cpu() if hasattr(cu_seqlens_q, "cpu") else cu_seqlens_q,
                        dtype=np.int64)
        ck = np.asarray(cu_seqlens_k.cpu() if hasattr(cu_seqlens_k, "cpu") else cu_seqlens_k,
                        dtype=np.int64)
        H, d = q.shape[1], q.shape[2]
        B = len(cq) - 1
        Q, K, V = (_f64(x).reshape(-1, H, d) for x in (q, k, v))
        qs = np.ascontiguousarray(cq[:-1], dtype=np.int32)
        ks = np.ascontiguousarray(ck[:-1], dtype=np.int32)
        ql = np.ascontiguousarray(np.diff(cq), dtype=np.int32)
        kl = np.ascontiguousarray(np.diff(ck), dtype=np.int32)
    Tq, Tk = Q.shape[0], K.shape[0]
    O = np.zeros_like(Q)
    L = np.zeros((H, Tq), dtype=np.float64)
    _check(_load().oracle_fwd_kv(_dp(Q), _dp(K), _dp(V), Tq, Tk, H, d, B, _ip(qs), _ip(ql),
                                 _ip(ks), _ip(kl), float(scale), int(bool(causal)), int(window),
                                 _dp(O), _dp(L)))
    if cu_seqlens_q is None:
        return O.reshape(B, Nq, H, d), L.reshape(H, B, Nq).transpose(1, 0, 2).copy()
    return O, L


def fwd_kvcache(q, k_cache, v_cache, scale, seqlens_k=None, causal=False, window=0):
    """Decode against a padded key/value cache: q [B, Nq, H, d], k_cache and
    v_cache [B, Nk, H, d] of which sequence b uses its first seqlens_k[b] rows
    (all Nk when None); the queries are the last Nq of those positions.
    Returns O [B, Nq, H, d], LSE [B, H, Nq]."""
    B, Nq, H, d = q.shape
    Nk = k_cache.shape[1]
    Q, K, V = (_f64(x).reshape(-1, H, d) for x in (q, k_cache, v_cache))
    if seqlens_k is None:
        kl = np.full(B, Nk, dtype=np.int32)
    else:
        sk = seqlens_k.cpu() if hasattr(seqlens_k, "cpu") else seqlens_k
        kl = np.ascontiguousarray(np.clip(np.asarray(sk, dtype=np.int64), 0, Nk), dtype=np.int32)
    qs = np.ascontiguousarray(np.arange(B, dtype=np.int32) * Nq)
    ks = np.ascontiguousarray(np.arange(B, dtype=np.int32) * Nk)
    ql = np.full(B, Nq, dtype=np.int32)
    O = np.zeros_like(Q)
    L = np.zeros((H, B * Nq), dtype=np.float64)
    _check(_load().oracle_fwd_kv(_dp(Q), _dp(K), _dp(V), B * Nq, B * Nk, H, d, B, _ip(qs),
                                 _ip(ql), _ip(ks), _ip(kl), float(scale), int(bool(causal)),
                                 int(window), _dp(O), _dp(L)))
    return O.reshape(B, Nq, H, d), L.reshape(H, B, Nq).transpose(1, 0, 2).copy()


# ------------------------------------------------------------ FP8 path ---
# Block-quantised e4m3 forward (see the header of fp8_oracle.c for the steps).

def _f32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _fp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def e4m3_round(x) -> np.ndarray:
    """Element-wise nearest e4m3 value (ties to even, saturating at 448)."""
    f = _load().oracle_e4m3_round
    a = _f32(x)
    return np.vectorize(lambda v: f(float(v)), otypes=[np.float32])(a) if a.size else a


def rotate_rows(x, signs) -> np.ndarray:
    """Random-sign Walsh-Hadamard rotation of the last axis (d = 128), float32."""
    a = _f32(x).copy()
    sg = _f32(signs)
    rows = a.size // a.shape[-1] if a.size else 0
    _check(_load().oracle_rotate_rows(_fp(a), rows, a.shape[-1], _fp(sg)))
    return a


def quantize_fp8(x, signs=None):
    """x [B, N, H, 128] -> (codes [B, N, H, 128] float32 e4m3 values,
    scales [B, H, ceil(N / 128)] float32); rotated first when signs is given."""
    a = _f32(x)
    B, N, H, d = a.shape
    nb = (N + 127) // 128
    codes = np.zeros_like(a)
    scales = np.zeros((B, H, nb), dtype=np.float32)
    sg = None if signs is None else _f32(signs)
    _check(_load().oracle_quantize_fp8(_fp(a), B, N, H, d, None if sg is None else _fp(sg),
                                       _fp(codes), _fp(scales)))
    return codes, scales


def fwd_fp8(qc, kc, vc, sq, sk, sv, scale, causal=False, window=0, quantize_p=True,
            terms=False):
    """FP8 forward from codes and block scales (fixed length [B, N, H, d]):
    the exact softmax of the dequantised scores, with the probabilities
    rounded to e4m3 against the row maximum before they multiply the
    dequantised V.  Returns O [B, N, H, d] and LSE [B, H, N] in float64; with
    ``terms`` also a dict of the per-element sums an error bound needs
    (``wa``, ``wa2``, ``wz``, ``wz2``; see fp8_oracle.c)."""
    q, k, v = _f32(qc), _f32(kc), _f32(vc)
    B, N, H, d = q.shape
    o = np.zeros(q.shape, dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    t = {n: np.zeros(q.shape, dtype=np.float64) for n in ("wa", "wa2", "wz", "wz2")} if terms \
        else None
    tp = [_dp(t[n]) if terms else None for n in ("wa", "wa2", "wz", "wz2")]
    _check(_load().oracle_fwd_fp8(_fp(q), _fp(k), _fp(v), _fp(_f32(sq)), _fp(_f32(sk)),
                                  _fp(_f32(sv)), B, N, H, d, float(scale), int(bool(causal)),
                                  int(window), int(bool(quantize_p)), _dp(o), _dp(lse), *tp))
    return (o, lse, t) if terms else (o, lse)
