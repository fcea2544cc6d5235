"""ctypes binding of the C ABI in include/fa.h.

Argument marshalling only: every step of the attention path runs in the CUDA
kernels of libfa_b200.so.  Tensors are torch CUDA tensors (torch provides the
device memory and the stream); nothing here computes attention, and there is
no fallback: if the library or a GPU is missing, the calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os

from . import build as _build

FA_OK = 0
STATUS = {
    0: "FA_OK", -1: "FA_ERR_NULLPTR", -2: "FA_ERR_UNSUPPORTED_D", -3: "FA_ERR_BAD_SHAPE",
    -4: "FA_ERR_MISALIGNED", -5: "FA_ERR_BAD_MASK", -6: "FA_ERR_WORKSPACE", -7: "FA_ERR_CUDA",
    -8: "FA_ERR_DEVICE_TIMEOUT", -9: "FA_ERR_BAD_SCALE", -10: "FA_ERR_SCRATCH_LIMIT",
}
NOALLOC_MAX_ROWS = 1 << 20   # FA_NOALLOC_MAX_ROWS in include/fa.h (8-byte entries)

# Exported entry points and their C signatures.
_VP, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I, _VP, _VP]),
    "fa_fwd_kv": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _I, _VP, _VP, _VP]),
    "fa_fwd_kvcache": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _I, _VP, _I,
                            _VP, _SZ, _VP]),
    "fa_fwd_kvcache_num_splits": (_I, [_I, _I, _I, _I, _I]),
    "fa_fwd_kvcache_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_fp8_vt_bytes": (_SZ, [_I, _I, _I, _I]),
    "fa_quantize_fp8": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP]),
    "fa_fwd_fp8": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I, _VP]),
    "fa_bwd_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I,
                    _VP, _VP, _SZ, _VP]),
    "fa_bwd_noalloc": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I,
                            _I, _VP, _VP]),
    "fa_bwd_fused_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_bwd_fused": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _F, _I, _I,
                          _VP, _VP, _SZ, _VP]),
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_get_device_error": (_I, [_VP]),
    "fa_debug_set_fault": (_I, [_I, ctypes.c_ulonglong]),
    "fa_profile_begin": (_I, []),
    "fa_profile_end": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
    "fa_profile_cta_balance": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]),
}

PROFILE_KINDS = ("fwd", "dot", "dkdv", "dq", "decode", "combine", "quant_fp8",
                 "fwd_fp8", "bwd_fused", "dq_convert")   # FA_PROFILE_KINDS order


class FaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%s)" % (where, STATUS.get(code, code),
                                                 status_string(code)))


_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def load_library():
    """Load libfa_b200.so (building it first when the sources are newer).
    Raises if it cannot be built or loaded: there is no other code path."""
    global _lib
    if _lib is None:
        path = _build.LIB_PATH
        if not os.path.exists(path) or _build.needs_build():
            _build.build()
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(code: int) -> str:
    return load_library().fa_status_string(int(code)).decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(code: int, where: str):
    if code != FA_OK:
        raise FaError(code, where)


# --------------------------------------------------------------- raw ABI ---

def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, window, cu_seqlens, stream=None) -> int:
    return load_library().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(H),
                                 int(N), int(d), float(scale), int(causal), int(window),
                                 _ptr(cu_seqlens), _stream(stream))


def fa_fwd_kv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, window, cu_seqlens_q,
              cu_seqlens_k, stream=None) -> int:
    return load_library().fa_fwd_kv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B),
                                    int(H), int(Nq), int(Nk), int(d), float(scale), int(causal),
                                    int(window), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
                                    _stream(stream))


def fa_fwd_kvcache(q, k_cache, v_cache, o, lse, B, H, Nq, Nk, d, scale, causal, window,
                   seqlens_k, num_splits, workspace, workspace_bytes, stream=None) -> int:
    return load_library().fa_fwd_kvcache(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o),
                                         _ptr(lse), int(B), int(H), int(Nq), int(Nk), int(d),
                                         float(scale), int(causal), int(window), _ptr(seqlens_k),
                                         int(num_splits), _ptr(workspace), int(workspace_bytes),
                                         _stream(stream))


def fa_fwd_kvcache_num_splits(B, H, Nq, Nk, d) -> int:
    return int(load_library().fa_fwd_kvcache_num_splits(int(B), int(H), int(Nq), int(Nk), int(d)))


def fa_fwd_kvcache_workspace_size(B, H, Nq, d, num_splits) -> int:
    return int(load_library().fa_fwd_kvcache_workspace_size(int(B), int(H), int(Nq), int(d),
                                                            int(num_splits)))


def fa_fp8_vt_bytes(B, H, N, d) -> int:
    return int(load_library().fa_fp8_vt_bytes(int(B), int(H), int(N), int(d)))


def fa_quantize_fp8(x, out, scales, B, N, H, d, transpose, signs, stream=None) -> int:
    return load_library().fa_quantize_fp8(_ptr(x), _ptr(out), _ptr(scales), int(B), int(N),
                                          int(H), int(d), int(transpose), _ptr(signs),
                                          _stream(stream))


def fa_fwd_fp8(q8, k8, vt8, sq, sk, sv, o, lse, B, H, N, d, scale, causal, window,
               stream=None) -> int:
    return load_library().fa_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(vt8), _ptr(sq), _ptr(sk),
                                     _ptr(sv), _ptr(o), _ptr(lse), int(B), int(H), int(N),
                                     int(d), float(scale), int(causal), int(window),
                                     _stream(stream))


def fa_bwd_workspace_size(B, H, N, d, varlen_total=0) -> int:
    return int(load_library().fa_bwd_workspace_size(int(B), int(H), int(N), int(d),
                                                    int(varlen_total)))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, window, cu_seqlens,
           workspace, workspace_bytes, stream=None) -> int:
    return load_library().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                 _ptr(dq), _ptr(dk), _ptr(dv), int(B), int(H), int(N), int(d),
                                 float(scale), int(causal), int(window), _ptr(cu_seqlens),
                                 _ptr(workspace), int(workspace_bytes), _stream(stream))


def fa_bwd_fused_workspace_size(B, H, N, d, varlen_total=0) -> int:
    return int(load_library().fa_bwd_fused_workspace_size(int(B), int(H), int(N), int(d),
                                                          int(varlen_total)))


def fa_bwd_fused(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, window, cu_seqlens,
                 workspace, workspace_bytes, stream=None) -> int:
    return load_library().fa_bwd_fused(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                       _ptr(dq), _ptr(dk), _ptr(dv), int(B), int(H), int(N),
                                       int(d), float(scale), int(causal), int(window),
                                       _ptr(cu_seqlens), _ptr(workspace), int(workspace_bytes),
                                       _stream(stream))


def fa_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, window,
                   cu_seqlens, stream=None) -> int:
    """fa_bwd without a workspace argument: for callers that cannot allocate
    device memory (its scratch is a fixed array inside the library)."""
    return load_library().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                         _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), int(B), int(H),
                                         int(N), int(d), float(scale), int(causal), int(window),
                                         _ptr(cu_seqlens), _stream(stream))


def fa_status_string(code: int) -> str:
    return status_string(code)


def fa_get_device_error(stream=None) -> int:
    return load_library().fa_get_device_error(_stream(stream))


def fa_debug_set_fault(mode: int, timeout_ns: int = 0) -> int:
    return load_library().fa_debug_set_fault(int(mode), int(timeout_ns))


def fa_profile_begin() -> int:
    return load_library().fa_profile_begin()


def fa_profile_cta_balance():
    """(mean CTA busy time / largest, grid size) of the last forward launch
    recorded while profiling was on."""
    b = ctypes.c_double()
    n = ctypes.c_int()
    _check(load_library().fa_profile_cta_balance(ctypes.byref(b), ctypes.byref(n)),
           "fa_profile_cta_balance")
    return b.value, n.value


def fa_profile_end():
    """Returns {kind: (total_ms, launches)} for the launches recorded since
    fa_profile_begin()."""
    ms = (ctypes.c_double * len(PROFILE_KINDS))()
    cnt = (ctypes.c_int * len(PROFILE_KINDS))()
    _check(load_library().fa_profile_end(ms, cnt), "fa_profile_end")
    return {k: (ms[i], cnt[i]) for i, k in enumerate(PROFILE_KINDS)}


# ------------------------------------------------------ tensor helpers ---
#
# The library reads and writes exactly the elements its size arguments imply,
# from each base pointer, in the documented dtype and dense layout.  The
# wrappers below derive those sizes from the tensors and refuse any tensor
# that does not match them (dtype, shape, contiguity, device), so that a
# mismatch raises here instead of making a kernel touch memory outside a
# tensor.  The raw fa_* functions above take pointers and do no such check.

def _require_cuda(t, name):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)


def _expect(t, name, shape, dtype, device):
    if t is None:
        raise ValueError("%s is required" % name)
    _require_cuda(t, name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if t.dtype != dtype:
        raise TypeError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _expect_bytes(t, name, nbytes, device):
    """A byte buffer (workspace): uint8, dense, at least nbytes long."""
    import torch
    _require_cuda(t, name)
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if t.dtype != torch.uint8 or not t.is_contiguous():
        raise TypeError("%s must be a contiguous uint8 tensor" % name)
    if t.numel() < nbytes:
        raise ValueError("%s holds %d bytes, %d needed" % (name, t.numel(), nbytes))


def _rank(t, name, ranks):
    if t is None or t.dim() not in ranks:
        raise ValueError("%s must have %s dimensions" % (name, " or ".join(map(str, ranks))))


def _shape(q, cu_seqlens):
    if cu_seqlens is None:
        _rank(q, "q", (4,))
        B, N, H, d = q.shape
        return B, H, N, d
    _rank(q, "q (packed)", (3,))
    _rank(cu_seqlens, "cu_seqlens", (1,))
    T, H, d = q.shape
    return cu_seqlens.numel() - 1, H, T, d


def forward(q, k, v, causal=False, window=0, cu_seqlens=None, scale=None, out=None, lse=None,
            stream=None):
    """O, LSE for bf16 CUDA tensors [B, N, H, d] (or packed [T, H, d] with
    int32 ``cu_seqlens``).  Outputs are allocated with torch when not given."""
    import torch
    B, H, N, d = _shape(q, cu_seqlens)
    dev = q.device
    lse_shape = (B, H, N) if cu_seqlens is None else (H, N)
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _expect(t, name, q.shape, torch.bfloat16, dev)
    if cu_seqlens is not None:
        _expect(cu_seqlens, "cu_seqlens", (B + 1,), torch.int32, dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
    _expect(out, "out", q.shape, torch.bfloat16, dev)
    _expect(lse, "lse", lse_shape, torch.float32, dev)
    _check(fa_fwd(q, k, v, out, lse, B, H, N, d, scale, causal, window, cu_seqlens, stream),
           "fa_fwd")
    return out, lse


def forward_kv(q, k, v, causal=False, window=0, cu_seqlens_q=None, cu_seqlens_k=None,
               scale=None, out=None, lse=None, stream=None):
    """O, LSE of queries q [B, Nq, H, d] against cached keys/values k, v
    [B, Nk, H, d] (or packed [Tq, H, d] / [Tk, H, d] with int32 cu_seqlens_q
    and cu_seqlens_k); queries are the last positions of their key sequence."""
    import torch
    if (cu_seqlens_q is None) != (cu_seqlens_k is None):
        raise ValueError("cu_seqlens_q and cu_seqlens_k go together")
    B, H, Nq, d = _shape(q, cu_seqlens_q)
    dev = q.device
    _expect(q, "q", q.shape, torch.bfloat16, dev)
    if cu_seqlens_q is None:
        _rank(k, "k", (4,))
        Nk = k.shape[1]
        kv_shape = (B, Nk, H, d)
    else:
        _rank(k, "k (packed)", (3,))
        Nk = k.shape[0]
        kv_shape = (Nk, H, d)
        _expect(cu_seqlens_q, "cu_seqlens_q", (B + 1,), torch.int32, dev)
        _expect(cu_seqlens_k, "cu_seqlens_k", (B + 1,), torch.int32, dev)
    _expect(k, "k", kv_shape, torch.bfloat16, dev)
    _expect(v, "v", kv_shape, torch.bfloat16, dev)
    lse_shape = (B, H, Nq) if cu_seqlens_q is None else (H, Nq)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
    _expect(out, "out", q.shape, torch.bfloat16, dev)
    _expect(lse, "lse", lse_shape, torch.float32, dev)
    _check(fa_fwd_kv(q, k, v, out, lse, B, H, Nq, Nk, d, scale, causal, window, cu_seqlens_q,
                     cu_seqlens_k, stream), "fa_fwd_kv")
    return out, lse


def forward_kvcache(q, k_cache, v_cache, seqlens_k=None, causal=False, window=0, scale=None,
                    num_splits=0, out=None, lse=None, workspace=None, stream=None):
    """Attention against a K/V cache: q [B, Nq, H, d] (a few decode queries, or
    a prefill chunk) against k_cache, v_cache [B, Nk, H, d], of which sequence
    b uses its first seqlens_k[b] rows (int32 CUDA tensor, or None for all Nk);
    queries are the last Nq of those positions.  Returns (O, LSE)."""
    import torch
    _rank(q, "q", (4,))
    _rank(k_cache, "k_cache", (4,))
    B, Nq, H, d = q.shape
    Nk = k_cache.shape[1]
    dev = q.device
    _expect(q, "q", q.shape, torch.bfloat16, dev)
    _expect(k_cache, "k_cache", (B, Nk, H, d), torch.bfloat16, dev)
    _expect(v_cache, "v_cache", (B, Nk, H, d), torch.bfloat16, dev)
    if seqlens_k is not None:
        _expect(seqlens_k, "seqlens_k", (B,), torch.int32, dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    _expect(out, "out", q.shape, torch.bfloat16, dev)
    _expect(lse, "lse", (B, H, Nq), torch.float32, dev)
    ns = num_splits if num_splits > 0 else fa_fwd_kvcache_num_splits(B, H, Nq, Nk, d)
    need = fa_fwd_kvcache_workspace_size(B, H, Nq, d, ns)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if workspace is not None:
        _expect_bytes(workspace, "workspace", need, dev)
    _check(fa_fwd_kvcache(q, k_cache, v_cache, out, lse, B, H, Nq, Nk, d, scale, causal, window,
                          seqlens_k, ns, workspace,
                          0 if workspace is None else workspace.numel(), stream),
           "fa_fwd_kvcache")
    return out, lse


def quantize_fp8(q, k, v, signs=None, stream=None):
    """Block-quantise bf16 q, k, v [B, N, H, 128] for forward_fp8: returns a
    dict with q8, k8 (uint8 e4m3 codes [B, N, H, 128]), vt8 (uint8 [B, H,
    128, Np]) and their scales sq, sk, sv [B, H, ceil(N / 128)].  signs (128
    floats of +-1 on the device) rotates Q and K first."""
    import torch
    _rank(q, "q", (4,))
    B, N, H, d = q.shape
    nb = (N + 127) // 128
    dev = q.device
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        _expect(t, name, q.shape, torch.bfloat16, dev)
    if signs is not None:
        _expect(signs, "signs", (d,), torch.float32, dev)
    out = {"q8": torch.empty((B, N, H, d), dtype=torch.uint8, device=dev),
           "k8": torch.empty((B, N, H, d), dtype=torch.uint8, device=dev),
           "vt8": torch.empty(max(1, fa_fp8_vt_bytes(B, H, N, d)), dtype=torch.uint8, device=dev),
           "sq": torch.empty((B, H, nb), dtype=torch.float32, device=dev),
           "sk": torch.empty((B, H, nb), dtype=torch.float32, device=dev),
           "sv": torch.empty((B, H, nb), dtype=torch.float32, device=dev)}
    _check(fa_quantize_fp8(q, out["q8"], out["sq"], B, N, H, d, 0, signs, stream), "fa_quantize_fp8")
    _check(fa_quantize_fp8(k, out["k8"], out["sk"], B, N, H, d, 0, signs, stream), "fa_quantize_fp8")
    _check(fa_quantize_fp8(v, out["vt8"], out["sv"], B, N, H, d, 1, None, stream), "fa_quantize_fp8")
    return out


def forward_fp8(qz, B, N, H, d=128, causal=False, window=0, scale=None, out=None, lse=None,
                stream=None):
    """FP8 forward from the output of quantize_fp8.  Returns (O bf16, LSE)."""
    import torch
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dev = qz["q8"].device
    nb = (N + 127) // 128
    _expect(qz["q8"], "q8", (B, N, H, d), torch.uint8, dev)
    _expect(qz["k8"], "k8", (B, N, H, d), torch.uint8, dev)
    _expect_bytes(qz["vt8"], "vt8", fa_fp8_vt_bytes(B, H, N, d), dev)
    for name in ("sq", "sk", "sv"):
        _expect(qz[name], name, (B, H, nb), torch.float32, dev)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    _expect(out, "out", (B, N, H, d), torch.bfloat16, dev)
    _expect(lse, "lse", (B, H, N), torch.float32, dev)
    _check(fa_fwd_fp8(qz["q8"], qz["k8"], qz["vt8"], qz["sq"], qz["sk"], qz["sv"], out, lse, B, H,
                      N, d, scale, causal, window, stream), "fa_fwd_fp8")
    return out, lse


def backward(q, k, v, o, lse, dout, causal=False, window=0, cu_seqlens=None, scale=None,
             grads=None, workspace=None, stream=None, fused=False):
    """dQ, dK, dV for the forward's (O, LSE) and the output gradient dO.
    fused=True runs the single-kernel backward (fa_bwd_fused, d = 128)."""
    import torch
    B, H, N, d = _shape(q, cu_seqlens)
    dev = q.device
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _expect(t, name, q.shape, torch.bfloat16, dev)
    _expect(lse, "lse", (B, H, N) if cu_seqlens is None else (H, N), torch.float32, dev)
    if cu_seqlens is not None:
        _expect(cu_seqlens, "cu_seqlens", (B + 1,), torch.int32, dev)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = grads
    for t, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _expect(t, name, q.shape, torch.bfloat16, dev)
    size_fn = fa_bwd_fused_workspace_size if fused else fa_bwd_workspace_size
    ws_bytes = size_fn(B, H, N, d, N if cu_seqlens is not None else 0)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    _expect_bytes(workspace, "workspace", ws_bytes, dev)
    fn = fa_bwd_fused if fused else fa_bwd
    _check(fn(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, window,
              cu_seqlens, workspace, workspace.numel(), stream), fn.__name__)
    return dq, dk, dv
