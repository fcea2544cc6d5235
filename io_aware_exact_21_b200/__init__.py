"""B200 (sm_100a) exact IO-aware attention: a C-ABI CUDA library
(include/fa.h, csrc/) and its thin Python binding.

    from io_aware_exact_21_b200 import forward, backward
    o, lse = forward(q, k, v, causal=True)
    dq, dk, dv = backward(q, k, v, o, lse, do, causal=True)
"""
from .binding import (FaError, backward, fa_bwd, fa_bwd_fused, fa_bwd_fused_workspace_size,
                      fa_bwd_noalloc, fa_bwd_workspace_size,
                      fa_debug_set_fault, fa_fp8_vt_bytes, fa_fwd, fa_fwd_fp8, fa_fwd_kv,
                      fa_fwd_kvcache, fa_quantize_fp8, forward_fp8, quantize_fp8,
                      fa_fwd_kvcache_num_splits, fa_fwd_kvcache_workspace_size,
                      fa_get_device_error, fa_profile_begin, fa_profile_cta_balance, fa_profile_end, fa_status_string,
                      forward, forward_kv, forward_kvcache, library_path, load_library)

__all__ = ["FaError", "backward", "fa_bwd", "fa_bwd_fused", "fa_bwd_fused_workspace_size",
           "fa_bwd_noalloc", "fa_bwd_workspace_size",
           "fa_debug_set_fault", "fa_fp8_vt_bytes", "fa_fwd", "fa_fwd_fp8", "fa_fwd_kv",
           "fa_fwd_kvcache", "fa_quantize_fp8", "forward_fp8", "quantize_fp8",
           "fa_fwd_kvcache_num_splits", "fa_fwd_kvcache_workspace_size", "fa_get_device_error",
           "fa_profile_begin", "fa_profile_cta_balance", "fa_profile_end", "fa_status_string", "forward", "forward_kv",
           "forward_kvcache", "library_path", "load_library"]
