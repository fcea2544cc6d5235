"""Failure path without a GPU fault: the test hook makes a kernel's load
thread skip one tile, so its consumers' bounded wait runs out; the kernel
returns, the host reads FA_ERR_DEVICE_TIMEOUT, and the context stays usable.
Covered for the forward kernel (mode 1) and the decode kernel (mode 2)."""
import math

import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import fixed_inputs, kvcache_inputs
from oracle import oracle as orc

from helpers import assert_close_bf16

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_recoverable():
    x = fixed_inputs(1, 512, 2, 128, seed=31)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    assert fa.fa_get_device_error() == 0
    fa.fa_debug_set_fault(1, 50_000_000)        # skip one V load, 50 ms limit
    try:
        fa.forward(q, k, v, causal=False)
        code = fa.fa_get_device_error()
    finally:
        fa.fa_debug_set_fault(0, 0)
    assert code == -8
    assert fa.fa_get_device_error() == 0        # the record was cleared
    o, lse = fa.forward(q, k, v, causal=False)  # the context still works
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    O, _ = orc.fwd(x["q"], x["k"], x["v"], 1 / math.sqrt(128))
    assert_close_bf16(o, O, "O")


def test_decode_bounded_wait_timeout_is_reported_and_recoverable():
    # two CTAs (B1 H2, one split), each skips its first K/V stage
    x = kvcache_inputs(1, 1, 512, 2, 128, seed=32)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    assert fa.fa_get_device_error() == 0
    fa.fa_debug_set_fault(2, 50_000_000)
    try:
        fa.forward_kvcache(q, k, v, causal=True, num_splits=1)
        code = fa.fa_get_device_error()
    finally:
        fa.fa_debug_set_fault(0, 0)
    assert code == -8
    assert fa.fa_get_device_error() == 0
    o, _ = fa.forward_kvcache(q, k, v, causal=True, num_splits=1)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    O, _ = orc.fwd_kvcache(x["q"], x["k"], x["v"], 1 / math.sqrt(128), causal=True)
    assert_close_bf16(o, O, "O")
