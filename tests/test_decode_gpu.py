"""Attention against a padded key/value cache on the GPU: fa_fwd_kvcache
through the C ABI against the float64 oracle's fwd_kvcache -- decode (few
queries per sequence, CUDA-core kernel) and prefill chunks (more than 16
queries, the tensor-core forward), both split along the keys with the
partials merged by a second kernel."""
import math

import numpy as np
import pytest
import torch

import io_aware_exact_21_b200 as fa
from io_aware_exact_21_b200.inputs import WORKLOADS, kvcache_inputs
from oracle import oracle as orc

from helpers import TOL_LSE, assert_close_bf16, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def poison_unused_rows(x):
    """NaN in every cache row past a sequence's used length: the kernel must
    never read them into a result."""
    lens = x["seqlens_k"]
    if lens is None:
        return x
    k, v = x["k"].clone(), x["v"].clone()
    for b, n in enumerate(lens.tolist()):
        k[b, n:] = float("nan")
        v[b, n:] = float("nan")
    return dict(x, k=k, v=v)


def run_decode(x, causal, window, num_splits):
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    lens = x["seqlens_k"]
    o, lse = fa.forward_kvcache(q, k, v, seqlens_k=None if lens is None else lens.to(DEV),
                                causal=causal, window=window, num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    return o, lse


def oracle_decode(x, causal, window):
    d = x["q"].shape[-1]
    return orc.fwd_kvcache(x["q"], x["k"], x["v"], 1 / math.sqrt(d), seqlens_k=x["seqlens_k"],
                           causal=causal, window=window)


def assert_lse_with_empty_rows(got, ref):
    g = to64(got)
    empty = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), empty), "rows without keys differ"
    if (~empty).any():
        err = np.abs(g[~empty] - ref[~empty]).max()
        assert err <= TOL_LSE, "lse: max %.3e" % err


SHAPES = [(1, 1, 1, 1, 128), (2, 1, 63, 2, 128), (3, 1, 64, 2, 64), (2, 2, 65, 3, 128),
          (2, 5, 1000, 2, 128), (1, 16, 300, 2, 64), (4, 1, 4096, 2, 128), (2, 3, 2, 1, 128)]
MASKS = [(False, 0), (True, 0), (True, 1), (True, 100)]


@pytest.mark.parametrize("B,Nq,Nk,H,d", SHAPES)
@pytest.mark.parametrize("causal,window", MASKS)
@pytest.mark.parametrize("num_splits", [1, 3, 0])
def test_decode_elementwise(B, Nq, Nk, H, d, causal, window, num_splits):
    # used cache rows drawn from [0, Nk]: includes empty caches and caches
    # shorter than the query count
    x = kvcache_inputs(B, Nq, Nk, H, d, seed=Nk + 13 * Nq, lens=(0, Nk))
    o, lse = run_decode(poison_unused_rows(x), causal, window, num_splits)
    O, L = oracle_decode(x, causal, window)
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


@pytest.mark.parametrize("num_splits", [1, 2, 5, 32])
def test_decode_full_cache_and_split_counts(num_splits):
    # seqlens_k = None (every row used); split counts up to the limit,
    # including more splits than some sequences have key tiles
    x = kvcache_inputs(3, 2, 2000, 4, 128, seed=5)
    o, lse = run_decode(x, True, 0, num_splits)
    O, L = oracle_decode(x, True, 0)
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


def test_decode_no_cache_rows():
    x = kvcache_inputs(2, 3, 0, 2, 128, seed=1)
    for ns in (1, 4):
        o, lse = run_decode(x, True, 0, ns)
        assert torch.count_nonzero(o) == 0
        assert torch.isneginf(lse).all()


def test_decode_workspace_is_checked():
    x = kvcache_inputs(1, 1, 512, 1, 128, seed=2)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, 1), device=DEV)
    rc = fa.fa_fwd_kvcache(q, k, v, o, lse, 1, 1, 1, 512, 128, 0.1, 1, 0, None, 4, None, 0)
    assert rc == -6


def test_decode_workload_parity():
    # one token per sequence, B16 H16 d128, caches of 4096..8192 rows in a
    # padded 8192-row buffer (unused rows NaN), library-chosen split count
    wl = WORKLOADS["decode"]
    x = wl.make()
    o, lse = run_decode(poison_unused_rows(x), wl.causal, wl.window, 0)
    O, L = oracle_decode(x, wl.causal, wl.window)
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


# ------------------------------------------- prefill chunks (Nq > 16) ---

PREFILL = [(2, 17, 300, 2, 128), (1, 200, 1000, 2, 64), (2, 300, 300, 1, 128),
           (1, 257, 4096, 2, 128), (3, 129, 2000, 1, 128)]


@pytest.mark.parametrize("B,Nq,Nk,H,d", PREFILL)
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 100)])
@pytest.mark.parametrize("num_splits", [1, 2, 5, 0])
def test_prefill_chunk_elementwise(B, Nq, Nk, H, d, causal, window, num_splits):
    # cache lengths drawn from [0, Nk]: includes empty caches and caches
    # shorter than the chunk (its first queries then see no key when causal)
    x = kvcache_inputs(B, Nq, Nk, H, d, seed=Nk + 7 * Nq, lens=(0, Nk))
    o, lse = run_decode(poison_unused_rows(x), causal, window, num_splits)
    O, L = oracle_decode(x, causal, window)
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


def test_prefill_chunk_workload():
    # the cached-KV prefill workload (B4 H16, 2048 queries after 6144 cached
    # keys, d128, causal) through the cache interface: 512 blocks fill the
    # GPU, so the library does not split; same kernel as fa_fwd_kv, so the
    # results agree bit for bit; two heads against the oracle
    wl = WORKLOADS["prefill_kv_causal"]
    x = wl.make()
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    assert fa.fa_fwd_kvcache_num_splits(wl.B, wl.H, wl.N, wl.Nk, wl.d) == 1
    o, lse = fa.forward_kvcache(q, k, v, causal=True)
    o1, lse1 = fa.forward_kv(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert fa.fa_get_device_error() == 0
    assert torch.equal(o, o1) and torch.equal(lse, lse1)
    for s, h in ((0, 3), (2, 11)):
        sl = {n: x[n][s:s + 1, :, h:h + 1] for n in ("q", "k", "v")}
        sl["seqlens_k"] = None
        O, L = oracle_decode(sl, True, 0)
        assert_close_bf16(o[s:s + 1, :, h:h + 1], O, "O")
        assert_lse_with_empty_rows(lse[s:s + 1, h:h + 1], L)


def test_prefill_chunk_few_blocks_split():
    # few blocks (B1 H2, 512 queries: 4 blocks of 256) against 8192 cached
    # keys: the library splits the keys so the blocks spread over the SMs
    x = kvcache_inputs(1, 512, 8192, 2, 128, seed=9, lens=[8000])
    ns = fa.fa_fwd_kvcache_num_splits(1, 2, 512, 8192, 128)
    assert ns > 1
    o, lse = run_decode(poison_unused_rows(x), True, 0, 0)
    O, L = oracle_decode(x, True, 0)
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)


@pytest.mark.parametrize("Nq", [17, 40, 200])
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 50)])
@pytest.mark.parametrize("num_splits", [1, 3])
def test_prefill_chunk_cache_ends(Nq, causal, window, num_splits):
    # used lengths at and around multiples of the 128-key tile, and below one
    # tile; every row past them NaN, in every sequence, so a tile that read a
    # row past its sequence's length (its own padding or the next sequence's
    # first rows) would put NaN into the result
    lens = [0, 1, 17, 127, 128, 129, 255, 256, 300, 383]
    x = kvcache_inputs(len(lens), Nq, 384, 1, 128, seed=31 + Nq, lens=lens)
    o, lse = run_decode(poison_unused_rows(x), causal, window, num_splits)
    O, L = oracle_decode(x, causal, window)
    assert_close_bf16(o, O, "O")
    assert_lse_with_empty_rows(lse, L)
