"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers; it holds none of the attention
arithmetic, so the CUDA path and the CPU oracle can both be fed from it
without sharing any of the method's code.

Recipe (the pages fix only "i.i.d. N(0,1) bf16, seed s"):
  * fixed length: ``g = torch.Generator('cpu').manual_seed(seed)``, then
    ``torch.randn([B, N, H, d], dtype=float32, generator=g).to(bfloat16)``
    for Q, K, V and (backward only) dO, drawn in that order;
  * packed variable length: sequence lengths are
    ``torch.randint(lo, hi + 1, (nseq,), generator=g)`` from the same seeded
    generator, then Q, K, V (and dO) with shape ``[T, H, d]``,
    ``T = sum(lengths)``; ``cu_seqlens`` is the int32 prefix sum with a
    leading 0;
  * queries against longer cached keys/values: as above, with Q drawn over
    the query rows and K, V over the key rows (fixed ``[B, Nq, H, d]`` and
    ``[B, Nk, H, d]``; packed ``[Tq, H, d]`` and ``[Tk, H, d]`` with
    ``cu_seqlens_q`` / ``cu_seqlens_k`` from explicit per-sequence lengths);
  * decode: Q ``[B, Nq, H, d]``, a padded cache K, V ``[B, Nk, H, d]``, then
    the used cache rows per sequence from ``torch.randint`` (``kvcache_inputs``).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


def fixed_inputs(B: int, N: int, H: int, d: int, seed: int, with_dout: bool = False):
    g = torch.Generator("cpu").manual_seed(seed)
    names = ["q", "k", "v"] + (["dout"] if with_dout else [])
    return {n: torch.randn([B, N, H, d], dtype=torch.float32, generator=g).to(torch.bfloat16)
            for n in names}


def varlen_lengths(nseq: int, lo: int, hi: int, g: torch.Generator):
    return torch.randint(lo, hi + 1, (nseq,), generator=g, dtype=torch.int64)


def varlen_inputs(nseq: int, lo: int, hi: int, H: int, d: int, seed: int,
                  with_dout: bool = False, lengths=None):
    """Packed inputs.  ``lengths`` overrides the random lengths (the random
    stream is then used for the tensors only)."""
    g = torch.Generator("cpu").manual_seed(seed)
    if lengths is None:
        lens = varlen_lengths(nseq, lo, hi, g)
    else:
        lens = torch.as_tensor(lengths, dtype=torch.int64)
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    T = int(cu[-1])
    names = ["q", "k", "v"] + (["dout"] if with_dout else [])
    out = {n: torch.randn([T, H, d], dtype=torch.float32, generator=g).to(torch.bfloat16)
           for n in names}
    out["cu_seqlens"] = cu
    out["max_seqlen"] = int(lens.max()) if len(lens) else 0
    return out


def kv_inputs(B: int, Nq: int, Nk: int, H: int, d: int, seed: int):
    g = torch.Generator("cpu").manual_seed(seed)
    shapes = {"q": [B, Nq, H, d], "k": [B, Nk, H, d], "v": [B, Nk, H, d]}
    return {n: torch.randn(shp, dtype=torch.float32, generator=g).to(torch.bfloat16)
            for n, shp in shapes.items()}


def varlen_kv_inputs(lens_q, lens_k, H: int, d: int, seed: int):
    """Packed queries and keys/values with the given per-sequence lengths."""
    g = torch.Generator("cpu").manual_seed(seed)
    out = {}
    for name, lens in (("q", lens_q), ("k", lens_k)):
        cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.as_tensor(lens, dtype=torch.int64), 0).to(torch.int32)
        out["cu_seqlens_" + name] = cu
    Tq, Tk = int(out["cu_seqlens_q"][-1]), int(out["cu_seqlens_k"][-1])
    for name, T in (("q", Tq), ("k", Tk), ("v", Tk)):
        out[name] = torch.randn([T, H, d], dtype=torch.float32, generator=g).to(torch.bfloat16)
    return out


def fp8_signs(seed: int, d: int = 128):
    """The random sign vector of the FP8 path's rotation: d entries of +-1
    from ``torch.randint(0, 2, (d,))`` of a generator seeded with ``seed``."""
    g = torch.Generator("cpu").manual_seed(seed)
    return (torch.randint(0, 2, (d,), generator=g) * 2 - 1).to(torch.float32)


def kvcache_inputs(B: int, Nq: int, Nk: int, H: int, d: int, seed: int, lens=None):
    """Decode inputs: q [B, Nq, H, d], a padded cache k, v [B, Nk, H, d] and
    the used cache rows per sequence (``lens`` = (lo, hi) draws them with
    ``torch.randint(lo, hi + 1, (B,))`` after the tensors; a list fixes them;
    None leaves all Nk rows in use and ``seqlens_k`` None)."""
    g = torch.Generator("cpu").manual_seed(seed)
    shapes = {"q": [B, Nq, H, d], "k": [B, Nk, H, d], "v": [B, Nk, H, d]}
    out = {n: torch.randn(shp, dtype=torch.float32, generator=g).to(torch.bfloat16)
           for n, shp in shapes.items()}
    if lens is None:
        out["seqlens_k"] = None
    elif isinstance(lens, tuple):
        out["seqlens_k"] = torch.randint(lens[0], lens[1] + 1, (B,), generator=g,
                                         dtype=torch.int64).to(torch.int32)
    else:
        out["seqlens_k"] = torch.as_tensor(lens, dtype=torch.int32)
    return out


@dataclass(frozen=True)
class Workload:
    """One named workload: shapes, seed and mask of a parity or bench case."""
    name: str
    B: int
    H: int
    N: int
    d: int
    seed: int
    causal: bool = False
    window: int = 0
    varlen: tuple = field(default=None)   # (nseq, lo, hi) for packed inputs
    backward: bool = False
    Nk: int = 0                           # > 0: keys/values per sequence (cached-KV prefill)
    cache_lens: tuple = None              # (lo, hi): decode against a padded cache of Nk rows

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def make(self):
        if self.cache_lens is not None:
            return kvcache_inputs(self.B, self.N, self.Nk, self.H, self.d, self.seed,
                                  lens=self.cache_lens)
        if self.Nk > 0:
            return kv_inputs(self.B, self.N, self.Nk, self.H, self.d, self.seed)
        if self.varlen is not None:
            nseq, lo, hi = self.varlen
            return varlen_inputs(nseq, lo, hi, self.H, self.d, self.seed, with_dout=self.backward)
        return fixed_inputs(self.B, self.N, self.H, self.d, self.seed, with_dout=self.backward)


# The five workloads of the parity contract.  Shapes and seeds are the ones
# the long-sequence training and long-prompt prefill scenarios are measured on.
WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=1, N=128, d=64, seed=0),
    "train": Workload("train", B=4, H=16, N=2048, d=128, seed=1),
    "train_causal": Workload("train_causal", B=4, H=16, N=2048, d=128, seed=1, causal=True),
    "prefill_b2_causal": Workload("prefill_b2_causal", B=2, H=16, N=8192, d=128, seed=2,
                                  causal=True),
    "prefill_b4_causal": Workload("prefill_b4_causal", B=4, H=16, N=8192, d=128, seed=2,
                                  causal=True),
    "prefill_b4": Workload("prefill_b4", B=4, H=16, N=8192, d=128, seed=2),
    "varlen_causal": Workload("varlen_causal", B=16, H=32, N=4096, d=128, seed=3, causal=True,
                              varlen=(16, 128, 4096)),
    "varlen_window": Workload("varlen_window", B=16, H=32, N=4096, d=128, seed=3, causal=True,
                              window=1024, varlen=(16, 128, 4096)),
    "bwd_causal": Workload("bwd_causal", B=2, H=16, N=4096, d=128, seed=4, causal=True,
                           backward=True),
    # one new token per sequence against caches of 4096..8192 tokens
    # (N is the query count, Nk the cache capacity)
    "decode": Workload("decode", B=16, H=16, N=1, d=128, seed=6, causal=True, Nk=8192,
                       cache_lens=(4096, 8192)),
    # a 2048-token prompt chunk after 6144 cached tokens
    "prefill_kv_causal": Workload("prefill_kv_causal", B=4, H=16, N=2048, d=128, seed=5,
                                  causal=True, Nk=8192),
}
