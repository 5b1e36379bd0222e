"""Seeded synthetic inputs shaped like the decode workloads.

This module draws random numbers and nothing else: it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can be fed
from it.  Every tensor comes from its own numpy PCG64 stream seeded by
(seed, tensor id[, sequence]), so any tensor can be regenerated alone and the
same values appear on every machine.

Value recipe (the workload descriptions): queries, RoPE keys and latents are
N(0, 1); weights are N(0, 0.02^2); hidden states N(0, 1); ragged lengths are
uniform integers in [1, N].  A latent row of 512 N(0,1) entries has unit RMS
in expectation, which is how "RMS-normalised N(0,1) latent rows" is read.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

# Tensor ids for the per-tensor streams.
TID = {"q_nope": 1, "q_pe": 2, "W_UK": 3, "W_UV": 4, "cache": 5, "seqlens": 6,
       "h": 7, "W_DKV": 8, "gamma": 9, "partials_o": 10, "partials_lse": 11,
       "fp8_codes": 12, "fp8_scale": 13, "fp8_rope": 14}


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d_c: int
    d_r: int
    d_nope: int
    d_v: int
    N: int            # cached tokens per sequence (upper end for ragged lengths)
    dtype: str        # "bf16" | "f32"
    ragged: bool = False
    append: bool = False
    hidden: int = 7168
    w_std: float = 0.02
    rope_base: float = 10000.0
    eps: float = 1e-6
    seed: int = 0

    @property
    def R(self) -> int:
        return self.d_c + self.d_r

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.d_nope + self.d_r)

    @property
    def capacity(self) -> int:
        # One spare row per sequence for the appended token.
        return self.N + 1

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, H=4, d_c=32, d_r=16, d_nope=16, d_v=16, N=64,
                         dtype="f32"),
    "v2lite_bf16": Workload("v2lite_bf16", B=4, H=16, d_c=512, d_r=64, d_nope=128, d_v=128,
                            N=4096, dtype="bf16"),
    "v3_bf16": Workload("v3_bf16", B=32, H=128, d_c=512, d_r=64, d_nope=128, d_v=128, N=8192,
                        dtype="bf16"),
    "longctx_bf16": Workload("longctx_bf16", B=4, H=128, d_c=512, d_r=64, d_nope=128, d_v=128,
                             N=131072, dtype="bf16"),
    "ragged_append_bf16": Workload("ragged_append_bf16", B=64, H=64, d_c=512, d_r=64,
                                   d_nope=128, d_v=128, N=32768, dtype="bf16", ragged=True,
                                   append=True, hidden=7168),
}


def _rng(seed: int, *ids: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), *map(int, ids)]))


def normal(shape, std: float, seed: int, *ids: int) -> np.ndarray:
    """float32 N(0, std^2) array from the stream (seed, *ids)."""
    a = _rng(seed, *ids).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def seqlens(w: Workload) -> np.ndarray:
    """Cached tokens per sequence: all N, or uniform in [1, N] if ragged."""
    if not w.ragged:
        return np.full(w.B, w.N, dtype=np.int32)
    return _rng(w.seed, TID["seqlens"]).integers(1, w.N + 1, size=w.B).astype(np.int32)


def query(w: Workload):
    """(q_nope [B,H,d_nope], q_pe [B,H,d_r]) float32."""
    return (normal((w.B, w.H, w.d_nope), 1.0, w.seed, TID["q_nope"]),
            normal((w.B, w.H, w.d_r), 1.0, w.seed, TID["q_pe"]))


def weights(w: Workload):
    """(W_UK [H,d_nope,d_c], W_UV [H,d_v,d_c]) float32."""
    return (normal((w.H, w.d_nope, w.d_c), w.w_std, w.seed, TID["W_UK"]),
            normal((w.H, w.d_v, w.d_c), w.w_std, w.seed, TID["W_UV"]))


def append_inputs(w: Workload):
    """(h [B,hidden], W_DKV [d_c+d_r, hidden]) float32; gamma is ones."""
    return (normal((w.B, w.hidden), 1.0, w.seed, TID["h"]),
            normal((w.R, w.hidden), w.w_std, w.seed, TID["W_DKV"]))


def cache_rows(w: Workload, b: int, n: int) -> np.ndarray:
    """The first n latent rows [n, d_c + d_r] of sequence b (float32)."""
    return normal((n, w.R), 1.0, w.seed, TID["cache"], b)


def fill_cache(w: Workload, cache, lens, fill_rest: float | None = None):
    """Write rows [0, L_b) of every sequence into a torch tensor
    [B, capacity, R] (any device/dtype; rounding happens in the copy).  Rows
    from L_b on are set to ``fill_rest`` when given (e.g. NaN to show that the
    decode never depends on them)."""
    import torch
    for b in range(w.B):
        L = int(lens[b])
        if L:
            cache[b, :L].copy_(torch.from_numpy(cache_rows(w, b, L)))
        if fill_rest is not None and L < cache.shape[1]:
            cache[b, L:].fill_(fill_rest)
    return cache


def fp8_cache_rows(w: Workload, b: int, n: int):
    """The first n rows of sequence b of an FP8 latent cache, drawn directly
    in the stored format: (codes [n, d_c] uint8, uniform over the 254 finite
    E4M3 bytes, i.e. every byte but 0x7F and 0xFF; exponents k [n] int,
    uniform in [-9, -6], the token's scale being 2^k; RoPE keys [n, d_r]
    float32 N(0, 1))."""
    r = _rng(w.seed, TID["fp8_codes"], b)
    draw = r.integers(0, 254, size=(n, w.d_c))
    codes = np.where(draw >= 0x7F, draw + 1, draw).astype(np.uint8)
    k = _rng(w.seed, TID["fp8_scale"], b).integers(-9, -5, size=n)
    rope = normal((n, w.d_r), 1.0, w.seed, TID["fp8_rope"], b)
    return codes, k, rope


def fill_fp8_cache(w: Workload, cache, scales, lens, fill_rest_byte: int | None = None):
    """Write rows [0, L_b) of every sequence into an FP8 cache: cache [B,
    capacity, d_c + 2 d_r] uint8 (codes, then the RoPE keys' bf16 bytes) and
    scales [B, capacity] float32 (2^k).  Rows from L_b on get
    ``fill_rest_byte`` in every byte and scale 1 when given (0xFF is an E4M3
    NaN code, to show that the decode never depends on them)."""
    import torch
    for b in range(w.B):
        L = int(lens[b])
        if L:
            codes, k, rope = fp8_cache_rows(w, b, L)
            cache[b, :L, :w.d_c].copy_(torch.from_numpy(codes))
            rb = torch.from_numpy(rope).to(torch.bfloat16).view(torch.uint8).reshape(L, 2 * w.d_r)
            cache[b, :L, w.d_c:].copy_(rb)
            scales[b, :L].copy_(torch.from_numpy(np.ldexp(np.ones(L, np.float32), k)))
        if fill_rest_byte is not None and L < cache.shape[1]:
            cache[b, L:].fill_(fill_rest_byte)
            scales[b, L:].fill_(1.0)
    return cache, scales


def partials(B: int, H: int, S: int, D: int, seed: int = 0, empty_frac: float = 0.2):
    """Synthetic split-KV partial results (o [B,H,S,D], lse [B,H,S]) for
    exercising a merge on its own; about ``empty_frac`` of the lse entries
    are -inf (empty chunks)."""
    o = normal((B, H, S, D), 1.0, seed, TID["partials_o"])
    r = _rng(seed, TID["partials_lse"])
    lse = (r.standard_normal(size=(B, H, S)) * 3.0).astype(np.float32)
    lse[r.random(size=(B, H, S)) < empty_frac] = -np.inf
    return o, lse
