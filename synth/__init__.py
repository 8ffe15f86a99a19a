"""Seeded synthetic inputs for the TurboQuant-style KV-cache path.

This module is shared by the CPU oracle, the tests and the benchmark.  It draws
numbers and nothing else: it holds none of the codec's arithmetic (no
normalisation, rotation, codebook, quantiser or sketch).  Every array is a pure
function of (config, data seed, tensor name, slab, token block), so any slice of
a full-size workload can be regenerated on its own, which is how the oracle
checks sampled outputs of the full-size runs.

Workload shapes and distributions (the pages give the shapes only; the numeric
recipe below is this project's reading of them):

* Llama-3.1-8B-shaped decode layer (TurboQuant blog relay, LongBench on
  Llama-3.1-8B-Instruct): batch 8, 32 query heads, 8 KV heads, head_dim 128,
  context 32768.
* long context: batch 1, 8 KV heads, 32 query heads, context 131072.
* ESM-2-650M-shaped prefill (TurboESM, "Resumo tecnico" section 4): batch 4,
  20 heads, head_dim 64, 4096 tokens, keys after RoPE (theta = 10000).
* K and V entries are iid Student-t with 3 degrees of freedom, and 1% of the
  layer's (KV head, channel) pairs (at least one) are multiplied by 100: the
  TurboQuant news page ("Implicacoes praticas") reports that the top 1% of KV
  values of LLaMA-2-7B reach 100x the median.
* queries are iid N(0, 1); the tiny case uses fp32 N(0, 1) keys with two
  channels scaled by 50.
* vector search: a 256-component Gaussian mixture in d = 1536 (centres
  N(0, I), spread 0.5), rows unit-normalised.

bf16 tensors are produced by rounding the fp32 draw to nearest-even (torch's
``.to(torch.bfloat16)``); the oracle then reads those bf16 values exactly.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import numpy as np
import torch

DATA_SEED = 1        # seed of the synthetic data
CODEC_SEED = 0       # seed of the codec's rotation signs and sketch matrix
TOKEN_BLOCK = 4096   # tokens per independently seeded block

_TENSOR_ID = {"K": 11, "V": 12, "Q": 13, "X": 14, "XQ": 15, "CENTRES": 16}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtypes and codec settings."""

    name: str
    B: int
    Hq: int
    Hkv: int
    T: int
    d: int
    dtype: str                     # "f32" or "bf16" for K/V/Q
    k_bits: Tuple[int, ...]        # one entry per segment (1 or 2 segments)
    k_m: int                       # QJL rows for keys
    v_bits: Tuple[int, ...] = ()   # empty: no values
    v_m: int = 0
    outlier_scale: float = 100.0
    n_outliers: Optional[int] = None   # None: 1% of Hkv*d, rounded, >= 1
    student_t: bool = True             # False: N(0, 1) keys (tiny case)
    rope: bool = False                 # RoPE on keys (prefill case)
    rope_theta: float = 10000.0
    data_seed: int = DATA_SEED
    codec_seed: int = CODEC_SEED

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def n_keys(self) -> int:
        return self.B * self.Hkv * self.T

    def outlier_count(self) -> int:
        if self.n_outliers is not None:
            return self.n_outliers
        return max(1, int(round(0.01 * self.Hkv * self.d)))


WORKLOADS = {
    # 1 head, 4096 fp32 keys, 16 queries; 2-bit Lloyd-Max + 1-bit QJL, m = 128
    "tiny": Workload("tiny", B=1, Hq=16, Hkv=1, T=4096, d=128, dtype="f32",
                     k_bits=(2,), k_m=128, outlier_scale=50.0, n_outliers=2,
                     student_t=False),
    # Llama-3.1-8B-shaped decode layer, 32k context
    "llama8b_decode": Workload("llama8b_decode", B=8, Hq=32, Hkv=8, T=32768,
                               d=128, dtype="bf16", k_bits=(3,), k_m=128,
                               v_bits=(4,), v_m=0),
    # long context, keys split 2 + 3 bits over coordinate halves, m = 64
    "longctx": Workload("longctx", B=1, Hq=32, Hkv=8, T=131072, d=128,
                        dtype="bf16", k_bits=(2, 3), k_m=64),
    # ESM-2-650M-shaped prefill: K (after RoPE) and V, 2 bits + QJL m = 64
    "esm_prefill": Workload("esm_prefill", B=4, Hq=20, Hkv=20, T=4096, d=64,
                            dtype="bf16", k_bits=(2,), k_m=64, v_bits=(2,),
                            v_m=64, rope=True),
}


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(k) & 0xFFFFFFFF for k in key]))


def outlier_channels(w: Workload, which: str) -> np.ndarray:
    """(KV head, channel) pairs scaled by ``outlier_scale``; shape [n, 2]."""
    n = w.outlier_count()
    flat = _rng(w.data_seed, _TENSOR_ID[which], 0xC4).choice(w.Hkv * w.d, size=n, replace=False)
    flat = np.sort(flat)
    return np.stack([flat // w.d, flat % w.d], axis=1)


def rope_rotate_half(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half convention: channel pairs (i, i + d/2)
    rotated by angle pos * theta^(-2i/d).  Works in the dtype of ``x``."""
    d = x.shape[-1]
    half = d // 2
    inv = theta ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = positions.astype(np.float64)[:, None] * inv[None, :]
    c = np.cos(ang).astype(x.dtype)
    s = np.sin(ang).astype(x.dtype)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _kv_block_f32(w: Workload, which: str, b: int, h: int, blk: int) -> np.ndarray:
    t0 = blk * TOKEN_BLOCK
    nt = min(TOKEN_BLOCK, w.T - t0)
    rng = _rng(w.data_seed, _TENSOR_ID[which], b, h, blk)
    if w.student_t:
        x = rng.standard_t(3, size=(nt, w.d))
    else:
        x = rng.standard_normal(size=(nt, w.d))
    x = x.astype(np.float32)
    ch = outlier_channels(w, which)
    for hh, c in ch:
        if hh == h:
            x[:, c] *= np.float32(w.outlier_scale)
    if w.rope and which == "K":
        x = rope_rotate_half(x, np.arange(t0, t0 + nt), w.rope_theta).astype(np.float32)
    return x


def kv_slab(w: Workload, which: str, b: int, h: int, t0: int = 0, t1: Optional[int] = None) -> torch.Tensor:
    """Rows [t0, t1) of the (b, h) slab of K or V, as a CPU tensor in the
    workload's dtype (bf16 values are the fp32 draw rounded to nearest-even)."""
    if t1 is None:
        t1 = w.T
    out = []
    for blk in range(t0 // TOKEN_BLOCK, (t1 - 1) // TOKEN_BLOCK + 1):
        base = blk * TOKEN_BLOCK
        x = _kv_block_f32(w, which, b, h, blk)
        lo = max(t0, base) - base
        hi = min(t1, base + x.shape[0]) - base
        out.append(x[lo:hi])
    x = torch.from_numpy(np.ascontiguousarray(np.concatenate(out, axis=0)))
    return x.to(torch.bfloat16) if w.dtype == "bf16" else x


def kv_full(w: Workload, which: str) -> torch.Tensor:
    """Whole K or V as a contiguous CPU tensor [B, Hkv, T, d]."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = torch.empty((w.B, w.Hkv, w.T, w.d), dtype=dt)
    for b in range(w.B):
        for h in range(w.Hkv):
            out[b, h] = kv_slab(w, which, b, h)
    return out


def queries(w: Workload) -> torch.Tensor:
    """Decode queries [B, Hq, d], iid N(0, 1) in the workload's dtype."""
    x = _rng(w.data_seed, _TENSOR_ID["Q"]).standard_normal(size=(w.B, w.Hq, w.d)).astype(np.float32)
    x = torch.from_numpy(x)
    return x.to(torch.bfloat16) if w.dtype == "bf16" else x


def gaussian_rows(seed: int, n: int, d: int, dtype=torch.float32) -> torch.Tensor:
    """n iid N(0, 1) rows of length d (small ad-hoc test inputs)."""
    x = torch.from_numpy(_rng(seed, _TENSOR_ID["X"], n, d).standard_normal(size=(n, d)).astype(np.float32))
    return x.to(dtype)


def heavy_rows(seed: int, n: int, d: int, n_out: int = 1, scale: float = 100.0,
               dtype=torch.bfloat16) -> torch.Tensor:
    """n Student-t(3) rows of length d with ``n_out`` channels scaled by ``scale``."""
    rng = _rng(seed, _TENSOR_ID["X"], n, d, 7)
    x = rng.standard_t(3, size=(n, d)).astype(np.float32)
    ch = rng.choice(d, size=n_out, replace=False)
    x[:, ch] *= np.float32(scale)
    return torch.from_numpy(x).to(dtype)


# ---------------------------------------------------------------- vector search
@dataclasses.dataclass(frozen=True)
class SearchWorkload:
    name: str = "vsearch"
    n: int = 1_000_000
    nq: int = 1024
    d: int = 1536
    clusters: int = 256
    spread: float = 0.5
    bits: Tuple[int, ...] = (3,)
    m: int = 256
    k: int = 10
    data_seed: int = DATA_SEED
    codec_seed: int = CODEC_SEED
    row_block: int = 16384


VSEARCH = SearchWorkload()


def search_centres(w: SearchWorkload) -> np.ndarray:
    return _rng(w.data_seed, _TENSOR_ID["CENTRES"]).standard_normal(size=(w.clusters, w.d)).astype(np.float32)


def _mixture_rows(w: SearchWorkload, rng: np.random.Generator, n: int) -> np.ndarray:
    c = search_centres(w)
    lab = rng.integers(0, w.clusters, size=n)
    x = c[lab] + np.float32(w.spread) * rng.standard_normal(size=(n, w.d)).astype(np.float32)
    nrm = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=1, keepdims=True))
    return (x / nrm).astype(np.float32)


def search_rows(w: SearchWorkload, r0: int, r1: int) -> torch.Tensor:
    """Database rows [r0, r1) (fp32, unit norm)."""
    out = []
    for blk in range(r0 // w.row_block, (r1 - 1) // w.row_block + 1):
        base = blk * w.row_block
        nb = min(w.row_block, w.n - base)
        x = _mixture_rows(w, _rng(w.data_seed, _TENSOR_ID["X"], blk), nb)
        lo = max(r0, base) - base
        hi = min(r1, base + nb) - base
        out.append(x[lo:hi])
    return torch.from_numpy(np.ascontiguousarray(np.concatenate(out, axis=0)))


def search_queries(w: SearchWorkload) -> torch.Tensor:
    return torch.from_numpy(_mixture_rows(w, _rng(w.data_seed, _TENSOR_ID["XQ"]), w.nq))


def sample_indices(seed: int, n: int, k: int) -> np.ndarray:
    """k distinct sorted indices in [0, n) (which outputs a full-size check samples)."""
    k = min(k, n)
    return np.sort(_rng(seed, 0x5A, n, k).choice(n, size=k, replace=False))
