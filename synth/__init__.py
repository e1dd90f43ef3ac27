"""Seeded synthetic inputs for TurboQuant encode, scoring and decode attention.

This module holds random draws and reshaping only: no quantization, rotation,
codebook or estimator arithmetic lives here.  It serves both the CPU oracle
(``oracle/``) and the CUDA library (``vector_compression_b200``); neither of
those imports the other.

Two kinds of draws:

* ``method_draws`` -- the random quantities the method itself draws once and
  shares between encoder and decoder: the Hadamard sign flips D, the QJL
  Gaussian matrix S, and the Gaussian matrix G whose QR factor is the dense
  rotation.  They are passed to both sides as inputs.  S is drawn standard
  normal and rounded to the nearest fp16 value, so that it is exactly
  representable on the tensor-core path.
* workload tensors -- vectors, KV caches and queries shaped like the pages'
  workloads (KV caches of Qwen2.5-3B / Llama-3.1-8B shape, a 1536-d embedding
  database, a long-context head_dim-192 cache), with seeded outlier channels
  and per-channel lognormal scales.  Real model caches, weights and datasets
  are not used; these synthetic tensors stand in for them.

Everything is a pure function of its seed.  Workload tensors are generated
with ``torch`` on the requested device (so large caches are produced directly
in HBM); the per-(layer, head) channel choices come from numpy so they do not
depend on the device.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "next_pow2",
    "method_draws",
    "outlier_plan",
    "gaussian_vectors",
    "kv_cache",
    "decode_queries",
    "KVConfig",
    "KV_CONFIGS",
    "RETRIEVAL",
    "TINY",
]


def next_pow2(d: int) -> int:
    p = 1
    while p < d:
        p *= 2
    return p


def method_draws(d: int, m: int, seed: int, *, dense: bool = False, stream: int = 0) -> dict:
    """Random draws the method makes once per (quantizer, seed).

    Returns ``signs`` (int8 +-1, length d_pad), ``S`` (float32 [m, d_pad],
    standard normal rounded to fp16) and, when ``dense``, ``G`` (float64
    [d, d] standard normal; its QR factor is the rotation).  ``stream``
    separates independent quantizers (e.g. keys and values) under one seed.
    """
    d_pad = d if dense else next_pow2(d)
    rng = np.random.default_rng([seed, stream, 0x7151])
    signs = np.where(rng.integers(0, 2, size=d_pad) == 0, 1, -1).astype(np.int8)
    S = rng.standard_normal((m, d_pad)).astype(np.float16).astype(np.float32)
    out = {"d": d, "d_pad": d_pad, "m": m, "signs": signs, "S": S, "G": None}
    if dense:
        out["G"] = rng.standard_normal((d, d))
    return out


def outlier_plan(seed: int, n_groups: int, d: int, n_outliers: int, lognormal: bool):
    """Per-group channel scale vectors (numpy float64 [n_groups, d]).

    Each group (a (layer, kv-head) pair, or the whole set for a flat vector
    set) gets ``n_outliers`` channels chosen without replacement and, when
    ``lognormal``, per-channel lognormal(0, 1) scales.  The outlier factor is
    applied by the caller-specific multiplier returned alongside.
    """
    rng = np.random.default_rng([seed, 0x0D71])
    scales = np.ones((n_groups, d))
    chans = np.zeros((n_groups, n_outliers), dtype=np.int64)
    for g in range(n_groups):
        if lognormal:
            scales[g] = rng.lognormal(0.0, 1.0, size=d)
        if n_outliers:
            chans[g] = rng.choice(d, size=n_outliers, replace=False)
    return scales, chans


def _torch():
    import torch

    return torch


def _gen(device, seed):
    torch = _torch()
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def gaussian_vectors(n: int, d: int, *, seed: int, dtype="float32", device="cpu",
                     n_outliers: int = 0, outlier_scale: float = 1.0,
                     normalize: bool = False):
    """N(0,1) vectors [n, d] with seeded outlier channels (flat vector set).

    ``normalize`` L2-normalizes each row after scaling (the embedding
    database of the retrieval workload).  Returns a torch tensor.
    """
    torch = _torch()
    scales, chans = outlier_plan(seed, 1, d, n_outliers, lognormal=False)
    mult = scales[0].copy()
    mult[chans[0]] *= outlier_scale
    x = torch.randn((n, d), generator=_gen(device, seed * 1000003 + 17), device=device,
                    dtype=torch.float32)
    x *= torch.as_tensor(mult, dtype=torch.float32, device=device)
    if normalize:
        x = x / x.norm(dim=1, keepdim=True).clamp_min(1e-30)
    return x.to(getattr(torch, dtype))


@dataclasses.dataclass(frozen=True)
class KVConfig:
    """Shape and value recipe of one synthetic KV-cache workload."""

    name: str
    layers: int
    batch: int
    kv_heads: int
    q_heads: int
    head_dim: int
    seq: int
    dtype: str
    key_bits: int
    value_bits: int
    seed: int
    key_lognormal: bool
    key_outliers: int
    key_outlier_scale: float
    value_lognormal: bool
    value_outliers: int
    value_outlier_scale: float

    @property
    def d_pad(self) -> int:
        return next_pow2(self.head_dim)

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    def with_bits(self, b: int) -> "KVConfig":
        return dataclasses.replace(self, key_bits=b, value_bits=b, name=f"{self.name.rsplit('_b', 1)[0]}_b{b}")

    def scaled(self, **kw) -> "KVConfig":
        return dataclasses.replace(self, **kw)


KV_CONFIGS = {
    # Qwen2.5-3B-shaped cache, 8K context (36 layers, 2 KV heads, head_dim 128,
    # bf16); keys N(0,1) x per-channel lognormal(0,1) with 3 outlier channels
    # x15 per head; values N(0,1); 16 query heads (GQA 8:1).
    "qwen2.5-3b_8k_b3": KVConfig("qwen2.5-3b_8k_b3", 36, 1, 2, 16, 128, 8192, "bfloat16", 3, 3, 2,
                                 True, 3, 15.0, False, 0, 1.0),
    # Llama-3.1-8B-shaped cache (32 layers, batch 4, 8 KV heads, head_dim
    # 128, seq 32768, fp16); keys and values N(0,1) with 4 outlier channels
    # x20 per head; 32 query heads (GQA 4:1).
    "llama3.1-8b_32k_b3": KVConfig("llama3.1-8b_32k_b3", 32, 4, 8, 32, 128, 32768, "float16", 3, 3, 3,
                                   False, 4, 20.0, False, 4, 20.0),
    # Long-context cache with head_dim 192 (padded to a 256-point Hadamard),
    # batch 1, 8 KV heads, seq 131072, fp16; keys and values N(0,1) x
    # per-channel lognormal scales; 32 query heads; 4 bits.
    "longctx-d192_128k_b4": KVConfig("longctx-d192_128k_b4", 1, 1, 8, 32, 192, 131072, "float16", 4, 4, 5,
                                     True, 0, 1.0, True, 0, 1.0),
}

# Tiny set: 4096 fp32 vectors, d=128, N(0,1) with 4 outlier channels x20;
# 64 N(0,1) queries; Q_prod at 3 bits with m=128; seed 0.
TINY = dict(n=4096, d=128, n_queries=64, bits=3, m=128, seed=0, n_outliers=4, outlier_scale=20.0)

# Retrieval: 1,000,000 unit vectors of d=1536 (N(0,1), 8 outlier channels
# x10, then L2-normalized), 1024 unit queries, dense rotation, Q_prod at 2
# and 4 bits, top-10.
RETRIEVAL = dict(n=1_000_000, d=1536, n_queries=1024, bits=(2, 4), m=1536, seed=4,
                 n_outliers=8, outlier_scale=10.0, topk=10)


def _group_multipliers(cfg: KVConfig, which: str):
    lognormal = cfg.key_lognormal if which == "k" else cfg.value_lognormal
    n_out = cfg.key_outliers if which == "k" else cfg.value_outliers
    factor = cfg.key_outlier_scale if which == "k" else cfg.value_outlier_scale
    scales, chans = outlier_plan(cfg.seed * 7 + (1 if which == "k" else 2),
                                 cfg.layers * cfg.kv_heads, cfg.head_dim, n_out, lognormal)
    for g in range(scales.shape[0]):
        scales[g, chans[g]] *= factor
    # [layers, kv_heads, d]
    return scales.reshape(cfg.layers, cfg.kv_heads, cfg.head_dim)


def kv_cache(cfg: KVConfig, *, device="cpu", layers: Optional[range] = None, which: str = "kv"):
    """Synthetic K and V caches, each [layers, batch, kv_heads, seq, head_dim].

    ``layers`` selects a subset of layer indices (each layer is generated from
    its own seed, so a subset equals the same slice of the full cache).
    Returns (K, V); an entry not asked for in ``which`` is None.
    """
    torch = _torch()
    layers = range(cfg.layers) if layers is None else layers
    dt = getattr(torch, cfg.dtype)
    out = {}
    for w in ("k", "v"):
        if w not in which:
            out[w] = None
            continue
        mult = torch.as_tensor(_group_multipliers(cfg, w), dtype=torch.float32, device=device)
        t = torch.empty((len(layers), cfg.batch, cfg.kv_heads, cfg.seq, cfg.head_dim), dtype=dt,
                        device=device)
        for i, l in enumerate(layers):
            g = _gen(device, (cfg.seed * 1009 + l) * 4 + (1 if w == "k" else 2))
            x = torch.randn((cfg.batch, cfg.kv_heads, cfg.seq, cfg.head_dim), generator=g,
                            device=device, dtype=torch.float32)
            x *= mult[l][None, :, None, :]
            t[i] = x.to(dt)
            del x
        out[w] = t
    return out["k"], out["v"]


def decode_queries(cfg: KVConfig, *, device="cpu", layers: Optional[range] = None):
    """Single-token decode queries [layers, batch, q_heads, head_dim], N(0,1) fp32."""
    torch = _torch()
    layers = range(cfg.layers) if layers is None else layers
    q = torch.empty((len(layers), cfg.batch, cfg.q_heads, cfg.head_dim), dtype=torch.float32,
                    device=device)
    for i, l in enumerate(layers):
        g = _gen(device, (cfg.seed * 1009 + l) * 4 + 3)
        q[i] = torch.randn((cfg.batch, cfg.q_heads, cfg.head_dim), generator=g, device=device,
                           dtype=torch.float32)
    return q


def softmax_scale(head_dim: int) -> float:
    """Scaled dot-product attention scale 1/sqrt(head_dim) used by the workloads."""
    return 1.0 / math.sqrt(head_dim)
