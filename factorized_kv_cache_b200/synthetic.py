"""Seeded synthetic inputs for the five TPA workloads.

This module is the one piece shared by the CPU oracle side and the CUDA side:
it draws random numbers and rounds them to the storage dtype, and it holds none
of the attention arithmetic (no RoPE, no factor contraction, no softmax).

Random numbers come from NumPy's Philox4x64-10 counter-based bit generator
(``numpy.random.Philox``), one stream per workload seed, drawn in float32 and
rounded once to the storage dtype with round-to-nearest-even.

Distributions (Tensor Product Attention Is All You Need, section
"Tensor product decomposition": per token the cache holds A_K in R^{R_K x h},
B_K in R^{R_K x d_h}, A_V in R^{R_V x h}, B_V in R^{R_V x d_h}):

* decode workloads: A ~ N(0, 1), B ~ N(0, 1/d_h), the query q ~ N(0, 1);
  cached token s sits at position s, the query at position L_b;
* causal prefill: hidden states x ~ N(0, 1) of width 2048 and six projection
  matrices W ~ N(0, 1/2048) whose products x W are the factors A_Q, B_Q, A_K,
  B_K, A_V, B_V of every prompt token (the "contextual factors produced from
  x_t" of the same section).  This product makes inputs; it is not a step of
  the attention path.

Tokens past a sequence's length are filled as well (with draws from the same
stream), so a cache buffer always has defined contents; tests overwrite them
with NaN to check masking.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import numpy as np
import torch

__all__ = [
    "DecodeWorkload",
    "PrefillWorkload",
    "WORKLOADS",
    "rng",
    "to_storage",
    "decode_inputs",
    "prefill_inputs",
]


@dataclass(frozen=True)
class DecodeWorkload:
    """One query token per sequence attending a factorized cache."""

    name: str
    batch: int
    heads: int
    head_dim: int
    r_k: int
    r_v: int
    length: int            # tokens per sequence (the maximum when min_length is set)
    dtype: str             # "f32" or "bf16": storage dtype of factors and query
    seed: int
    min_length: int = 0    # >0: lengths drawn uniformly from [min_length, length]
    rope_base: float = 10000.0
    b_std: float = 0.0     # std of the B factors; 0 means 1/sqrt(d_h)

    @property
    def capacity(self) -> int:
        return self.length

    def replace(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)


@dataclass(frozen=True)
class PrefillWorkload:
    """Causal prefill of T prompt tokens with R_Q-factorized queries."""

    name: str
    batch: int
    tokens: int
    heads: int
    head_dim: int
    r_q: int
    r_k: int
    r_v: int
    hidden: int
    dtype: str
    seed: int
    rope_base: float = 10000.0

    def replace(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # tiny fp32 decode: B=1, h=4, d_h=16, R=1, 64 cached tokens, query at 64, seed 0
    "decode_tiny_f32": DecodeWorkload("decode_tiny_f32", 1, 4, 16, 1, 1, 64, "f32", seed=0),
    # bf16 decode, the 8192 -> 320 elements/token case: B=8, L=8192
    "decode_b8_l8k": DecodeWorkload("decode_b8_l8k", 8, 32, 128, 1, 1, 8192, "bf16", seed=1),
    # bf16 decode, R=2, B=32, lengths uniform in [16384, 32768], capacity 32768
    "decode_b32_var32k": DecodeWorkload(
        "decode_b32_var32k", 32, 32, 128, 2, 2, 32768, "bf16", seed=2, min_length=16384),
    # bf16 causal prefill, B=4, T=4096, R_Q=6, R_K=R_V=2, hidden width 2048
    "prefill_b4_t4k": PrefillWorkload("prefill_b4_t4k", 4, 4096, 32, 128, 6, 2, 2, 2048, "bf16", seed=3),
    # bf16 long-context decode, B=1, R=1, L=524288
    "decode_long_512k": DecodeWorkload("decode_long_512k", 1, 32, 128, 1, 1, 524288, "bf16", seed=4),
}


def rng(seed: int, stream: int = 0) -> np.random.Generator:
    """Philox4x64-10 generator keyed by (seed, stream)."""
    return np.random.Generator(np.random.Philox(key=[seed, stream]))


def to_storage(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Round a float array once to the storage dtype (RNE), as a CPU tensor."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "f32":
        return t
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    raise ValueError(f"unknown dtype {dtype!r}")


def _normal(g: np.random.Generator, shape, std: float) -> np.ndarray:
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def decode_inputs(w: DecodeWorkload, batch: int | None = None, length: int | None = None,
                  min_length: int | None = None) -> dict:
    """Unrotated cache factors, lengths and query for a decode workload.

    Returns CPU tensors in the storage dtype:
      a_k [B, cap, R_K, h], b_k [B, cap, R_K, d_h], a_v [B, cap, R_V, h],
      b_v [B, cap, R_V, d_h], q [B, h, d_h]; int32 tensors lengths [B],
      positions [B, cap] (slot s holds position s) and q_pos [B] (= lengths).
    ``batch``/``length``/``min_length`` shrink the workload (same distributions).
    """
    B = w.batch if batch is None else batch
    cap = w.length if length is None else length
    lo = w.min_length if min_length is None else min_length
    h, d, rk, rv = w.heads, w.head_dim, w.r_k, w.r_v
    g = rng(w.seed)
    if lo > 0:
        lengths = g.integers(lo, cap, size=B, endpoint=True).astype(np.int32)
    else:
        lengths = np.full(B, cap, dtype=np.int32)
    a_k = _normal(g, (B, cap, rk, h), 1.0)
    b_std = w.b_std if w.b_std > 0 else 1.0 / np.sqrt(d)
    b_k = _normal(g, (B, cap, rk, d), b_std)
    a_v = _normal(g, (B, cap, rv, h), 1.0)
    b_v = _normal(g, (B, cap, rv, d), b_std)
    q = _normal(g, (B, h, d), 1.0)
    positions = np.broadcast_to(np.arange(cap, dtype=np.int32), (B, cap)).copy()
    return {
        "a_k": to_storage(a_k, w.dtype),
        "b_k": to_storage(b_k, w.dtype),
        "a_v": to_storage(a_v, w.dtype),
        "b_v": to_storage(b_v, w.dtype),
        "q": to_storage(q, w.dtype),
        "lengths": torch.from_numpy(lengths),
        "positions": torch.from_numpy(positions),
        "q_pos": torch.from_numpy(lengths.copy()),
    }


def prefill_inputs(w: PrefillWorkload, batch: int | None = None, tokens: int | None = None) -> dict:
    """Factors of every prompt token, produced from synthetic hidden states.

    x ~ N(0,1) [B*T, hidden]; W ~ N(0, 1/hidden) [hidden, total] with total =
    R_Q*h + R_Q*d_h + R_K*h + R_K*d_h + R_V*h + R_V*d_h; the factors are x W
    (computed in float64, rounded once to the storage dtype).  Returns CPU
    tensors a_q [B,T,R_Q,h], b_q [B,T,R_Q,d_h] (unrotated), a_k, b_k (unrotated),
    a_v, b_v, and int32 positions [B, T] = 0..T-1 (used by both Q and K/V).
    """
    B = w.batch if batch is None else batch
    T = w.tokens if tokens is None else tokens
    h, d = w.heads, w.head_dim
    widths = [w.r_q * h, w.r_q * d, w.r_k * h, w.r_k * d, w.r_v * h, w.r_v * d]
    total = sum(widths)
    gx = rng(w.seed, 0)
    gw = rng(w.seed, 1)
    x = gx.standard_normal(size=(B * T, w.hidden), dtype=np.float32)
    proj = gw.standard_normal(size=(w.hidden, total), dtype=np.float32)
    proj *= np.float32(1.0 / np.sqrt(w.hidden))
    f = x.astype(np.float64) @ proj.astype(np.float64)
    parts = np.split(f, np.cumsum(widths)[:-1], axis=1)
    shapes = [(w.r_q, h), (w.r_q, d), (w.r_k, h), (w.r_k, d), (w.r_v, h), (w.r_v, d)]
    names = ["a_q", "b_q", "a_k", "b_k", "a_v", "b_v"]
    out = {}
    for name, part, shp in zip(names, parts, shapes):
        out[name] = to_storage(part.reshape(B, T, *shp), w.dtype)
    out["positions"] = torch.from_numpy(
        np.broadcast_to(np.arange(T, dtype=np.int32), (B, T)).copy())
    return out
