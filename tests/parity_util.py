"""Shared helpers of the GPU parity tests: tolerance checks and oracle drivers.

Tolerance reading: for every output row (sequence, [query,] head) the largest
absolute difference over the head_dim features must stay within tol times the
largest absolute oracle value of that row; tol = 1e-5 for fp32 factors and
2e-3 for bf16 factors (fp32 accumulation in both).
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.tpa_oracle as O

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-3}


def row_errors(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    num = np.abs(got - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), np.where(num == 0, 0.0, np.inf))


def assert_rows_close(got, ref, tol, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    e = row_errors(got, ref)
    worst = float(e.max()) if e.size else 0.0
    assert worst <= tol, f"{what}: worst row error {worst:.3e} > {tol:.1e} at {np.unravel_index(np.argmax(e), e.shape)}"
    return worst


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def oracle_decode_rows(cache_cpu: dict, q, q_pos, lengths, scale, base, batches=None, heads=None):
    """Oracle decode from a cache read back from the GPU (B_K already rotated).

    cache_cpu: float64 arrays a_k [B,cap,R,h], b_k, a_v, b_v.  Returns
    [len(batches), len(heads), d].
    """
    B = q.shape[0]
    batches = range(B) if batches is None else batches
    out = []
    for b in batches:
        L = int(lengths[b])
        sel = slice(None) if heads is None else list(heads)
        ak = cache_cpu["a_k"][b, :L][:, :, sel]
        av = cache_cpu["a_v"][b, :L][:, :, sel]
        o = O.decode_attention(ak, cache_cpu["b_k"][b, :L], av, cache_cpu["b_v"][b, :L], q[b][sel],
                               float(q_pos[b]), scale, base)
        out.append(o)
    return np.stack(out)


def default_scale(d):
    return 1.0 / math.sqrt(d)
