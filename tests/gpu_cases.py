"""Builders shared by the GPU parity tests: seeded inputs -> device cache via
tpa_cache_append (the product path), with NaN in every slot past a
sequence's length."""
from __future__ import annotations

import numpy as np
import torch

from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T

DEV = "cuda"
TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def build_decode_cache(w: S.DecodeWorkload, batch=None, length=None, min_length=None, lengths=None,
                       nan_tail=True):
    if lengths is not None:
        min_length = 0          # explicit lengths replace the drawn ones
    x = S.decode_inputs(w, batch=batch, length=length, min_length=min_length)
    B, cap = x["a_k"].shape[:2]
    if lengths is not None:
        x["lengths"] = torch.tensor(lengths, dtype=torch.int32)
        x["q_pos"] = x["lengths"].clone()
    dt = TORCH_DTYPE[w.dtype]
    cache = T.TpaCache.allocate(B, cap, w.heads, w.head_dim, w.r_k, w.r_v, dtype=dt, rope_base=w.rope_base,
                                fill=float("nan"))
    T.tpa_cache_append(cache, x["positions"].to(DEV), x["a_k"].to(DEV), x["b_k"].to(DEV), x["a_v"].to(DEV),
                       x["b_v"].to(DEV))
    cache.seq_lens.copy_(x["lengths"].to(DEV))
    if nan_tail:
        for b in range(B):
            L = int(x["lengths"][b])
            for plane in (cache.a_k, cache.b_k, cache.a_v, cache.b_v):
                plane[b, L:] = float("nan")
    q = x["q"].to(DEV)
    q_pos = x["q_pos"].to(DEV)
    return cache, x, q, q_pos


def readback(cache: T.TpaCache, batches=None):
    sel = slice(None) if batches is None else list(batches)
    return {k: getattr(cache, k)[sel].double().cpu().numpy() for k in ("a_k", "b_k", "a_v", "b_v")}
