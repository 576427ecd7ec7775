"""GPU parity of tpa_prefill_attention (causal, R_Q-factorized queries)."""
import numpy as np
import pytest
import torch

import oracle.tpa_oracle as O
from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T
from tests.gpu_cases import DEV, TORCH_DTYPE
from tests.parity_util import TOL, assert_rows_close, default_scale, f64

pytestmark = pytest.mark.gpu

KERNELS = [T.TPA_KERNEL_SIMT, T.TPA_KERNEL_AUTO]


def _prefill_case(w, batch, tokens, prior=0, nan_fill=True):
    """Cache holding `prior` earlier tokens, then the chunk's own factors appended."""
    x = S.prefill_inputs(w, batch=batch, tokens=prior + tokens)
    dt = TORCH_DTYPE[w.dtype]
    cap = prior + tokens + 9
    cache = T.TpaCache.allocate(batch, cap, w.heads, w.head_dim, w.r_k, w.r_v, dtype=dt, rope_base=w.rope_base,
                                fill=float("nan") if nan_fill else 0.0)
    pos = x["positions"].to(DEV)
    if prior:
        T.tpa_cache_append(cache, pos[:, :prior].contiguous(), *(x[k][:, :prior].contiguous().to(DEV)
                                                                 for k in ("a_k", "b_k", "a_v", "b_v")))
    T.tpa_cache_append(cache, pos[:, prior:].contiguous(), *(x[k][:, prior:].contiguous().to(DEV)
                                                             for k in ("a_k", "b_k", "a_v", "b_v")))
    a_q = x["a_q"][:, prior:].contiguous().to(DEV)
    b_q = x["b_q"][:, prior:].contiguous().to(DEV)
    q_pos = pos[:, prior:].contiguous()
    return cache, x, a_q, b_q, q_pos


def _oracle(w, cache, x, prior, tokens, b, rows=None, heads=None, end_to_end=False):
    L = prior + tokens
    scale = default_scale(w.head_dim)
    sel = slice(None) if heads is None else list(heads)
    if end_to_end:   # the oracle's own RoPE, stored in the cache dtype as the append stores it
        bk = O.append_rope(f64(x["b_k"][b, :L]), np.arange(L), w.rope_base, storage=w.dtype)
    else:
        bk = f64(cache.b_k[b, :L])
    ak = f64(cache.a_k[b, :L])[:, :, sel]
    av = f64(cache.a_v[b, :L])[:, :, sel]
    aq = f64(x["a_q"][b, prior:L])[:, :, sel]
    return O.prefill_attention(ak, bk, av, f64(cache.b_v[b, :L]), aq, f64(x["b_q"][b, prior:L]),
                               np.arange(prior, L), scale, w.rope_base, rows=rows)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("rank", [2, 1])
@pytest.mark.parametrize("tokens,prior", [(1, 0), (200, 0), (130, 37), (257, 0), (128, 300)])
def test_prefill_small(kernel, rank, tokens, prior):
    w = S.WORKLOADS["prefill_b4_t4k"].replace(r_k=rank, r_v=rank)
    cache, x, a_q, b_q, q_pos = _prefill_case(w, 2, tokens, prior)
    out = T.tpa_prefill_attention(cache, a_q, b_q, q_pos, kernel=kernel)
    assert T.tpa_read_device_error() == 0
    got = f64(out)
    for b in range(2):
        ref = _oracle(w, cache, x, prior, tokens, b)
        assert_rows_close(got[b], ref, TOL[cache.dtype], f"prefill b={b}")
    ref = _oracle(w, cache, x, prior, tokens, 0, rows=[0, tokens - 1], end_to_end=True)
    assert_rows_close(got[0][[0, tokens - 1]], ref, TOL[cache.dtype], "prefill end-to-end")


@pytest.mark.parametrize("rq,rk,rv,h,d,dt", [
    (1, 1, 1, 8, 64, "bf16"), (3, 2, 1, 16, 32, "bf16"), (8, 4, 4, 32, 128, "bf16"),
    (2, 1, 1, 4, 16, "f32"), (6, 2, 2, 32, 128, "f32"),
])
def test_prefill_other_shapes(rq, rk, rv, h, d, dt):
    w = S.PrefillWorkload("shape", 2, 70, h, d, rq, rk, rv, 256, dt, seed=rq + rk + h)
    cache, x, a_q, b_q, q_pos = _prefill_case(w, 2, 70, prior=11)
    out = T.tpa_prefill_attention(cache, a_q, b_q, q_pos)
    got = f64(out)
    for b in range(2):
        assert_rows_close(got[b], _oracle(w, cache, x, 11, 70, b), TOL[cache.dtype], f"shape b={b}")


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_longer_than_cache_is_reported(kernel):
    w = S.WORKLOADS["prefill_b4_t4k"]
    cache, x, a_q, b_q, q_pos = _prefill_case(w, 2, 50)
    cache.seq_lens[1] = 20                         # sequence 1 holds fewer tokens than the chunk
    out = torch.full((2, 50, 32, 128), 7.0, device=DEV)
    T.tpa_prefill_attention(cache, a_q, b_q, q_pos, out=out, kernel=kernel)
    assert T.tpa_read_device_error() & T.TPA_DEVERR_PREFILL_LEN
    assert bool((out[1] == 7.0).all())


@pytest.mark.slow
@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_workload_full_size(kernel):
    """The full causal prefill (B=4, T=4096); oracle on sampled rows x heads."""
    w = S.WORKLOADS["prefill_b4_t4k"]
    cache, x, a_q, b_q, q_pos = _prefill_case(w, w.batch, w.tokens, nan_fill=False)
    out = T.tpa_prefill_attention(cache, a_q, b_q, q_pos, kernel=kernel)
    assert T.tpa_read_device_error() == 0
    got = f64(out)
    g = np.random.default_rng(0)
    for b in range(w.batch):
        rows = sorted(set([0, 1, 127, 128, w.tokens - 1] + g.integers(0, w.tokens, 12).tolist()))
        heads = [0, 9, 31]
        ref = _oracle(w, cache, x, 0, w.tokens, b, rows=rows, heads=heads)
        assert_rows_close(got[b][rows][:, heads], ref, TOL[cache.dtype], f"prefill full b={b}")


@pytest.mark.parametrize("tokens,prior", [(200, 0), (130, 37), (1000, 3000)])
def test_last_prefill_row_equals_factored_decode(tokens, prior):
    """Two kernels, one quantity: the prefill's last query row (slot L - 1, attending slots
    0 .. L - 1) is the decode of a query in TPA form (A_Q, B_Q of that token, at position L - 1)
    over the same cache.  The decode keeps ~16 bits of its query and weights (bf16 high + low
    parts), the tensor-core prefill rounds both once to fp16 (11 bits, ~4e-4 relative each), so
    the two agree to the prefill's own error, well inside the 2e-3 parity budget."""
    w = S.WORKLOADS["prefill_b4_t4k"]
    cache, x, a_q, b_q, q_pos = _prefill_case(w, 2, tokens, prior)
    out = T.tpa_prefill_attention(cache, a_q, b_q, q_pos)
    L = prior + tokens
    dec = T.tpa_decode_attention_factored(cache, a_q[:, -1].contiguous(), b_q[:, -1].contiguous(),
                                          q_pos[:, -1].contiguous(), max_len=L)
    assert T.tpa_read_device_error() == 0
    assert_rows_close(f64(dec), f64(out[:, -1]), 1.5e-3, "prefill last row vs factored decode")


@pytest.mark.parametrize("kernel", KERNELS)
def test_prefill_ragged_prior(kernel):
    """Sequences with different numbers of cached tokens before the chunk (P = seq_lens[b] - T
    differs per sequence): each query t of sequence b sits at slot P_b + t and attends slots
    0 .. P_b + t.  The cache is written with explicit slots, so each sequence holds its own count."""
    w = S.WORKLOADS["prefill_b4_t4k"]
    priors, tokens = [37, 300, 0], 133
    B, n = len(priors), max(priors) + tokens
    x = S.prefill_inputs(w, batch=B, tokens=n)
    cap = n + 5
    cache = T.TpaCache.allocate(B, cap, w.heads, w.head_dim, w.r_k, w.r_v, dtype=TORCH_DTYPE[w.dtype],
                                rope_base=w.rope_base, fill=float("nan"))
    # sequence b: its first priors[b] + tokens tokens at slots 0.., the rest of the n written rows
    # to the slots above, which its length excludes
    slots = torch.empty(B, n, dtype=torch.int32)
    for b, pr in enumerate(priors):
        L = pr + tokens
        slots[b, :L] = torch.arange(L, dtype=torch.int32)
        slots[b, L:] = torch.arange(L, n, dtype=torch.int32)
    T.tpa_cache_write_slots(cache, slots.to(DEV), x["positions"].to(DEV), *(x[k].to(DEV) for k in ("a_k", "b_k", "a_v", "b_v")))
    cache.seq_lens.copy_(torch.tensor([pr + tokens for pr in priors], dtype=torch.int32, device=DEV))
    a_q = torch.stack([x["a_q"][b, pr:pr + tokens] for b, pr in enumerate(priors)]).contiguous().to(DEV)
    b_q = torch.stack([x["b_q"][b, pr:pr + tokens] for b, pr in enumerate(priors)]).contiguous().to(DEV)
    q_pos = torch.stack([x["positions"][b, pr:pr + tokens] for b, pr in enumerate(priors)]).contiguous().to(DEV)
    out = T.tpa_prefill_attention(cache, a_q, b_q, q_pos, kernel=kernel)
    assert T.tpa_read_device_error() == 0
    got = f64(out)
    for b, pr in enumerate(priors):
        ref = _oracle(w, cache, x, pr, tokens, b)
        assert_rows_close(got[b], ref, TOL[cache.dtype], f"prefill ragged b={b}")
