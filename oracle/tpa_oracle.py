"""Plain float64 CPU oracle for Tensor Product Attention over a factorized KV cache.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` may import this module.  It shares no code with
the CUDA library and never imports it.

Everything here is the plain definition written out in float64 NumPy, with a
matrix product or ``einsum`` as the only library step.  Inputs are the exact
float64 upcasts of whatever the caller stores (fp32 or bf16 values).

Sources (page "Tensor Product Attention Is All You Need", NeurIPS 2025 notes):

* section 解决思路 (approach): a query is a tensor product of factors,
  Q_t = (1/R) A_Q(x_t)^T B_Q(x_t).
* section 关键设计 / 张量积分解 (key design: tensor product decomposition):
  K_t = (1/R_K) A_K(x_t)^T B_K(x_t) with A in R^{R x h} (head factor) and
  B in R^{R x d_h} (feature factor); the same for V with R_V.  The cache keeps
  A_K, B_K, A_V, B_V, i.e. (R_K + R_V)(h + d_h) numbers per token instead of
  2 h d_h (320 instead of 8192 at R_K = R_V = 1, h = 32, d_h = 128).
* section RoPE 兼容性 (Theorem 3.1): the rotation T is applied to the B
  factors only and keeps the relative-position property
  Q~_t K~_s^T = Q_t T_{t-s} K_s^T.
* section FlashTPA: attention is evaluated from the factors; the result is the
  ordinary softmax attention of the expanded Q, K, V, which is what this file
  computes.

Readings of points the page leaves open (each is stated where it is used):

* RoPE pairs are adjacent elements (2j, 2j+1) rotated by the angle
  pos * theta_j, theta_j = base^(-2j/d_h), as
  (x, y) -> (x cos a - y sin a, x sin a + y cos a).
* The softmax scale is 1/sqrt(d_h); 1/R_K, 1/R_V, 1/R_Q sit inside the factor
  products as the page writes them.
* Decode attends to exactly the tokens stored in the cache (slots 0..L-1);
  the query's own position only sets its rotation.
* Causal prefill: the T queries of a chunk are the last T cache slots; query
  t (slot P + t, P = L - T) attends slots 0..P+t inclusive.
* Outputs are float64 here; the CUDA library writes fp32.
* The cache stores its factors in the storage dtype (bf16 or fp32), and B_K
  is rotated before it is stored (append applies RoPE): the stored B~_K is
  the rotated value rounded once to the storage dtype (round to nearest,
  ties to even).  ``append_rope(..., storage=...)`` models that rounding.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_to_storage",
    "factor_elements_per_token",
    "dense_elements_per_token",
    "rope_frequencies",
    "rope",
    "tensor_product",
    "append_rope",
    "decode_attention",
    "decode_attention_factored_query",
    "decode_attention_from_unrotated",
    "decode_step",
    "decode_attention_lse",
    "merge_lse",
    "prefill_queries",
    "prefill_attention",
    "softmax_attention",
]


def factor_elements_per_token(h: int, d_h: int, r_k: int, r_v: int) -> int:
    """Numbers stored per token by the factorized cache: (R_K + R_V)(h + d_h).

    Section 关键设计 / 张量积分解 (cache size from 2 h d_h to (R_K+R_V)(h+d_h)).
    """
    return (r_k + r_v) * (h + d_h)


def dense_elements_per_token(h: int, d_h: int) -> int:
    """Numbers stored per token by a dense K/V cache: 2 h d_h (same section)."""
    return 2 * h * d_h


def round_to_storage(x: np.ndarray, storage: str | None) -> np.ndarray:
    """Round float64 values once to the storage dtype, ties to even.

    ``"f32"``: IEEE binary32.  ``"bf16"``: 8 significant bits (binary32
    exponent range), written out as m * 2^e with m rounded at 2^-8 relative
    to the leading bit (np.rint rounds half to even); values below the
    smallest normal use the subnormal spacing 2^-133.  ``None``: unchanged.
    """
    x = np.asarray(x, dtype=np.float64)
    if storage is None:
        return x
    if storage == "f32":
        return x.astype(np.float32).astype(np.float64)
    if storage != "bf16":
        raise ValueError(storage)
    mant, expo = np.frexp(x)                     # x = mant * 2^expo, 0.5 <= |mant| < 1
    normal = np.ldexp(np.rint(np.ldexp(mant, 8)), expo - 8)
    tiny = np.ldexp(np.rint(np.ldexp(x, 133)), -133)
    out = np.where(np.abs(x) >= 2.0 ** -126, normal, tiny)
    return np.where(np.abs(out) > 3.3895313892515355e38, np.copysign(np.inf, x), out)


def rope_frequencies(d_h: int, base: float) -> np.ndarray:
    """theta_j = base^(-2j/d_h) for the pair j = 0 .. d_h/2 - 1 (reading)."""
    j = np.arange(d_h // 2, dtype=np.float64)
    return np.power(np.float64(base), -2.0 * j / d_h)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate the last axis of ``x`` by the RoPE operator at position ``pos``.

    ``pos`` broadcasts against ``x.shape[:-1]``.  Pair j = (x[2j], x[2j+1]) is
    rotated by the angle pos * theta_j (section RoPE 兼容性, the operator T;
    pair layout and orientation are readings).
    """
    x = np.asarray(x, dtype=np.float64)
    d_h = x.shape[-1]
    theta = rope_frequencies(d_h, base)
    angle = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(angle), np.sin(angle)
    even, odd = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, angle.shape[:-1] + (d_h,)), dtype=np.float64)
    out[..., 0::2] = even * c - odd * s
    out[..., 1::2] = even * s + odd * c
    return out


def tensor_product(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """(1/R) A^T B per token: a [..., R, h], b [..., R, d_h] -> [..., h, d_h].

    Section 关键设计 / 张量积分解 (K_t = (1/R_K) A_K^T B_K, likewise V and Q).
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    rank = a.shape[-2]
    return np.einsum("...ri,...rk->...ik", a, b) / rank


def append_rope(b_k: np.ndarray, positions: np.ndarray, base: float, storage: str | None = None) -> np.ndarray:
    """B~_K: every rank row of token s rotated at that token's position.

    b_k [..., S, R_K, d_h], positions [..., S].  RoPE acts on the B factor only
    (section RoPE 兼容性, Theorem 3.1); A_K, A_V and B_V are stored unchanged.
    ``storage`` rounds the rotated rows once to the cache dtype, as the cache
    keeps them.
    """
    return round_to_storage(rope(b_k, np.asarray(positions)[..., None], base), storage)


def softmax_attention(z: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Textbook softmax attention: z [n, S] scores, v [S, d] -> [n, d].

    Rows whose scores are all -inf (no admissible token) return zeros.
    """
    m = np.max(z, axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.exp(z - m)
    l = p.sum(axis=-1, keepdims=True)
    o = p @ v
    return np.divide(o, l, out=np.zeros_like(o), where=l > 0)


def decode_attention(a_k, b_k_rot, a_v, b_v, q, q_pos, scale, base, block: int = 8192):
    """Decode attention of one sequence over its cached tokens.

    a_k [L, R_K, h], b_k_rot [L, R_K, d_h] (already rotated, as the cache
    stores it), a_v [L, R_V, h], b_v [L, R_V, d_h], q [h, d_h] unrotated at
    position q_pos.  Returns o [h, d_h] (float64):

      q~_i = RoPE(q_i, q_pos)
      K_s = (1/R_K) A_K[s]^T B~_K[s],  V_s = (1/R_V) A_V[s]^T B_V[s]
      z[i, s] = scale * q~_i . K_s[i],  o_i = sum_s softmax_s(z[i, :]) V_s[i]
    """
    return _attend_rotated_query(a_k, b_k_rot, a_v, b_v, rope(q, q_pos, base), scale, block)


def decode_attention_factored_query(a_k, b_k_rot, a_v, b_v, a_q, b_q, q_pos, scale, base, block: int = 8192):
    """Decode attention with the query in TPA form (section 解决思路:
    Q = (1/R_Q) A_Q^T B_Q; RoPE on the B factor, Theorem 3.1).

    a_q [R_Q, h], b_q [R_Q, d_h] unrotated at position q_pos; the cache as in
    decode_attention.  q~_i = (1/R_Q) sum_j A_Q[j, i] RoPE(B_Q[j], q_pos), then
    the same attention.  Returns o [h, d_h] (float64).
    """
    return _attend_rotated_query(a_k, b_k_rot, a_v, b_v, tensor_product(a_q, rope(b_q, q_pos, base)), scale, block)


def _attend_rotated_query(a_k, b_k_rot, a_v, b_v, q_rot, scale, block):
    """Softmax attention of rotated per-head queries q_rot [h, d_h] over the
    cached tokens (see decode_attention)."""
    return _attend_rotated_query_lse(a_k, b_k_rot, a_v, b_v, q_rot, scale, block)[0]


def _attend_rotated_query_lse(a_k, b_k_rot, a_v, b_v, q_rot, scale, block):
    """(o [h, d_h], lse [h]): the attention of _attend_rotated_query and the natural log of
    each head's sum of exp(score).  K and V are expanded ``block`` tokens at a time only to
    bound memory: every score is computed on its own, the softmax is taken over the full
    score row, and the output sum is split into consecutive partial sums."""
    L = np.asarray(a_k).shape[0]
    h, d_h = np.asarray(q_rot).shape
    if L == 0:
        return np.zeros((h, d_h)), np.full(h, -np.inf)
    z = np.empty((h, L))
    for s0 in range(0, L, block):
        s1 = min(L, s0 + block)
        k = tensor_product(a_k[s0:s1], b_k_rot[s0:s1])            # [n, h, d_h]
        z[:, s0:s1] = scale * np.einsum("ik,sik->is", q_rot, k)
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    total = p.sum(axis=1, keepdims=True)
    p /= total
    o = np.zeros((h, d_h))
    for s0 in range(0, L, block):
        s1 = min(L, s0 + block)
        v = tensor_product(a_v[s0:s1], b_v[s0:s1])                # [n, h, d_h]
        o += np.einsum("is,sik->ik", p[:, s0:s1], v)
    return o, (m + np.log(total))[:, 0]


def decode_attention_lse(a_k, b_k_rot, a_v, b_v, q, q_pos, scale, base, block: int = 8192):
    """decode_attention plus lse [h] = log sum_s exp(scale q~_i . K_s[i]) (natural log; -inf
    with nothing cached, where o = 0).  (o, lse) is the state a shard of the token range hands
    to merge_lse when one sequence is split across devices (the split-KV reduction)."""
    return _attend_rotated_query_lse(a_k, b_k_rot, a_v, b_v, rope(q, q_pos, base), scale, block)


def merge_lse(outs, lses):
    """Attention over the union of disjoint token sets from each set's (o_r, lse_r):
    lse = log sum_r exp(lse_r), o = sum_r exp(lse_r - lse) o_r; parts with lse_r = -inf (no
    tokens) drop out, and with no tokens at all o = 0, lse = -inf.  outs [n, h, d_h],
    lses [n, h] -> (o [h, d_h], lse [h])."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    top = lses.max(axis=0)                                            # [h]
    safe = np.where(np.isfinite(top), top, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - safe[None]), 0.0)   # [n, h]
    tot = w.sum(axis=0)
    o = np.einsum("rh,rhk->hk", w, outs)
    o = np.divide(o, tot[:, None], out=np.zeros_like(o), where=tot[:, None] > 0)
    lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    return o, lse


def decode_attention_from_unrotated(a_k, b_k, a_v, b_v, positions, q, q_pos, scale, base, storage=None):
    """End-to-end decode: rotate B_K at each token's position (stored in the
    cache dtype when ``storage`` is given), then attend."""
    return decode_attention(a_k, append_rope(b_k, positions, base, storage), a_v, b_v, q, q_pos, scale, base)


def decode_step(a_k, b_k_rot, a_v, b_v, new_a_k, new_b_k, new_a_v, new_b_v, pos, scale, base, q=None, a_q=None,
                b_q=None, storage=None):
    """One generation step of token x_t: append its factors, then attend with its query.

    Section 解决思路 derives Q_t, K_t and V_t from the same token x_t, and section
    RoPE 兼容性 (Theorem 3.1) rotates every B factor at that token's position, so
    the new key and the query are both rotated at ``pos``.  The cache (a_k ..
    b_v, L tokens, B_K stored rotated) gains slot L: new_a_k [R_K, h],
    new_b_k [R_K, d_h] (unrotated, stored as append_rope(..., storage) does),
    new_a_v [R_V, h], new_b_v [R_V, d_h].  The query is dense (q [h, d_h]) or in
    TPA form (a_q [R_Q, h], b_q [R_Q, d_h]); it attends slots 0 .. L, its own
    token included.  Returns (o [h, d_h], the stored new B~_K row [R_K, d_h]).
    """
    new_rot = append_rope(np.asarray(new_b_k, dtype=np.float64)[None], np.array([pos], dtype=np.float64), base,
                          storage)[0]
    cat = lambda old, new: np.concatenate([np.asarray(old, dtype=np.float64).reshape((-1,) + np.shape(new)),
                                           np.asarray(new, dtype=np.float64)[None]], axis=0)
    ak, bk, av, bv = cat(a_k, new_a_k), cat(b_k_rot, new_rot), cat(a_v, new_a_v), cat(b_v, new_b_v)
    if q is not None:
        o = decode_attention(ak, bk, av, bv, q, pos, scale, base)
    else:
        o = decode_attention_factored_query(ak, bk, av, bv, a_q, b_q, pos, scale, base)
    return o, new_rot


def prefill_queries(a_q, b_q, q_pos, base):
    """Dense queries of a prompt chunk: Q_t = (1/R_Q) A_Q[t]^T RoPE(B_Q[t], pos_t).

    a_q [T, R_Q, h], b_q [T, R_Q, d_h] unrotated, q_pos [T] -> [T, h, d_h].
    Section 解决思路 (Q factorization) with RoPE on the B factor (Theorem 3.1).
    """
    b_q_rot = rope(b_q, np.asarray(q_pos)[:, None], base)
    return tensor_product(a_q, b_q_rot)


def prefill_attention(a_k, b_k_rot, a_v, b_v, a_q, b_q, q_pos, scale, base, rows=None, heads=None):
    """Causal prefill of one sequence.

    The cache (a_k .. b_v, L tokens, B_K already rotated) holds the prompt's
    own factors in its last T slots; query t sits at slot P + t with
    P = L - T and attends slots 0 .. P + t.  ``rows`` restricts the computation
    to some query indices (all by default), ``heads`` to some heads.
    Returns o [len(rows), h_sel, d_h] (float64).
    """
    L = np.asarray(a_k).shape[0]
    T = np.asarray(a_q).shape[0]
    h = np.asarray(a_q).shape[2]
    P = L - T
    rows = np.arange(T) if rows is None else np.asarray(rows)
    heads = np.arange(h) if heads is None else np.asarray(heads)
    q_all = prefill_queries(a_q[rows], b_q[rows], np.asarray(q_pos)[rows], base)   # [n, h, d]
    k = tensor_product(a_k, b_k_rot)                                                 # [L, h, d]
    v = tensor_product(a_v, b_v)
    slots = np.arange(L)
    allowed = slots[None, :] <= (P + rows)[:, None]                                  # [n, L]
    out = np.zeros((len(rows), len(heads), q_all.shape[-1]))
    for n, i in enumerate(heads):
        z = scale * (q_all[:, i, :] @ k[:, i, :].T)                                  # [n, L]
        z = np.where(allowed, z, -np.inf)
        out[:, n, :] = softmax_attention(z, v[:, i, :])
    return out
