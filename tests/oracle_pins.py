"""Checks that pin the CPU oracle to facts outside itself.

Each ``pin_*`` function takes the oracle module and raises AssertionError when
the oracle disagrees with a printed value, a closed form, an invariant, a
library routine or a brute-force evaluation.  ``test_oracle_pins.py`` runs them
on the oracle as it is; ``test_oracle_mutations.py`` plants plausible mistakes
in the oracle and checks that some pin fails for each.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_case(seed, L, h, d, rk, rv, ab_std=1.0):
    g = np.random.default_rng(seed)
    return dict(
        a_k=g.standard_normal((L, rk, h)) * ab_std,
        b_k=g.standard_normal((L, rk, d)) / math.sqrt(d),
        a_v=g.standard_normal((L, rv, h)) * ab_std,
        b_v=g.standard_normal((L, rv, d)) / math.sqrt(d),
        q=g.standard_normal((h, d)),
    )


# --------------------------------------------------------------------------- printed values
def pin_cache_size(O):
    """The page's printed per-token sizes: 2 h d_h = 8192 vs (R_K+R_V)(h+d_h) = 320."""
    g = _golden("cache_size.json")
    assert O.dense_elements_per_token(g["h"], g["d_h"]) == g["dense_elements_per_token"]
    assert O.factor_elements_per_token(g["h"], g["d_h"], g["r_k"], g["r_v"]) == g["factor_elements_per_token"]
    # the R=2 decode workload: 32 seqs x 32768 tokens x (2+2)(32+128) bf16 = 1.342 GB ("about 1.3 GB")
    assert 32 * 32768 * O.factor_elements_per_token(32, 128, 2, 2) * 2 == 1_342_177_280


# --------------------------------------------------------------------------- RoPE
def pin_rope_closed_form(O):
    """RoPE on unit vectors has closed forms: angle pos * base^(-2j/d_h)."""
    # d_h = 2: theta_0 = 1, so e_0 at position p becomes (cos p, sin p)
    for p in (0.0, 1.0, 2.5, 1000.0):
        r = O.rope(np.array([1.0, 0.0]), p, 10000.0)
        assert np.allclose(r, [math.cos(p), math.sin(p)], rtol=0, atol=1e-12)
        r = O.rope(np.array([0.0, 1.0]), p, 10000.0)
        assert np.allclose(r, [-math.sin(p), math.cos(p)], rtol=0, atol=1e-12)
    # d_h = 4, base 100: theta_1 = 100^(-1/2) = 0.1, so pair 1 at position 10 turns by 1 rad
    r = O.rope(np.array([0.0, 0.0, 1.0, 0.0]), 10.0, 100.0)
    assert np.allclose(r, [0.0, 0.0, math.cos(1.0), math.sin(1.0)], rtol=0, atol=1e-12)
    r = O.rope(np.array([1.0, 0.0, 0.0, 0.0]), 10.0, 100.0)
    assert np.allclose(r, [math.cos(10.0), math.sin(10.0), 0.0, 0.0], rtol=0, atol=1e-12)
    # d_h = 8, base 10000: theta_j = 10^(-j), pair 3 at position 1000 turns by 1 rad
    x = np.zeros(8)
    x[6] = 1.0
    assert np.allclose(O.rope(x, 1000.0, 10000.0)[6:], [math.cos(1.0), math.sin(1.0)], atol=1e-12)


def pin_rope_complex(O):
    """Pairs rotate as complex numbers: (x + iy) * exp(i pos theta_j)."""
    g = np.random.default_rng(7)
    d = 16
    x = g.standard_normal((5, d))
    pos = np.array([0.0, 3.0, 17.0, 4095.0, 524287.0])
    r = O.rope(x, pos, 10000.0)
    j = np.arange(d // 2)
    theta = 10000.0 ** (-(2.0 * j) / d)
    zc = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * theta[None, :])
    assert np.allclose(r[:, 0::2], zc.real, atol=1e-12)
    assert np.allclose(r[:, 1::2], zc.imag, atol=1e-12)
    # rotations keep norms and position 0 is the identity
    assert np.allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), atol=1e-12)
    assert np.array_equal(O.rope(x, 0.0, 10000.0), x)


def _block_rotation(d, delta, base):
    """T_delta as an explicit block-diagonal matrix (row-vector convention x T)."""
    Tm = np.zeros((d, d))
    for j in range(d // 2):
        a = delta * base ** (-(2.0 * j) / d)
        c, s = math.cos(a), math.sin(a)
        # row vector (x, y) maps to (x c - y s, x s + y c)
        Tm[2 * j, 2 * j], Tm[2 * j, 2 * j + 1] = c, s
        Tm[2 * j + 1, 2 * j], Tm[2 * j + 1, 2 * j + 1] = -s, c
    return Tm


def pin_theorem_3_1(O):
    """Theorem 3.1: Q~_t K~_s^T = Q_t T_{t-s} K_s^T with RoPE on the B factors only.

    Built from factors: K_s from A_K, B_K with B_K rotated at s; Q_t from A_Q, B_Q
    with B_Q rotated at t.  Also: scores do not change under a common shift.
    """
    g = np.random.default_rng(11)
    h, d, rq, rk = 3, 8, 2, 2
    base = 10000.0
    a_q, b_q = g.standard_normal((rq, h)), g.standard_normal((rq, d))
    a_k, b_k = g.standard_normal((rk, h)), g.standard_normal((rk, d))
    q_plain = O.tensor_product(a_q, b_q)                  # [h, d]
    k_plain = O.tensor_product(a_k, b_k)
    for t, s in ((5, 2), (2, 5), (700, 3), (400000, 123456)):
        q_rot = O.tensor_product(a_q, O.rope(b_q, float(t), base))
        k_rot = O.tensor_product(a_k, O.rope(b_k, float(s), base))
        lhs = np.einsum("ik,ik->i", q_rot, k_rot)
        rhs = np.einsum("ik,kl,il->i", q_plain, _block_rotation(d, t - s, base), k_plain)
        assert np.allclose(lhs, rhs, rtol=1e-9, atol=1e-9), (t, s, lhs, rhs)
    # common shift of every position leaves decode scores (hence outputs) unchanged
    c = _rand_case(3, 40, 4, 16, 2, 2)
    pos = np.arange(40, dtype=np.float64)
    o0 = O.decode_attention(c["a_k"], O.append_rope(c["b_k"], pos, base), c["a_v"], c["b_v"], c["q"], 40.0, 0.25, base)
    for delta in (1.0, 1000.0, 400000.0):
        o1 = O.decode_attention(c["a_k"], O.append_rope(c["b_k"], pos + delta, base), c["a_v"], c["b_v"],
                                c["q"], 40.0 + delta, 0.25, base)
        assert np.allclose(o0, o1, rtol=1e-9, atol=1e-11), delta


# --------------------------------------------------------------------------- closed forms
def pin_two_token_golden(O):
    """Worked two-token example (tests/golden/two_token_decode.json), closed form."""
    g = _golden("two_token_decode.json")
    a_k, b_k = np.array(g["a_k"]), np.array(g["b_k"])
    a_v, b_v = np.array(g["a_v"]), np.array(g["b_v"])
    pos = np.array(g["positions"], dtype=np.float64)
    q = np.array(g["q"])
    o = O.decode_attention(a_k, O.append_rope(b_k, pos, g["rope_base"]), a_v, b_v, q, float(g["q_pos"]),
                           1.0 / math.sqrt(g["d_h"]), g["rope_base"])
    z0 = math.sqrt(2.0) * math.sin(1.0)
    z1 = 1.0 / math.sqrt(2.0)
    p0 = 1.0 / (1.0 + math.exp(z1 - z0))
    assert np.allclose(o, [[p0, 3.0 * (1.0 - p0)]], rtol=0, atol=1e-13), o


def pin_single_token(O):
    """One cached token: softmax weight 1, so o_i = V_0[i] = (1/R_V) sum_r A_V[0,r,i] B_V[0,r,:]."""
    c = _rand_case(5, 1, 3, 8, 2, 2)
    o = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], c["q"], 9.0, 0.3, 10000.0)
    v0 = np.zeros((3, 8))
    for i in range(3):
        for k in range(8):
            v0[i, k] = (c["a_v"][0, 0, i] * c["b_v"][0, 0, k] + c["a_v"][0, 1, i] * c["b_v"][0, 1, k]) / 2.0
    assert np.allclose(o, v0, rtol=0, atol=1e-13)


def pin_zero_query_mean(O):
    """q = 0: every score is 0, the weights are uniform and o is the mean of V."""
    c = _rand_case(6, 9, 2, 8, 1, 2)
    o = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], np.zeros((2, 8)), 3.0, 0.3, 10000.0)
    v = np.einsum("sri,srk->sik", c["a_v"], c["b_v"]) / 2.0
    assert np.allclose(o, v.mean(axis=0), rtol=0, atol=1e-13)


def pin_duplicate_ranks(O):
    """R copies of the same rank-1 factors equal the rank-1 result (the 1/R sits in the product)."""
    c = _rand_case(8, 30, 4, 16, 1, 1)
    o1 = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], c["q"], 30.0, 0.25, 10000.0)
    for r in (2, 3):
        rep = {k: np.repeat(c[k], r, axis=1) for k in ("a_k", "b_k", "a_v", "b_v")}
        o2 = O.decode_attention(rep["a_k"], rep["b_k"], rep["a_v"], rep["b_v"], c["q"], 30.0, 0.25, 10000.0)
        assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14)


def pin_factor_rescale(O):
    """A -> cA, B -> B/c leaves the output unchanged (only the product A^T B matters)."""
    c = _rand_case(9, 25, 3, 8, 2, 2)
    o1 = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], c["q"], 25.0, 0.4, 10000.0)
    o2 = O.decode_attention(c["a_k"] * 4.0, c["b_k"] / 4.0, c["a_v"] * 0.5, c["b_v"] * 2.0, c["q"], 25.0, 0.4,
                            10000.0)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------- library routines
def pin_mqa_sdpa(O):
    """A_K = A_V = 1 with rank 1 makes every head share K and V (multi-query attention).

    Compared with PyTorch's float64 scaled_dot_product_attention on the rotated
    keys and values.
    """
    g = np.random.default_rng(12)
    L, h, d = 37, 4, 16
    b_k = g.standard_normal((L, 1, d)) / 4
    b_v = g.standard_normal((L, 1, d))
    q = g.standard_normal((h, d))
    ones = np.ones((L, 1, h))
    pos = np.arange(L, dtype=np.float64)
    bkr = O.append_rope(b_k, pos, 500.0)
    o = O.decode_attention(ones, bkr, ones, b_v, q, 44.0, 0.37, 500.0)
    qr = torch.from_numpy(O.rope(q, 44.0, 500.0))[None, :, None, :]            # [1, h, 1, d]
    kk = torch.from_numpy(bkr[:, 0, :]).expand(h, L, d)[None]
    vv = torch.from_numpy(b_v[:, 0, :]).expand(h, L, d)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kk, vv, scale=0.37)[0, :, 0, :].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)


def pin_general_sdpa(O):
    """For any factors, decode equals SDPA on K, V expanded per token by scalar loops."""
    c = _rand_case(13, 21, 3, 8, 2, 1)
    L, h, d = 21, 3, 8
    k = np.zeros((h, L, d))
    v = np.zeros((h, L, d))
    for s in range(L):
        for i in range(h):
            for kk in range(d):
                k[i, s, kk] = sum(c["a_k"][s, r, i] * c["b_k"][s, r, kk] for r in range(2)) / 2.0
                v[i, s, kk] = c["a_v"][s, 0, i] * c["b_v"][s, 0, kk]
    o = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], c["q"], 0.0, 0.5, 10000.0)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(c["q"])[:, None, :], torch.from_numpy(k), torch.from_numpy(v), scale=0.5)[:, 0, :].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)


def pin_prefill_causal_sdpa(O):
    """Causal prefill equals SDPA with a causal mask on queries/keys expanded by loops."""
    g = np.random.default_rng(14)
    T, h, d, rq, rk, rv = 11, 2, 8, 3, 2, 2
    a_q, b_q = g.standard_normal((T, rq, h)), g.standard_normal((T, rq, d))
    a_k, b_k = g.standard_normal((T, rk, h)), g.standard_normal((T, rk, d))
    a_v, b_v = g.standard_normal((T, rv, h)), g.standard_normal((T, rv, d))
    pos = np.arange(T, dtype=np.float64)
    bkr = O.append_rope(b_k, pos, 10000.0)
    o = O.prefill_attention(a_k, bkr, a_v, b_v, a_q, b_q, pos, 0.3, 10000.0)
    bqr = O.rope(b_q, pos[:, None], 10000.0)
    Q = np.zeros((h, T, d)); K = np.zeros((h, T, d)); V = np.zeros((h, T, d))
    for t in range(T):
        for i in range(h):
            for k in range(d):
                Q[i, t, k] = sum(a_q[t, j, i] * bqr[t, j, k] for j in range(rq)) / rq
                K[i, t, k] = sum(a_k[t, r, i] * bkr[t, r, k] for r in range(rk)) / rk
                V[i, t, k] = sum(a_v[t, r, i] * b_v[t, r, k] for r in range(rv)) / rv
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q), torch.from_numpy(K), torch.from_numpy(V), is_causal=True, scale=0.3).numpy()
    assert np.allclose(o, ref.transpose(1, 0, 2), rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------- brute force
def _brute_rot(x, pos, base):
    d = len(x)
    out = [0.0] * d
    for j in range(d // 2):
        a = pos * base ** (-(2.0 * j) / d)
        out[2 * j] = x[2 * j] * math.cos(a) - x[2 * j + 1] * math.sin(a)
        out[2 * j + 1] = x[2 * j] * math.sin(a) + x[2 * j + 1] * math.cos(a)
    return out


def pin_brute_force_decode(O):
    """Every step by scalar loops (math.cos/sin/exp, math.fsum) on tiny inputs."""
    for seed, (L, h, d, rk, rv) in enumerate([(1, 1, 2, 1, 1), (3, 2, 4, 2, 1), (3, 2, 4, 1, 2), (5, 1, 6, 3, 3)]):
        c = _rand_case(100 + seed, L, h, d, rk, rv)
        pos = [float(3 * s + 1) for s in range(L)]
        qpos, scale, base = 17.0, 0.7, 50.0
        o = O.decode_attention(c["a_k"], O.append_rope(c["b_k"], np.array(pos), base), c["a_v"], c["b_v"],
                               c["q"], qpos, scale, base)
        for i in range(h):
            qr = _brute_rot(list(c["q"][i]), qpos, base)
            z = []
            for s in range(L):
                key = [0.0] * d
                for r in range(rk):
                    br = _brute_rot(list(c["b_k"][s, r]), pos[s], base)
                    for k in range(d):
                        key[k] += c["a_k"][s, r, i] * br[k] / rk
                z.append(scale * math.fsum(qr[k] * key[k] for k in range(d)))
            m = max(z)
            w = [math.exp(x - m) for x in z]
            tot = math.fsum(w)
            for k in range(d):
                ref = math.fsum(w[s] / tot * math.fsum(c["a_v"][s, r, i] * c["b_v"][s, r, k] / rv for r in range(rv))
                                for s in range(L))
                assert abs(o[i, k] - ref) <= 1e-12 * (1 + abs(ref)), (seed, i, k, o[i, k], ref)


def pin_brute_force_from_unrotated(O):
    """End-to-end decode from unrotated factors by scalar loops: each cached key row rotated
    at its own token's position (not the query's), rounded to the storage dtype when one is
    given (round_to_storage is itself pinned against PyTorch's conversion), the query rotated
    at its position, then softmax over the cached tokens with math.fsum."""
    cases = [(3, 2, 4, 2, 1, None), (4, 2, 6, 1, 2, "bf16"), (2, 1, 4, 2, 2, "f32"), (5, 3, 8, 2, 2, "bf16")]
    for seed, (L, h, d, rk, rv, storage) in enumerate(cases):
        c = _rand_case(140 + seed, L, h, d, rk, rv)
        pos = [float(5 * s + 2) for s in range(L)]
        qpos, scale, base = 31.0, 0.9, 100.0
        o = O.decode_attention_from_unrotated(c["a_k"], c["b_k"], c["a_v"], c["b_v"], np.array(pos), c["q"], qpos,
                                              scale, base, storage=storage)
        rows = [[O.round_to_storage(np.array(_brute_rot(list(c["b_k"][s, r]), pos[s], base)), storage).tolist()
                 for r in range(rk)] for s in range(L)]
        for i in range(h):
            qr = _brute_rot(list(c["q"][i]), qpos, base)
            z = []
            for s in range(L):
                key = [math.fsum(c["a_k"][s, r, i] * rows[s][r][k] for r in range(rk)) / rk for k in range(d)]
                z.append(scale * math.fsum(qr[k] * key[k] for k in range(d)))
            m = max(z)
            w = [math.exp(x - m) for x in z]
            tot = math.fsum(w)
            for k in range(d):
                ref = math.fsum(w[s] / tot * math.fsum(c["a_v"][s, r, i] * c["b_v"][s, r, k] for r in range(rv)) / rv
                                for s in range(L))
                assert abs(o[i, k] - ref) <= 1e-12 * (1 + abs(ref)), (seed, storage, i, k, o[i, k], ref)


def pin_brute_force_prefill(O):
    """Causal prefill with a previous chunk (P > 0) by scalar loops on tiny inputs."""
    g = np.random.default_rng(21)
    P, T, h, d, rq, rk, rv = 2, 3, 2, 4, 2, 1, 2
    L = P + T
    a_k, b_k = g.standard_normal((L, rk, h)), g.standard_normal((L, rk, d))
    a_v, b_v = g.standard_normal((L, rv, h)), g.standard_normal((L, rv, d))
    a_q, b_q = g.standard_normal((T, rq, h)), g.standard_normal((T, rq, d))
    kpos = [float(s) for s in range(L)]
    qpos = [float(P + t) for t in range(T)]
    base, scale = 10000.0, 0.5
    o = O.prefill_attention(a_k, O.append_rope(b_k, np.array(kpos), base), a_v, b_v, a_q, b_q,
                            np.array(qpos), scale, base)
    for t in range(T):
        for i in range(h):
            qv = [0.0] * d
            for j in range(rq):
                br = _brute_rot(list(b_q[t, j]), qpos[t], base)
                for k in range(d):
                    qv[k] += a_q[t, j, i] * br[k] / rq
            z = []
            for s in range(P + t + 1):
                key = [0.0] * d
                for r in range(rk):
                    br = _brute_rot(list(b_k[s, r]), kpos[s], base)
                    for k in range(d):
                        key[k] += a_k[s, r, i] * br[k] / rk
                z.append(scale * math.fsum(qv[k] * key[k] for k in range(d)))
            m = max(z)
            w = [math.exp(x - m) for x in z]
            tot = math.fsum(w)
            for k in range(d):
                ref = math.fsum(w[s] / tot * math.fsum(a_v[s, r, i] * b_v[s, r, k] / rv for r in range(rv))
                                for s in range(len(z)))
                assert abs(o[t, i, k] - ref) <= 1e-12 * (1 + abs(ref)), (t, i, k)


def pin_prefill_first_row(O):
    """Prefill query 0 with no earlier chunk sees only slot 0: o = V_0."""
    g = np.random.default_rng(22)
    T, h, d = 5, 2, 8
    a_k, b_k = g.standard_normal((T, 2, h)), g.standard_normal((T, 2, d))
    a_v, b_v = g.standard_normal((T, 2, h)), g.standard_normal((T, 2, d))
    a_q, b_q = g.standard_normal((T, 6, h)), g.standard_normal((T, 6, d))
    o = O.prefill_attention(a_k, b_k, a_v, b_v, a_q, b_q, np.arange(T, dtype=np.float64), 0.3, 10000.0, rows=[0])
    v0 = (a_v[0].T @ b_v[0]) / 2.0
    assert np.allclose(o[0], v0, rtol=0, atol=1e-13)


def pin_storage_rounding(O):
    """bf16 storage rounding: closed-form ties to even and PyTorch's float32 -> bfloat16 conversion."""
    r = lambda v: float(O.round_to_storage(np.array([v]), "bf16")[0])
    assert r(1.0 + 2.0 ** -8) == 1.0                    # exact tie, round to the even significand
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6    # exact tie, round up to even
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    assert r(-(1.0 + 2.0 ** -9)) == -1.0
    assert r(0.0) == 0.0 and r(2.0 ** -130) == 2.0 ** -130
    g = np.random.default_rng(31)
    x = (g.standard_normal(200000) * np.exp(g.uniform(-30, 30, 200000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.round_to_storage(x.astype(np.float64), "bf16"), ref)
    f = O.round_to_storage(np.array([1.0 + 2.0 ** -30]), "f32")
    assert f[0] == 1.0
    # the stored rotated rows are bf16 values within half a bf16 ulp (2^-8 relative) of the rotation
    b = g.standard_normal((5, 2, 8))
    pos = np.arange(5)
    st, ex = O.append_rope(b, pos, 100.0, "bf16"), O.append_rope(b, pos, 100.0)
    assert np.array_equal(torch.from_numpy(st).to(torch.bfloat16).double().numpy(), st)
    assert (np.abs(st - ex) <= 2.0 ** -8 * np.abs(ex) * (1 + 1e-12)).all()


# --------------------------------------------------------------------------- factorized decode query
def _rand_q_factors(seed, rq, h, d):
    g = np.random.default_rng(seed)
    return g.standard_normal((rq, h)), g.standard_normal((rq, d))


def pin_factored_query_rank_one(O):
    """R_Q = 1 with a unit head factor: every head's query is the one rotated B_Q row,
    i.e. the dense decode with q_i = B_Q[0] for all i."""
    c = _rand_case(31, 40, 4, 16, 2, 2)
    _, b_q = _rand_q_factors(32, 1, 4, 16)
    o1 = O.decode_attention_factored_query(c["a_k"], c["b_k"], c["a_v"], c["b_v"], np.ones((1, 4)), b_q, 41.0,
                                           0.25, 10000.0)
    o2 = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], np.repeat(b_q, 4, axis=0), 41.0, 0.25,
                            10000.0)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14)


def pin_factored_query_linearity(O):
    """RoPE is linear, so rotating each B_Q row and then forming (1/R_Q) A_Q^T B~_Q equals
    rotating the summed dense query: the factored decode must equal the dense decode with
    q_i = (1/R_Q) sum_j A_Q[j, i] B_Q[j] (summed here by explicit loops)."""
    c = _rand_case(33, 37, 3, 8, 1, 2)
    rq = 3
    a_q, b_q = _rand_q_factors(34, rq, 3, 8)
    q = np.zeros((3, 8))
    for i in range(3):
        for k in range(8):
            q[i, k] = math.fsum(a_q[j, i] * b_q[j, k] for j in range(rq)) / rq
    o1 = O.decode_attention_factored_query(c["a_k"], c["b_k"], c["a_v"], c["b_v"], a_q, b_q, 777.0, 0.3, 10000.0)
    o2 = O.decode_attention(c["a_k"], c["b_k"], c["a_v"], c["b_v"], q, 777.0, 0.3, 10000.0)
    assert np.allclose(o1, o2, rtol=1e-11, atol=1e-13)


def pin_factored_query_duplicate_ranks(O):
    """R_Q copies of one rank equal the single rank (the 1/R_Q sits in the product)."""
    c = _rand_case(35, 20, 4, 8, 2, 1)
    a_q, b_q = _rand_q_factors(36, 1, 4, 8)
    o1 = O.decode_attention_factored_query(c["a_k"], c["b_k"], c["a_v"], c["b_v"], a_q, b_q, 20.0, 0.5, 10000.0)
    for r in (2, 6):
        o2 = O.decode_attention_factored_query(c["a_k"], c["b_k"], c["a_v"], c["b_v"], np.repeat(a_q, r, axis=0),
                                               np.repeat(b_q, r, axis=0), 20.0, 0.5, 10000.0)
        assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14)


def pin_factored_query_brute_force(O):
    """Tiny case by scalar loops: rotate each B_Q row pair by pair, weight by A_Q / R_Q,
    expand K and V token by token, softmax with math.fsum."""
    c = _rand_case(37, 3, 2, 4, 2, 1)
    rq, h, d, L, qp, scale, base = 2, 2, 4, 3, 5.0, 0.7, 100.0
    a_q, b_q = _rand_q_factors(38, rq, h, d)
    qr = np.zeros((h, d))
    for j in range(rq):
        rot = _brute_rot(b_q[j], qp, base)
        for i in range(h):
            for k in range(d):
                qr[i, k] += a_q[j, i] * rot[k] / rq
    want = np.zeros((h, d))
    for i in range(h):
        z = []
        for s in range(L):
            kk = [math.fsum(c["a_k"][s, r, i] * c["b_k"][s, r, k] for r in range(2)) / 2 for k in range(d)]
            z.append(scale * math.fsum(qr[i, k] * kk[k] for k in range(d)))
        mz = max(z)
        e = [math.exp(v - mz) for v in z]
        tot = math.fsum(e)
        for k in range(d):
            want[i, k] = math.fsum(e[s] / tot * c["a_v"][s, 0, i] * c["b_v"][s, 0, k] for s in range(L))
    got = O.decode_attention_factored_query(c["a_k"], c["b_k"], c["a_v"], c["b_v"], a_q, b_q, qp, scale, base)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------- decode step (append + attend)
def _step_case(seed, L, h, d, rk, rv):
    g = np.random.default_rng(seed)
    c = _rand_case(seed, L, h, d, rk, rv)
    c.update(new_a_k=g.standard_normal((rk, h)), new_b_k=g.standard_normal((rk, d)) / math.sqrt(d),
             new_a_v=g.standard_normal((rv, h)), new_b_v=g.standard_normal((rv, d)) / math.sqrt(d))
    return c


def pin_step_empty_cache(O):
    """With nothing cached the token attends only itself (softmax over one key is 1):
    o_i = (1/R_V) sum_r A_V[r, i] B_V[r], summed here by explicit loops, whatever the query."""
    for rk, rv in ((1, 1), (2, 3)):
        c = _step_case(41 + rk, 0, 3, 8, rk, rv)
        o, _ = O.decode_step(c["a_k"], c["b_k"], c["a_v"], c["b_v"], c["new_a_k"], c["new_b_k"], c["new_a_v"],
                             c["new_b_v"], 12.0, 0.4, 10000.0, q=c["q"])
        for i in range(3):
            for k in range(8):
                want = math.fsum(c["new_a_v"][r, i] * c["new_b_v"][r, k] for r in range(rv)) / rv
                assert abs(o[i, k] - want) <= 1e-14 * (1 + abs(want))


def pin_step_brute_force(O):
    """Tiny steps by scalar loops: the old keys rotated at their own positions, the new key
    and the query both rotated at the step's position, softmax over old + new with math.fsum;
    dense and TPA-form queries.  The stored new row, when rounded to bf16, is a bf16 value
    within half an ulp of the exact rotation."""
    h, d, rk, rv, L = 2, 4, 2, 1, 3
    c = _step_case(45, L, h, d, rk, rv)
    kpos = [2.0, 5.0, 9.0]
    pos, scale, base = 11.0, 0.6, 100.0
    old_rot = O.append_rope(c["b_k"], np.array(kpos), base)
    a_q, b_q = _rand_q_factors(46, 2, h, d)
    for form in ("dense", "factored"):
        if form == "dense":
            o, row = O.decode_step(c["a_k"], old_rot, c["a_v"], c["b_v"], c["new_a_k"], c["new_b_k"], c["new_a_v"],
                                   c["new_b_v"], pos, scale, base, q=c["q"])
            qr = [_brute_rot(list(c["q"][i]), pos, base) for i in range(h)]
        else:
            o, row = O.decode_step(c["a_k"], old_rot, c["a_v"], c["b_v"], c["new_a_k"], c["new_b_k"], c["new_a_v"],
                                   c["new_b_v"], pos, scale, base, a_q=a_q, b_q=b_q)
            rots = [_brute_rot(list(b_q[j]), pos, base) for j in range(2)]
            qr = [[math.fsum(a_q[j, i] * rots[j][k] for j in range(2)) / 2 for k in range(d)] for i in range(h)]
        for i in range(h):
            keys, vals = [], []
            for s in range(L + 1):
                ak = c["a_k"][s] if s < L else c["new_a_k"]
                bk = c["b_k"][s] if s < L else c["new_b_k"]
                av = c["a_v"][s] if s < L else c["new_a_v"]
                bv = c["b_v"][s] if s < L else c["new_b_v"]
                p_s = kpos[s] if s < L else pos
                rot = [_brute_rot(list(bk[r]), p_s, base) for r in range(rk)]
                keys.append([math.fsum(ak[r, i] * rot[r][k] for r in range(rk)) / rk for k in range(d)])
                vals.append([math.fsum(av[r, i] * bv[r, k] for r in range(rv)) / rv for k in range(d)])
            z = [scale * math.fsum(qr[i][k] * key[k] for k in range(d)) for key in keys]
            m = max(z)
            w = [math.exp(x - m) for x in z]
            tot = math.fsum(w)
            for k in range(d):
                want = math.fsum(w[s] / tot * vals[s][k] for s in range(L + 1))
                assert abs(o[i, k] - want) <= 1e-12 * (1 + abs(want)), (form, i, k)
        exact = np.array([_brute_rot(list(c["new_b_k"][r]), pos, base) for r in range(rk)])
        assert np.allclose(row, exact, rtol=1e-14, atol=1e-15)
    _, st = O.decode_step(c["a_k"], old_rot, c["a_v"], c["b_v"], c["new_a_k"], c["new_b_k"], c["new_a_v"],
                          c["new_b_v"], pos, scale, base, q=c["q"], storage="bf16")
    assert np.array_equal(torch.from_numpy(st).to(torch.bfloat16).double().numpy(), st)
    assert (np.abs(st - exact) <= 2.0 ** -8 * np.abs(exact) * (1 + 1e-12)).all()


def pin_step_shift_invariance(O):
    """Theorem 3.1: scores depend on position differences only, so moving every cached
    token and the step's token by the same offset leaves the step's output unchanged."""
    c = _step_case(47, 30, 4, 16, 2, 2)
    kpos = np.arange(30, dtype=np.float64) * 3 + 1
    a_q, b_q = _rand_q_factors(48, 3, 4, 16)
    for shift in (0.0, 517.0):
        rot = O.append_rope(c["b_k"], kpos + shift, 10000.0)
        args = (c["a_k"], rot, c["a_v"], c["b_v"], c["new_a_k"], c["new_b_k"], c["new_a_v"], c["new_b_v"],
                95.0 + shift, 0.5, 10000.0)
        od, _ = O.decode_step(*args, q=c["q"])
        of, _ = O.decode_step(*args, a_q=a_q, b_q=b_q)
        if shift == 0.0:
            ref_d, ref_f = od, of
    assert np.allclose(od, ref_d, rtol=1e-9, atol=1e-12)
    assert np.allclose(of, ref_f, rtol=1e-9, atol=1e-12)


# --------------------------------------------------------------------------- token-sharded decode (lse merge)
def pin_lse_brute_force(O):
    """The log-sum-exp of each head's scaled scores by scalar loops (math.exp, math.fsum,
    math.log), and -inf with nothing cached."""
    c = _rand_case(51, 4, 2, 4, 2, 1)
    kpos = [1.0, 4.0, 6.0, 9.0]
    qpos, scale, base = 12.0, 0.8, 100.0
    rot = O.append_rope(c["b_k"], np.array(kpos), base)
    o, lse = O.decode_attention_lse(c["a_k"], rot, c["a_v"], c["b_v"], c["q"], qpos, scale, base)
    for i in range(2):
        qr = _brute_rot(list(c["q"][i]), qpos, base)
        z = []
        for s in range(4):
            key = [math.fsum(c["a_k"][s, r, i] * _brute_rot(list(c["b_k"][s, r]), kpos[s], base)[k] for r in range(2)) / 2
                   for k in range(4)]
            z.append(scale * math.fsum(qr[k] * key[k] for k in range(4)))
        want = math.log(math.fsum(math.exp(v) for v in z))
        assert abs(lse[i] - want) <= 1e-13 * (1 + abs(want)), (i, lse[i], want)
    o0, l0 = O.decode_attention_lse(c["a_k"][:0], rot[:0], c["a_v"][:0], c["b_v"][:0], c["q"], qpos, scale, base)
    assert (o0 == 0).all() and np.isneginf(l0).all()


def pin_merge_lse_union(O):
    """Softmax over a disjoint union: decoding the token range in shards (global positions,
    an empty shard among them) and merging (o, lse) gives the decode of the whole range,
    and the lse of the whole."""
    c = _rand_case(53, 61, 4, 16, 2, 2)
    pos = np.arange(61, dtype=np.float64) * 2 + 3
    rot = O.append_rope(c["b_k"], pos, 10000.0)
    args = (200.0, 0.4, 10000.0)
    whole, whole_lse = O.decode_attention_lse(c["a_k"], rot, c["a_v"], c["b_v"], c["q"], *args)
    cuts = [0, 17, 17, 40, 61]
    parts = [O.decode_attention_lse(c["a_k"][a:e], rot[a:e], c["a_v"][a:e], c["b_v"][a:e], c["q"], *args)
             for a, e in zip(cuts[:-1], cuts[1:])]
    o, lse = O.merge_lse([p[0] for p in parts], [p[1] for p in parts])
    assert np.allclose(o, whole, rtol=1e-12, atol=1e-14)
    assert np.allclose(lse, whole_lse, rtol=1e-13, atol=1e-13)
    assert np.allclose(o, O.decode_attention(c["a_k"], rot, c["a_v"], c["b_v"], c["q"], *args), rtol=1e-12,
                       atol=1e-14)
    o1, l1 = O.merge_lse([whole], [whole_lse])                      # one part: itself
    assert np.allclose(o1, whole, rtol=1e-15, atol=0) and np.allclose(l1, whole_lse, rtol=1e-15, atol=0)
    oe, le = O.merge_lse([np.zeros_like(whole)] * 2, [np.full(4, -np.inf)] * 2)   # no tokens anywhere
    assert (oe == 0).all() and np.isneginf(le).all()


ALL_PINS = [
    pin_storage_rounding,
    pin_cache_size,
    pin_rope_closed_form,
    pin_rope_complex,
    pin_theorem_3_1,
    pin_two_token_golden,
    pin_single_token,
    pin_zero_query_mean,
    pin_duplicate_ranks,
    pin_factor_rescale,
    pin_mqa_sdpa,
    pin_general_sdpa,
    pin_prefill_causal_sdpa,
    pin_brute_force_decode,
    pin_brute_force_from_unrotated,
    pin_brute_force_prefill,
    pin_prefill_first_row,
    pin_factored_query_rank_one,
    pin_factored_query_linearity,
    pin_factored_query_duplicate_ranks,
    pin_factored_query_brute_force,
    pin_step_empty_cache,
    pin_step_brute_force,
    pin_step_shift_invariance,
    pin_lse_brute_force,
    pin_merge_lse_union,
]
