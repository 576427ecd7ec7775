"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

A pin set that let one of these through would not be pinning the oracle.
"""
import numpy as np
import pytest

import oracle.tpa_oracle as O
from tests.oracle_pins import ALL_PINS

_rope = O.rope
_tp = O.tensor_product
_freq = O.rope_frequencies
_decode = O.decode_attention
_prefill_q = O.prefill_queries
_round = O.round_to_storage


def _rope_flipped(x, pos, base):              # wrong rotation sense
    return _rope(x, -np.asarray(pos, dtype=np.float64), base)


def _rope_rotate_half(x, pos, base):          # pairs (j, j + d/2) instead of (2j, 2j+1)
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    perm = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
    inv = np.argsort(perm)
    y = x[..., inv]
    return _rope(y, pos, base)[..., perm]


def _freq_no_two(d_h, base):                  # theta_j = base^(-j/d_h)
    j = np.arange(d_h // 2, dtype=np.float64)
    return np.power(np.float64(base), -j / d_h)


def _tp_no_rank_scale(a, b):                  # dropped 1/R
    return _tp(a, b) * np.asarray(a).shape[-2]


def _tp_first_rank_only(a, b):                # dropped terms of the rank sum
    a = np.asarray(a, dtype=np.float64)
    return _tp(a[..., :1, :], np.asarray(b, dtype=np.float64)[..., :1, :])


def _tp_transposed(a, b):                     # head/feature factor roles swapped in a square case
    out = _tp(a, b)
    if out.shape[-1] == out.shape[-2]:
        return np.swapaxes(out, -1, -2)
    return np.flip(out, axis=-2)


def _decode_no_query_rope(a_k, b_k_rot, a_v, b_v, q, q_pos, scale, base, block=8192):
    return _decode(a_k, b_k_rot, a_v, b_v, q, 0.0, scale, base, block)


def _decode_scale_squared(a_k, b_k_rot, a_v, b_v, q, q_pos, scale, base, block=8192):
    return _decode(a_k, b_k_rot, a_v, b_v, q, q_pos, scale * scale, base, block)


def _prefill_q_no_rope(a_q, b_q, q_pos, base):
    return _tp(a_q, b_q)


_factored = O.decode_attention_factored_query


def _factored_no_q_rope(a_k, b_k_rot, a_v, b_v, a_q, b_q, q_pos, scale, base, block=8192):
    return _factored(a_k, b_k_rot, a_v, b_v, a_q, b_q, 0.0, scale, base, block)


def _factored_no_rq_scale(a_k, b_k_rot, a_v, b_v, a_q, b_q, q_pos, scale, base, block=8192):
    return _factored(a_k, b_k_rot, a_v, b_v, np.asarray(a_q) * np.asarray(a_q).shape[0], b_q, q_pos, scale, base,
                     block)


_step = O.decode_step


def _step_parts(a_k, b_k_rot, a_v, b_v, new_a_k, new_rot, new_a_v, new_b_v):
    cat = lambda old, new: np.concatenate([np.asarray(old, dtype=np.float64).reshape((-1,) + np.shape(new)),
                                           np.asarray(new, dtype=np.float64)[None]], axis=0)
    return cat(a_k, new_a_k), cat(b_k_rot, new_rot), cat(a_v, new_a_v), cat(b_v, new_b_v)


def _step_new_key_unrotated(a_k, b_k_rot, a_v, b_v, new_a_k, new_b_k, new_a_v, new_b_v, pos, scale, base, q=None,
                            a_q=None, b_q=None, storage=None):
    nb = O.round_to_storage(np.asarray(new_b_k, dtype=np.float64), storage)
    ak, bk, av, bv = _step_parts(a_k, b_k_rot, a_v, b_v, new_a_k, nb, new_a_v, new_b_v)
    if q is not None:
        return O.decode_attention(ak, bk, av, bv, q, pos, scale, base), nb
    return O.decode_attention_factored_query(ak, bk, av, bv, a_q, b_q, pos, scale, base), nb


def _step_new_key_next_position(a_k, b_k_rot, a_v, b_v, new_a_k, new_b_k, new_a_v, new_b_v, pos, scale, base,
                                q=None, a_q=None, b_q=None, storage=None):
    return _step(a_k, b_k_rot, a_v, b_v, new_a_k, new_b_k, new_a_v, new_b_v, pos + 1, scale, base, q, a_q, b_q,
                 storage)[0], O.append_rope(np.asarray(new_b_k)[None], np.array([pos]), base, storage)[0]


def _step_without_new_token(a_k, b_k_rot, a_v, b_v, new_a_k, new_b_k, new_a_v, new_b_v, pos, scale, base, q=None,
                            a_q=None, b_q=None, storage=None):
    _, row = _step(a_k, b_k_rot, a_v, b_v, new_a_k, new_b_k, new_a_v, new_b_v, pos, scale, base, q, a_q, b_q, storage)
    if q is not None:
        return O.decode_attention(a_k, b_k_rot, a_v, b_v, q, pos, scale, base), row
    return O.decode_attention_factored_query(a_k, b_k_rot, a_v, b_v, a_q, b_q, pos, scale, base), row


_merge = O.merge_lse
_lse = O.decode_attention_lse


def _merge_unnormalised(outs, lses):        # weights exp(lse_r - max) not divided by their sum
    o, lse = _merge(outs, lses)
    lses = np.asarray(lses, dtype=np.float64)
    top = lses.max(axis=0)
    w = np.where(np.isfinite(lses), np.exp(lses - np.where(np.isfinite(top), top, 0.0)[None]), 0.0)
    return o * w.sum(axis=0)[:, None], lse


def _merge_plain_mean(outs, lses):          # parts averaged, lse ignored
    return np.asarray(outs, dtype=np.float64).mean(axis=0), _merge(outs, lses)[1]


def _lse_log2(a_k, b_k_rot, a_v, b_v, q, q_pos, scale, base, block=8192):   # base-2 log-sum-exp
    o, lse = _lse(a_k, b_k_rot, a_v, b_v, q, q_pos, scale, base, block)
    return o, lse / np.log(2.0)


_from_unrot = O.decode_attention_from_unrotated


def _unrot_keys_at_query_position(a_k, b_k, a_v, b_v, positions, q, q_pos, scale, base, storage=None):
    return _from_unrot(a_k, b_k, a_v, b_v, np.full(np.shape(positions), q_pos, dtype=np.float64), q, q_pos, scale,
                       base, storage)


def _unrot_storage_ignored(a_k, b_k, a_v, b_v, positions, q, q_pos, scale, base, storage=None):
    return _from_unrot(a_k, b_k, a_v, b_v, positions, q, q_pos, scale, base, None)


def _unrot_keys_left_unrotated(a_k, b_k, a_v, b_v, positions, q, q_pos, scale, base, storage=None):
    return O.decode_attention(a_k, O.round_to_storage(b_k, storage), a_v, b_v, q, q_pos, scale, base)


def _round_truncate(x, storage):               # truncation instead of round-to-nearest-even
    if storage != "bf16":
        return _round(x, storage)
    x = np.asarray(x, dtype=np.float64)
    mant, expo = np.frexp(x)
    return np.ldexp(np.trunc(np.ldexp(mant, 8)), expo - 8)


def _round_ties_away(x, storage):              # ties away from zero instead of to even
    if storage != "bf16":
        return _round(x, storage)
    x = np.asarray(x, dtype=np.float64)
    mant, expo = np.frexp(x)
    m = np.ldexp(mant, 8)
    return np.ldexp(np.sign(m) * np.floor(np.abs(m) + 0.5), expo - 8)


MUTANTS = {
    "round_truncate": ("round_to_storage", _round_truncate),
    "round_ties_away": ("round_to_storage", _round_ties_away),
    "rope_flipped": ("rope", _rope_flipped),
    "rope_rotate_half": ("rope", _rope_rotate_half),
    "freq_no_two": ("rope_frequencies", _freq_no_two),
    "no_rank_scale": ("tensor_product", _tp_no_rank_scale),
    "first_rank_only": ("tensor_product", _tp_first_rank_only),
    "transposed_product": ("tensor_product", _tp_transposed),
    "decode_no_query_rope": ("decode_attention", _decode_no_query_rope),
    "decode_scale_squared": ("decode_attention", _decode_scale_squared),
    "prefill_no_query_rope": ("prefill_queries", _prefill_q_no_rope),
    "factored_no_query_rope": ("decode_attention_factored_query", _factored_no_q_rope),
    "factored_no_rq_scale": ("decode_attention_factored_query", _factored_no_rq_scale),
    "step_new_key_unrotated": ("decode_step", _step_new_key_unrotated),
    "step_new_key_next_position": ("decode_step", _step_new_key_next_position),
    "step_without_new_token": ("decode_step", _step_without_new_token),
    "merge_unnormalised": ("merge_lse", _merge_unnormalised),
    "merge_plain_mean": ("merge_lse", _merge_plain_mean),
    "lse_log2": ("decode_attention_lse", _lse_log2),
    "unrotated_keys_at_query_position": ("decode_attention_from_unrotated", _unrot_keys_at_query_position),
    "unrotated_storage_ignored": ("decode_attention_from_unrotated", _unrot_storage_ignored),
    "unrotated_keys_left_unrotated": ("decode_attention_from_unrotated", _unrot_keys_left_unrotated),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_some_pin_catches(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(O)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
