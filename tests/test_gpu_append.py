"""GPU parity of tpa_cache_append against the oracle's RoPE (section RoPE 兼容性)."""
import numpy as np
import pytest
import torch

import oracle.tpa_oracle as O
from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T
from tests.parity_util import f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(dtype, B, n, h, d, rk, rv, seed):
    g = S.rng(seed, 9)
    sd = "f32" if dtype == torch.float32 else "bf16"
    mk = lambda *s, std=1.0: S.to_storage(g.standard_normal(s, dtype=np.float32) * np.float32(std), sd).to(DEV)
    return mk(B, n, rk, h), mk(B, n, rk, d, std=d ** -0.5), mk(B, n, rv, h), mk(B, n, rv, d, std=d ** -0.5)


def _bf16_midpoint_distance(y):
    """Distance from each value to the nearest midpoint between adjacent bf16 values (8
    significant bits: within the binade of |y| the bf16 spacing is 2^(e - 8) for y = m 2^e,
    0.5 <= |m| < 1; the midpoint below the next power of two lies in the same binade)."""
    y = np.abs(np.asarray(y, dtype=np.float64))
    _, e = np.frexp(y)
    ulp = np.ldexp(1.0, e - 8)
    r = y / ulp
    return np.abs(r - np.floor(r) - 0.5) * ulp


def test_bf16_midpoint_distance():
    """The helper on values whose distance to a bf16 midpoint is known."""
    u = 2.0 ** -7                                   # bf16 spacing in [1, 2)
    vals = np.array([1.0, 1.0 + u / 2, 1.0 + u / 4, -(1.5 + u / 2), 2.0 - u / 2, 0.75 + 2.0 ** -9])
    want = np.array([u / 2, 0.0, u / 4, 0.0, 0.0, 0.0])
    assert np.allclose(_bf16_midpoint_distance(vals), want, rtol=0, atol=1e-18)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n_new", [1, 5, 32, 33, 300])
@pytest.mark.parametrize("rk,rv", [(1, 1), (2, 2), (1, 3)])
def test_append_matches_oracle(dtype, n_new, rk, rv):
    B, cap, h, d = 3, 400, 32, 128
    cache = T.TpaCache.allocate(B, cap, h, d, rk, rv, dtype=dtype, fill=float("nan"))
    start = torch.tensor([0, 7, 99], dtype=torch.int32, device=DEV)
    cache.seq_lens.copy_(start)
    a_k, b_k, a_v, b_v = _inputs(dtype, B, n_new, h, d, rk, rv, seed=n_new + 10 * rk + rv)
    g = np.random.default_rng(n_new)
    pos = torch.from_numpy(g.integers(0, 524288, size=(B, n_new)).astype(np.int32)).to(DEV)
    T.tpa_cache_append(cache, pos, a_k, b_k, a_v, b_v)
    assert T.tpa_read_device_error() == 0
    assert cache.seq_lens.tolist() == [s + n_new for s in start.tolist()]
    ref_bk = O.append_rope(f64(b_k), f64(pos), cache.rope_base)        # [B, n, rk, d]
    for b in range(B):
        s0 = int(start[b])
        sl = slice(s0, s0 + n_new)
        assert torch.equal(cache.a_k[b, sl], a_k[b])
        assert torch.equal(cache.a_v[b, sl], a_v[b])
        assert torch.equal(cache.b_v[b, sl], b_v[b])
        got = f64(cache.b_k[b, sl])
        ref = ref_bk[b]
        x = f64(b_k[b])
        pair_norm = np.sqrt(x[..., 0::2] ** 2 + x[..., 1::2] ** 2).repeat(2, axis=-1)
        rot_err = 1e-6 * pair_norm + 1e-12      # the fp32 rotation's error bound (reduced fp64 angle, fp32 sincos)
        if dtype == torch.bfloat16:
            # the stored row is the exact rotation rounded once to bf16 (nearest, ties to even), as the
            # oracle's append_rope(..., storage="bf16") models it: equal bit for bit, except where the
            # exact rotation lies within the rotation error of a bf16 rounding midpoint (either
            # neighbour is then a correct rounding of the kernel's fp32 value)
            want = O.append_rope(f64(b_k[b]), f64(pos[b]), cache.rope_base, "bf16")
            near = _bf16_midpoint_distance(ref) <= rot_err
            mismatch = got != want
            assert not (mismatch & ~near).any(), np.argwhere(mismatch & ~near)[:5]
            assert near.sum() <= max(4, near.size // 100), (int(near.sum()), near.size)   # about 0.1% expected
            assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + rot_err).all()
        else:
            assert (np.abs(got - ref) <= rot_err).all(), np.abs(got - ref).max()
        # untouched slots keep their NaN
        assert torch.isnan(cache.b_k[b, :s0].float()).all() and torch.isnan(cache.b_k[b, s0 + n_new:].float()).all()


def test_append_overflow_is_reported_and_length_kept():
    B, cap, h, d = 2, 40, 32, 128
    cache = T.TpaCache.allocate(B, cap, h, d, 1, 1, dtype=torch.bfloat16, fill=0.0)
    cache.seq_lens.copy_(torch.tensor([30, 5], dtype=torch.int32))
    for n in (12, 36):   # single-CTA and multi-CTA paths
        a_k, b_k, a_v, b_v = _inputs(torch.bfloat16, B, n, h, d, 1, 1, seed=3)
        pos = torch.zeros(B, n, dtype=torch.int32, device=DEV)
        before = cache.seq_lens.clone()
        T.tpa_cache_append(cache, pos, a_k, b_k, a_v, b_v)
        err = T.tpa_read_device_error()
        assert err & T.TPA_DEVERR_APPEND_OVERFLOW
        assert int(cache.seq_lens[0]) == int(before[0])              # sequence 0 overflowed
        if int(before[1]) + n <= cap:
            assert int(cache.seq_lens[1]) == int(before[1]) + n
    assert T.tpa_read_device_error() == 0                             # read clears the word


def test_rope_identity_holds_on_gpu_written_keys():
    """Theorem 3.1 on the GPU-rotated keys: shifting every position leaves scores unchanged."""
    B, n, h, d = 1, 64, 32, 128
    a_k, b_k, a_v, b_v = _inputs(torch.float32, B, n, h, d, 1, 1, seed=5)
    q = torch.randn(1, h, d, dtype=torch.float32, device=DEV)
    outs = []
    for delta in (0, 1000, 400000):
        cache = T.TpaCache.allocate(B, n, h, d, 1, 1, dtype=torch.float32)
        pos = (torch.arange(n, dtype=torch.int32, device=DEV) + delta)[None]
        T.tpa_cache_append(cache, pos, a_k, b_k, a_v, b_v)
        qp = torch.tensor([n + delta], dtype=torch.int32, device=DEV)
        outs.append(T.tpa_decode_attention(cache, q, qp, max_len=n).cpu())
    for o in outs[1:]:
        assert torch.allclose(o, outs[0], rtol=2e-5, atol=2e-6)
