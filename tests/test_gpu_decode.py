"""GPU parity of tpa_decode_attention against the float64 oracle.

Two levels: (i) the oracle reads the cache the GPU wrote (so storage rounding
of the rotated B_K is not charged to attention); (ii) end to end, the oracle
starts from the unrotated factors and applies its own RoPE.
"""
import numpy as np
import pytest
import torch

import oracle.tpa_oracle as O
from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T
from tests.gpu_cases import DEV, build_decode_cache, readback
from tests.parity_util import TOL, assert_rows_close, default_scale, f64, oracle_decode_rows

pytestmark = pytest.mark.gpu

KERNELS = [T.TPA_KERNEL_SIMT, T.TPA_KERNEL_AUTO, T.TPA_KERNEL_TENSOR_SYNC]
TENSOR_KERNELS = [T.TPA_KERNEL_TENSOR, T.TPA_KERNEL_TENSOR_SYNC]


def _check(w, cache, x, q, q_pos, out, batches=None, heads=None, end_to_end=True):
    d = w.head_dim
    scale = default_scale(d)
    lengths = x["lengths"].numpy()
    batches = list(range(cache.batch)) if batches is None else list(batches)
    cpu = readback(cache, batches)
    qn = f64(q)[batches]
    ref = oracle_decode_rows(cpu, qn, x["q_pos"].numpy()[batches], lengths[batches], scale, w.rope_base,
                             heads=heads)
    got = f64(out)[batches]
    if heads is not None:
        got = got[:, list(heads)]
    tol = TOL[cache.dtype]
    worst = assert_rows_close(got, ref, tol, f"{w.name} cache-level")
    if end_to_end:
        for n, b in enumerate(batches[:2]):
            L = int(lengths[b])
            sel = slice(None) if heads is None else list(heads)
            ak = f64(x["a_k"][b, :L])[:, :, sel]
            av = f64(x["a_v"][b, :L])[:, :, sel]
            r = O.decode_attention_from_unrotated(ak, f64(x["b_k"][b, :L]), av, f64(x["b_v"][b, :L]),
                                                  np.arange(L), f64(x["q"][b])[sel], float(x["q_pos"][b]),
                                                  scale, w.rope_base, storage=w.dtype)
            assert_rows_close(got[n], r, tol, f"{w.name} end-to-end b={b}")
    return worst


@pytest.mark.parametrize("kernel", [T.TPA_KERNEL_SIMT, T.TPA_KERNEL_AUTO])
def test_tiny_f32_workload(kernel):
    w = S.WORKLOADS["decode_tiny_f32"]
    cache, x, q, q_pos = build_decode_cache(w)
    for splits in (0, 1, 2, 4):
        out = T.tpa_decode_attention(cache, q, q_pos, max_len=64, num_splits=splits, kernel=kernel)
        _check(w, cache, x, q, q_pos, out)
    assert T.tpa_read_device_error() == 0


@pytest.mark.parametrize("kernel", KERNELS)
def test_b8_l8k_workload_full_size(kernel):
    """The full bf16 decode workload (B=8, L=8192); oracle on 6 heads of every sequence."""
    w = S.WORKLOADS["decode_b8_l8k"]
    cache, x, q, q_pos = build_decode_cache(w)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=w.length, kernel=kernel)
    _check(w, cache, x, q, q_pos, out, heads=[0, 5, 13, 21, 30, 31])
    assert T.tpa_read_device_error() == 0


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("lengths", [[0, 1, 2, 63], [64, 65, 127, 129], [1000, 777, 4095, 3]])
@pytest.mark.parametrize("splits", [1, 3, 0])
def test_ragged_lengths_and_splits(kernel, lengths, splits):
    w = S.WORKLOADS["decode_b8_l8k"]
    cache, x, q, q_pos = build_decode_cache(w, batch=4, length=max(lengths) + 5, lengths=lengths)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=max(lengths), num_splits=splits, kernel=kernel)
    _check(w, cache, x, q, q_pos, out, end_to_end=False)
    empty = [b for b, L in enumerate(lengths) if L == 0]
    for b in empty:
        assert torch.count_nonzero(out[b]) == 0
    assert T.tpa_read_device_error() == 0


@pytest.mark.parametrize("kernel", KERNELS)
def test_rank2_varlen_small(kernel):
    w = S.WORKLOADS["decode_b32_var32k"]
    cache, x, q, q_pos = build_decode_cache(w, batch=5, length=3000, min_length=1)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=3000, kernel=kernel)
    _check(w, cache, x, q, q_pos, out)


@pytest.mark.parametrize("h,d,rk,rv,dt", [
    (8, 64, 1, 2, "bf16"), (16, 32, 3, 1, "bf16"), (32, 16, 4, 4, "bf16"),
    (4, 16, 2, 1, "f32"), (12, 128, 1, 1, "f32"), (32, 64, 2, 2, "f32"),
])
def test_other_shapes_simt(h, d, rk, rv, dt):
    w = S.DecodeWorkload("shape", 3, h, d, rk, rv, 700, dt, seed=h + d + rk + rv, min_length=1)
    cache, x, q, q_pos = build_decode_cache(w)
    for splits in (1, 5):
        out = T.tpa_decode_attention(cache, q, q_pos, max_len=700, num_splits=splits)
        _check(w, cache, x, q, q_pos, out)


def test_length_above_max_len_is_reported():
    w = S.WORKLOADS["decode_b8_l8k"]
    cache, x, q, q_pos = build_decode_cache(w, batch=2, length=256)
    T.tpa_decode_attention(cache, q, q_pos, max_len=100, kernel=T.TPA_KERNEL_SIMT)
    assert T.tpa_read_device_error() & T.TPA_DEVERR_LEN_RANGE


_E2E_REFS = {}


def _end_to_end_all_heads(w, x, b, got, kernel):
    """Sequence b on all heads, end to end: the oracle rotates the unrotated factors itself
    (RoPE at each token's position, the stored rows rounded to the cache dtype) and attends
    with its own query RoPE.  The float64 reference is computed once per workload and reused
    by every kernel."""
    key = (w.name, b)
    if key not in _E2E_REFS:
        L = int(x["lengths"][b])
        _E2E_REFS[key] = O.decode_attention_from_unrotated(
            f64(x["a_k"][b, :L]), f64(x["b_k"][b, :L]), f64(x["a_v"][b, :L]), f64(x["b_v"][b, :L]), np.arange(L),
            f64(x["q"][b]), float(x["q_pos"][b]), default_scale(w.head_dim), w.rope_base, storage=w.dtype)
    assert_rows_close(f64(got[b]), _E2E_REFS[key], TOL[torch.bfloat16], f"{w.name} end-to-end b={b} kernel={kernel}")


@pytest.mark.slow
@pytest.mark.parametrize("kernel", KERNELS)
def test_b32_var32k_workload_full_size(kernel):
    """The full R=2 variable-length workload; oracle on 4 sequences x 4 heads at cache level,
    and the longest sequence end to end on all 32 heads."""
    w = S.WORKLOADS["decode_b32_var32k"]
    cache, x, q, q_pos = build_decode_cache(w, nan_tail=False)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=w.length, kernel=kernel)
    L = x["lengths"].numpy()
    picks = [int(np.argmin(L)), int(np.argmax(L)), 7, 19]
    _check(w, cache, x, q, q_pos, out, batches=picks, heads=[0, 11, 22, 31], end_to_end=False)
    _end_to_end_all_heads(w, x, int(np.argmax(L)), out, kernel)
    assert T.tpa_read_device_error() == 0


@pytest.mark.slow
@pytest.mark.parametrize("kernel", KERNELS)
def test_long_512k_workload_full_size(kernel):
    """The long-context workload (B=1, L=524288); oracle on 3 heads at cache level, and end to
    end on all 32 heads."""
    w = S.WORKLOADS["decode_long_512k"]
    cache, x, q, q_pos = build_decode_cache(w, nan_tail=False)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=w.length, kernel=kernel)
    _check(w, cache, x, q, q_pos, out, heads=[0, 17, 31], end_to_end=False)
    _end_to_end_all_heads(w, x, 0, out, kernel)
    assert T.tpa_read_device_error() == 0


@pytest.mark.parametrize("kernel", TENSOR_KERNELS)
@pytest.mark.parametrize("grid", [1, 2, 5, 37, 148, 300])
@pytest.mark.parametrize("name", ["decode_b8_l8k", "decode_b32_var32k"])
def test_tensor_kernel_partition_grids(kernel, grid, name):
    """The tensor-core kernel's even split of all tiles over `grid` CTAs: sequences spanning
    many CTAs, CTAs spanning many sequences, empty sequences, more CTAs than tiles."""
    w = S.WORKLOADS[name]
    lengths = [5000, 1, 0, 64, 65, 130, 3000, 7]
    cache, x, q, q_pos = build_decode_cache(w, batch=8, length=5000, lengths=lengths)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=5000, num_splits=grid, kernel=kernel)
    _check(w, cache, x, q, q_pos, out, end_to_end=False)
    assert torch.count_nonzero(out[2]) == 0
    assert T.tpa_read_device_error() == 0


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("grid", [0, 5, 300])
def test_workspace_contents_do_not_matter(kernel, grid):
    """A workspace full of NaN (unwritten partial slots included) gives the same result."""
    w = S.WORKLOADS["decode_b8_l8k"]
    cache, x, q, q_pos = build_decode_cache(w, batch=4, length=600, lengths=[600, 1, 0, 333])
    nbytes = T.tpa_decode_workspace_size(cache, 600, grid, kernel)
    ws = torch.full((max(nbytes, 4) // 4,), float("nan"), dtype=torch.float32, device=DEV).view(torch.uint8)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=600, num_splits=grid, kernel=kernel, workspace_buf=ws)
    _check(w, cache, x, q, q_pos, out, end_to_end=False)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("rank", [1, 2])
def test_unit_variance_factors(kernel, rank):
    """B factors ~ N(0, 1) (the prefill workload's scale): scores ~10x larger than the decode
    workloads'.  A single bf16 rounding of the rotated query would exceed 2e-3 here."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="unit_var", r_k=rank, r_v=rank, b_std=1.0, seed=77)
    cache, x, q, q_pos = build_decode_cache(w, batch=3, length=4000, min_length=1000)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=4000, kernel=kernel)
    _check(w, cache, x, q, q_pos, out)


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("rank", [1, 2])
@pytest.mark.parametrize("direction", [1, -1])
def test_score_ramp(kernel, rank, direction):
    """Scores that climb steadily along the sequence (direction 1: the running maximum grows on
    almost every tile, so every rescale path runs) or fall (direction -1: the first tile holds
    the maximum).  B_K is overwritten with multiples of the rotated query; the oracle reads the
    cache back, so only the attention is compared."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="ramp", r_k=rank, r_v=rank, seed=91)
    lengths = [4000, 2500, 129]
    cache, x, q, q_pos = build_decode_cache(w, batch=3, length=4000, lengths=lengths)
    for b, L in enumerate(lengths):
        qr = O.rope(f64(q[b]).astype(np.float64), float(q_pos[b]), w.rope_base)  # [h, d]
        u = qr.mean(axis=0)
        u /= np.linalg.norm(u)
        ramp = np.arange(L, dtype=np.float64) / L
        if direction < 0:
            ramp = ramp[::-1].copy()
        # head-averaged query direction times a ramp: scores span ~60 natural-log units per head
        bk = (60.0 * np.sqrt(w.head_dim) / np.abs(qr @ u).max()) * ramp[:, None, None] * u[None, None, :]
        bk = np.repeat(bk, rank, axis=1)
        cache.b_k[b, :L] = torch.from_numpy(bk).to(cache.b_k.dtype).to(DEV)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=4000, kernel=kernel)
    _check(w, cache, x, q, q_pos, out, end_to_end=False)
    assert T.tpa_read_device_error() == 0


@pytest.mark.parametrize("rank", [1, 2])
@pytest.mark.parametrize("r_q,q_scale", [(1, 1.0), (6, 1.0), (8, 1.0), (6, 3.0)])
def test_factored_query_decode(rank, r_q, q_scale):
    """Decode with the query in TPA form (A_Q, B_Q; the full-TPA variant) against the oracle's
    factored decode, on ragged lengths (empty and one-token sequences included).  B_Q rows are
    scaled so that the summed query has about unit (or q_scale^2) variance per element."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="factored", r_k=rank, r_v=rank, seed=60 + r_q)
    lengths = [1000, 1, 0, 333, 4000, 129]
    cache, x, q, q_pos = build_decode_cache(w, batch=6, length=4000, lengths=lengths)
    g = S.rng(w.seed, 17)
    a_q = S.to_storage(g.standard_normal((6, r_q, w.heads), dtype=np.float32), "bf16").to(DEV)
    b_q = S.to_storage(g.standard_normal((6, r_q, w.head_dim), dtype=np.float32) *
                       np.float32(q_scale * np.sqrt(r_q)), "bf16").to(DEV)
    out = T.tpa_decode_attention_factored(cache, a_q, b_q, q_pos, max_len=4000)
    cpu = readback(cache)
    scale = default_scale(w.head_dim)
    got = f64(out)
    for b, L in enumerate(lengths):
        ref = O.decode_attention_factored_query(cpu["a_k"][b, :L], cpu["b_k"][b, :L], cpu["a_v"][b, :L],
                                                cpu["b_v"][b, :L], f64(a_q[b]), f64(b_q[b]), float(q_pos[b]),
                                                scale, w.rope_base)
        if L == 0:
            assert torch.count_nonzero(out[b]) == 0
            continue
        assert_rows_close(got[b], ref, TOL[torch.bfloat16], f"factored r_q={r_q} b={b}")
    assert T.tpa_read_device_error() == 0


def test_factored_query_rank_one_matches_dense_decode():
    """R_Q = 1 with A_Q = 1 is the dense decode with q = B_Q for every head (same kernel path
    for the attention; only the query stage differs)."""
    w = S.WORKLOADS["decode_b8_l8k"]
    cache, x, q, q_pos = build_decode_cache(w, batch=3, length=2000, min_length=100)
    b_q = q[:, :1, :].contiguous()
    a_q = torch.ones(3, 1, w.heads, dtype=torch.bfloat16, device=DEV)
    o_f = T.tpa_decode_attention_factored(cache, a_q, b_q, q_pos, max_len=2000)
    o_d = T.tpa_decode_attention(cache, b_q.expand(3, w.heads, w.head_dim).contiguous(), q_pos, max_len=2000,
                                 kernel=T.TPA_KERNEL_TENSOR)
    assert torch.equal(o_f, o_d)


@pytest.mark.parametrize("kernel", KERNELS)
def test_maximum_batch(kernel):
    """The largest batch the tensor-core decodes take (1024 sequences), short ragged lengths with
    empty ones among them, so that CTAs span many sequences; the oracle on a sample of them."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="max_batch", seed=131)
    g = np.random.default_rng(131)
    lengths = g.integers(0, 300, size=1024)
    lengths[::97] = 0
    lengths[5] = 300
    cache, x, q, q_pos = build_decode_cache(w, batch=1024, length=300, lengths=lengths.tolist(), nan_tail=False)
    out = T.tpa_decode_attention(cache, q, q_pos, max_len=300, kernel=kernel)
    assert T.tpa_read_device_error() == 0
    sample = sorted(set(g.choice(1024, 48, replace=False).tolist()) | {0, 5, 97, 1023})
    _check(w, cache, x, q, q_pos, out, batches=sample, end_to_end=False)
    for b in np.nonzero(lengths == 0)[0]:
        assert torch.count_nonzero(out[b]) == 0
