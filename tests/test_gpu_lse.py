"""GPU parity of tpa_decode_attention_lse and tpa_merge_lse (the token-sharded decode):
the log-sum-exp against the oracle, and shards of one cache, emulated on one GPU, merged
back into the decode of the whole range."""
import numpy as np
import pytest
import torch

import oracle.tpa_oracle as O
from factorized_kv_cache_b200 import sharded
from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T
from tests.gpu_cases import DEV, build_decode_cache, readback
from tests.parity_util import TOL, assert_rows_close, default_scale, f64

pytestmark = pytest.mark.gpu

BF16 = TOL[torch.bfloat16]


def _lse_close(got, ref, what):
    """lse is a log: an absolute error e is a relative error e in exp(lse)."""
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    assert np.array_equal(np.isneginf(got), np.isneginf(ref)), what
    fin = np.isfinite(ref)
    if fin.any():
        err = np.abs(got[fin] - ref[fin]).max()
        assert err <= BF16, f"{what}: lse error {err:.3e}"


@pytest.mark.parametrize("rank", [1, 2])
@pytest.mark.parametrize("splits", [0, 1, 5, 300])
def test_decode_lse_matches_oracle(rank, splits):
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="lse", r_k=rank, r_v=rank, seed=90 + rank)
    lengths = [1000, 0, 1, 127, 128, 4000]
    cache, x, q, q_pos = build_decode_cache(w, batch=6, length=4000, lengths=lengths)
    out, lse = T.tpa_decode_attention_lse(cache, q, q_pos, max_len=4000, num_splits=splits)
    plain = T.tpa_decode_attention(cache, q, q_pos, max_len=4000, num_splits=splits, kernel=T.TPA_KERNEL_TENSOR)
    assert T.tpa_read_device_error() == 0
    assert torch.equal(out, plain)                      # the same kernels; lse is an extra output
    cpu = readback(cache)
    scale = default_scale(w.head_dim)
    for b, L in enumerate(lengths):
        o, l = O.decode_attention_lse(cpu["a_k"][b, :L], cpu["b_k"][b, :L], cpu["a_v"][b, :L], cpu["b_v"][b, :L],
                                      f64(q[b]), float(q_pos[b]), scale, w.rope_base)
        _lse_close(f64(lse[b]), l, f"lse R={rank} splits={splits} b={b}")
        if L:
            assert_rows_close(f64(out[b]), o, BF16, f"out b={b}")


def _shard_cache(cache, start, end):
    """A cache holding tokens [start, end) of every sequence of `cache` (clipped to its
    length), at their global positions: what one rank of a token-sharded decode holds."""
    cap = max(1, end - start)
    planes = [getattr(cache, k)[:, start:start + cap].clone() for k in ("a_k", "b_k", "a_v", "b_v")]
    lens = (cache.seq_lens.clamp(max=end) - start).clamp(min=0).to(torch.int32)
    return T.TpaCache(*planes, lens, rope_base=cache.rope_base)


@pytest.mark.parametrize("world", [2, 3, 8])
def test_token_sharded_decode_emulated_on_one_gpu(world):
    """Every rank's token range as its own cache on this GPU; (out, lse) stacked as an
    all-gather lays them out; tpa_merge_lse gives the whole decode."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="sharded", seed=95)
    lengths = [5000, 3, 0, 2048]
    cache, x, q, q_pos = build_decode_cache(w, batch=4, length=5000, lengths=lengths)
    whole, whole_lse = T.tpa_decode_attention_lse(cache, q, q_pos, max_len=5000)
    parts_out, parts_lse = [], []
    for r in range(world):
        s, e = sharded.token_range(5000, world, r)
        sc = _shard_cache(cache, s, e)
        o, l = T.tpa_decode_attention_lse(sc, q, q_pos, max_len=sc.capacity)
        parts_out.append(o)
        parts_lse.append(l)
    merged, merged_lse = T.tpa_merge_lse(torch.stack(parts_out), torch.stack(parts_lse))
    assert T.tpa_read_device_error() == 0
    assert_rows_close(f64(merged), f64(whole), 1e-4, f"{world} shards vs whole")
    _lse_close(f64(merged_lse), f64(whole_lse), "merged lse")
    cpu = readback(cache)
    scale = default_scale(w.head_dim)
    for b, L in enumerate(lengths):
        ref = O.decode_attention(cpu["a_k"][b, :L], cpu["b_k"][b, :L], cpu["a_v"][b, :L], cpu["b_v"][b, :L],
                                 f64(q[b]), float(q_pos[b]), scale, w.rope_base)
        if L == 0:
            assert torch.count_nonzero(merged[b]) == 0
            continue
        assert_rows_close(f64(merged[b]), ref, BF16, f"{world} shards b={b}")


@pytest.mark.parametrize("head_dim", [16, 64, 128])
@pytest.mark.parametrize("n_parts", [1, 2, 7, 40])
def test_merge_lse_against_oracle(head_dim, n_parts):
    """Random partial results, some parts and one whole row without tokens (lse = -inf)."""
    g = np.random.default_rng(head_dim + n_parts)
    rows = 37
    outs = g.standard_normal((n_parts, rows, head_dim)).astype(np.float32)
    lses = (g.standard_normal((n_parts, rows)) * 5).astype(np.float32)
    lses[g.random((n_parts, rows)) < 0.2] = -np.inf
    lses[:, 3] = -np.inf
    o, l = T.tpa_merge_lse(torch.from_numpy(outs).to(DEV), torch.from_numpy(lses).to(DEV))
    ro, rl = O.merge_lse(outs.astype(np.float64), lses.astype(np.float64))
    got = f64(o)
    assert np.abs(got - ro).max() <= 2e-6 * (1 + np.abs(ro).max())
    assert (got[3] == 0).all()
    _lse_close(f64(l), rl, "merge lse")


def test_merge_lse_long_workload_in_shards():
    """The long-context workload (B=1, L=524288) as 4 token ranges on this GPU, merged;
    against the unsharded decode, and the oracle on sampled heads."""
    w = S.WORKLOADS["decode_long_512k"]
    cache, x, q, q_pos = build_decode_cache(w, nan_tail=False)
    L = int(x["lengths"][0])
    whole = T.tpa_decode_attention(cache, q, q_pos, max_len=L)
    parts = [T.tpa_decode_attention_lse(_shard_cache(cache, *sharded.token_range(L, 4, r)), q, q_pos,
                                        max_len=sharded.token_range(L, 4, r)[1] - sharded.token_range(L, 4, r)[0])
             for r in range(4)]
    merged, _ = T.tpa_merge_lse(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    assert T.tpa_read_device_error() == 0
    assert_rows_close(f64(merged), f64(whole), 1e-4, "long workload, 4 shards vs whole")
    heads = [0, 17, 31]
    cpu = readback(cache)
    ref = O.decode_attention(cpu["a_k"][0, :L][:, :, heads], cpu["b_k"][0, :L], cpu["a_v"][0, :L][:, :, heads],
                             cpu["b_v"][0, :L], f64(q[0])[heads], float(q_pos[0]), default_scale(w.head_dim),
                             w.rope_base)
    assert_rows_close(f64(merged[0])[heads], ref, BF16, "long workload vs oracle")


def test_decode_token_sharded_through_a_process_group():
    """sharded.decode_token_sharded end to end through torch.distributed (a one-rank NCCL
    group: the all-gather runs, the merge combines one part) equals the plain decode."""
    import os
    import socket

    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device(DEV, 0))
    try:
        w = S.WORKLOADS["decode_b8_l8k"].replace(name="sharded_pg", seed=97)
        cache, x, q, q_pos = build_decode_cache(w, batch=3, length=3000, lengths=[3000, 0, 1700])
        out, lse = sharded.decode_token_sharded(cache, q, q_pos, max_len=3000)
        ref, ref_lse = T.tpa_decode_attention_lse(cache, q, q_pos, max_len=3000)
        assert T.tpa_read_device_error() == 0
        assert torch.equal(out, ref)
        assert torch.equal(lse, ref_lse)
    finally:
        dist.destroy_process_group()
