"""Token-sharded decode on CPU: gloo ranks (no GPU) run the oracle on their token range,
exchange (out, lse) with the all-gather of factorized_kv_cache_b200.sharded, and merge; the
result must be the decode of the whole range.  Also the split of a range into shares."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.tpa_oracle as O
from factorized_kv_cache_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("length", [0, 1, 5, 7, 64, 1001])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_token_ranges_cover_the_range_once(length, world):
    ranges = [sharded.token_range(length, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == length
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))     # contiguous, in rank order
    sizes = [e - s for s, e in ranges]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == length


def test_token_range_rejects_bad_ranks():
    with pytest.raises(ValueError):
        sharded.token_range(10, 2, 2)
    with pytest.raises(ValueError):
        sharded.token_range(10, 0, 0)


def _case(lengths, h=4, d=16, r=2, seed=61):
    g = np.random.default_rng(seed)
    L = max(lengths)
    c = dict(a_k=g.standard_normal((len(lengths), L, r, h)), b_k=g.standard_normal((len(lengths), L, r, d)) / math.sqrt(d),
             a_v=g.standard_normal((len(lengths), L, r, h)), b_v=g.standard_normal((len(lengths), L, r, d)) / math.sqrt(d),
             q=g.standard_normal((len(lengths), h, d)))
    c["b_k"] = O.append_rope(c["b_k"], np.broadcast_to(np.arange(L, dtype=np.float64), (len(lengths), L)), 10000.0)
    return c


def _worker(rank, world, port, lengths, res):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = _case(lengths)
        outs, lses = [], []
        for b, L in enumerate(lengths):
            s, e = sharded.token_range(L, world, rank)
            o, l = O.decode_attention_lse(c["a_k"][b, s:e], c["b_k"][b, s:e], c["a_v"][b, s:e], c["b_v"][b, s:e],
                                          c["q"][b], float(L), 0.25, 10000.0)
            outs.append(o)
            lses.append(l)
        parts_out, parts_lse = sharded.all_gather_partials(torch.from_numpy(np.stack(outs)),
                                                           torch.from_numpy(np.stack(lses)))
        assert tuple(parts_out.shape) == (world, len(lengths), 4, 16)
        worst = 0.0
        for b, L in enumerate(lengths):
            o, l = O.merge_lse(parts_out[:, b].numpy(), parts_lse[:, b].numpy())
            ref, ref_l = O.decode_attention_lse(c["a_k"][b, :L], c["b_k"][b, :L], c["a_v"][b, :L], c["b_v"][b, :L],
                                                c["q"][b], float(L), 0.25, 10000.0)
            worst = max(worst, float(np.abs(o - ref).max()))
            same_inf = np.array_equal(np.isneginf(l), np.isneginf(ref_l))
            fin = np.isfinite(ref_l)
            worst = max(worst, 0.0 if not fin.any() else float(np.abs(l[fin] - ref_l[fin]).max()),
                        0.0 if same_inf else 1.0)
        res[rank] = worst
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_with_gloo_ranks_equals_the_whole(world):
    lengths = [40, 2, 0, 17]          # some ranks hold nothing of the short sequences
    res = mp.get_context("spawn").Array("d", world)
    mp.spawn(_worker, args=(world, _free_port(), lengths, res), nprocs=world, join=True)
    assert max(res) <= 1e-12, list(res)
