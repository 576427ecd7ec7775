"""The multi-rank logic of bench.py on CPU: two gloo ranks (no GPU).

Under torchrun every rank runs its own batch (weak scaling, no collective on the
data path); the only cross-rank steps are the timing barrier and the maximum
over ranks of each measured time, which these tests exercise with world size 2.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from factorized_kv_cache_b200 import synthetic as S


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        t_local = [3.0, 7.5][rank]
        dist.barrier()
        out[rank] = bench.max_over_ranks(t_local, world, dev)
        out[world + rank] = bench.max_over_ranks(-1.0 * (rank + 1), world, dev)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    world = 2
    out = mp.get_context("spawn").Array("d", 2 * world)
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert list(out[:world]) == [7.5, 7.5]       # every rank reports the slowest rank's time
    assert list(out[world:]) == [-1.0, -1.0]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(4.25, 1, torch.device("cpu")) == 4.25


@pytest.mark.parametrize("name", ["decode_b8_l8k", "prefill_b4_t4k"])
def test_each_rank_gets_its_own_batch_of_the_same_shape(name):
    w = S.WORKLOADS[name]
    w0, w1 = bench.rank_workload(w, 0), bench.rank_workload(w, 1)
    assert w0 == w                                # rank 0 runs the workload itself
    assert w1.replace(seed=w.seed) == w and w1.seed != w.seed
    if isinstance(w, S.DecodeWorkload):
        small = dict(batch=2, length=64)
        x0 = S.decode_inputs(w0, **small)
        x1 = S.decode_inputs(w1, **small)
    else:
        x0 = S.prefill_inputs(w0, batch=1, tokens=16)
        x1 = S.prefill_inputs(w1, batch=1, tokens=16)
    for k in ("a_k", "b_k", "a_v", "b_v"):
        assert x0[k].shape == x1[k].shape
        assert not torch.equal(x0[k], x1[k])      # independent data, no duplicated work
