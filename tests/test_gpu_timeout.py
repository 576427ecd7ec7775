"""The bounded pipeline waits end as an error status, not as a hung GPU.

The tensor-core kernels wait on shared-memory barriers that other roles of the CTA complete; each
wait gives up after a limit and records TPA_DEVERR_TIMEOUT.  tpa_selftest_wait_timeout runs that
wait on a barrier that nothing ever completes, with a short limit: the kernel must return, set the
bit, and leave the context usable for the next call."""
import time

import numpy as np
import pytest
import torch

from factorized_kv_cache_b200 import tpa as T
from tests.gpu_cases import DEV

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports():
    assert T.tpa_read_device_error() == 0
    t0 = time.perf_counter()
    T.tpa_selftest_wait_timeout(20_000_000)  # 20 ms
    code = T.tpa_read_device_error()  # synchronises
    elapsed = time.perf_counter() - t0
    assert code == T.TPA_DEVERR_TIMEOUT
    assert 0.015 < elapsed < 5.0
    assert T.tpa_read_device_error() == 0  # read clears the word


def test_context_usable_after_timeout():
    T.tpa_selftest_wait_timeout(5_000_000)
    assert T.tpa_read_device_error() == T.TPA_DEVERR_TIMEOUT
    # a plain tensor-core decode right after: correct result, clean error word
    cache = T.TpaCache.allocate(1, 256, 32, 128, 1, 1, dtype=torch.bfloat16, device=DEV)
    g = torch.Generator(device="cpu").manual_seed(3)
    n = 200
    pos = torch.arange(n, dtype=torch.int32).view(1, n).to(DEV)
    ak = torch.randn(1, n, 1, 32, generator=g).to(torch.bfloat16).to(DEV)
    bk = (torch.randn(1, n, 1, 128, generator=g) / 11.3).to(torch.bfloat16).to(DEV)
    av = torch.randn(1, n, 1, 32, generator=g).to(torch.bfloat16).to(DEV)
    bv = (torch.randn(1, n, 1, 128, generator=g) / 11.3).to(torch.bfloat16).to(DEV)
    T.tpa_cache_append(cache, pos, ak, bk, av, bv)
    q = torch.randn(1, 32, 128, generator=g).to(torch.bfloat16).to(DEV)
    qpos = torch.tensor([n], dtype=torch.int32, device=DEV)
    out_t = T.tpa_decode_attention(cache, q, qpos, kernel=T.TPA_KERNEL_TENSOR)
    out_s = T.tpa_decode_attention(cache, q, qpos, kernel=T.TPA_KERNEL_SIMT)
    assert T.tpa_read_device_error() == 0
    a, b = out_t.double().cpu().numpy(), out_s.double().cpu().numpy()
    assert np.isfinite(a).all()
    assert np.abs(a - b).max() <= 2e-3 * np.abs(b).max()
