"""tpa_decode_attention_noalloc against tpa_decode_attention.

Some callers cannot allocate device memory at all: a plugin inside an
inference engine that owns the whole memory budget, or a serving loop that
must never reach cudaMalloc because it can stall every stream on the device.
They call tpa_decode_attention_noalloc, which keeps the split-KV partials in a
scratch array built into libtpa instead of a caller workspace.  These tests
drive it through the C ABI and compare it with the workspace entry point,
for two calls in a row on different caches (the array keeps the previous
call's contents, which must not leak into the next result).

The file name sorts last, so a run that stops at the first failure has
already run every other test.
"""
import pytest
import torch

from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T
from tests.gpu_cases import DEV, build_decode_cache
from tests.parity_util import TOL, assert_rows_close

pytestmark = pytest.mark.gpu


def _cases():
    a = build_decode_cache(S.WORKLOADS["decode_b8_l8k"], batch=3, length=3000, min_length=100)
    b = build_decode_cache(S.WORKLOADS["decode_b32_var32k"], batch=2, length=5000, min_length=1)
    c = build_decode_cache(S.WORKLOADS["decode_tiny_f32"])
    return [a, b, c]


@pytest.mark.parametrize("splits", [0, 1, 7])
def test_noalloc_matches_workspace_entry_point_two_calls(splits):
    cases = _cases()
    outs = []
    for cache, x, q, q_pos in cases:                       # consecutive calls, different caches
        out = torch.empty(cache.batch, cache.heads, cache.head_dim, dtype=torch.float32, device=DEV)
        T.tpa_decode_attention_noalloc(cache, q, q_pos, out, max_len=cache.capacity, num_splits=splits)
        outs.append(out)
    for (cache, x, q, q_pos), got in zip(cases, outs):
        ref = T.tpa_decode_attention(cache, q, q_pos, max_len=cache.capacity, num_splits=splits)
        assert_rows_close(got.double().cpu().numpy(), ref.double().cpu().numpy(), TOL[cache.dtype], "noalloc")
    assert T.tpa_read_device_error() == 0


def test_noalloc_too_many_splits_is_rejected_and_default_fits():
    w = S.WORKLOADS["decode_b8_l8k"]
    cache, x, q, q_pos = build_decode_cache(w, batch=64, length=600, min_length=300)
    out = torch.full((64, 32, 128), 3.0, dtype=torch.float32, device=DEV)
    # 2000 splits: CUDA-core partials 64 x 38 x 32 x (128 + 2) floats = 40 MB, tensor-core
    # partials 2 x 2000 x 32 x (128 + 2) floats = 33 MB; either way above the 16 MiB of scratch
    with pytest.raises(T.TpaError) as e:
        T.tpa_decode_attention_noalloc(cache, q, q_pos, out, max_len=600, num_splits=2000)
    assert e.value.status == 5 and "scratch" in str(e.value)
    assert bool((out == 3.0).all())                        # nothing was launched
    # 512 sequences on the CUDA-core kernel: the default split count would need more than
    # 16 MiB of partials, so the entry point lowers it
    big, xb, qb, qpb = build_decode_cache(w, batch=512, length=600, min_length=1)
    simt = T.TPA_KERNEL_SIMT
    assert T.tpa_decode_workspace_size(big, 600, 0, simt) > (16 << 20)
    out_big = torch.empty(512, 32, 128, dtype=torch.float32, device=DEV)
    calls = ((cache, q, q_pos, out, T.TPA_KERNEL_AUTO), (big, qb, qpb, out_big, simt))
    for c, qq, qp, o, k in calls:                          # two calls in a row
        T.tpa_decode_attention_noalloc(c, qq, qp, o, max_len=600, kernel=k)
    for c, qq, qp, o, k in calls:
        ref = T.tpa_decode_attention(c, qq, qp, max_len=600, kernel=k)
        assert_rows_close(o.double().cpu().numpy(), ref.double().cpu().numpy(), TOL[c.dtype], "default")
    assert T.tpa_read_device_error() == 0
