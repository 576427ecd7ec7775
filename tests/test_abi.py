"""libtpa.so loads, exports every declared symbol, and its host-side checks
reject bad arguments before touching the GPU (no GPU needed)."""
import ctypes

import pytest
import torch

from factorized_kv_cache_b200 import tpa as T


def test_exports_every_declared_symbol():
    lib = T.load_library()
    names = T.declared_functions()
    assert "tpa_decode_attention" in names and "tpa_cache_append" in names
    for n in names:
        assert hasattr(lib, n), n


def test_factor_elements_per_token_printed_value():
    # section 关键设计: 2*h*d_h = 8192 -> (R_K+R_V)(h+d_h) = 320 at R=1, h=32, d_h=128
    assert T.tpa_factor_elements_per_token(32, 128, 1, 1) == 320
    assert T.tpa_factor_elements_per_token(32, 128, 2, 2) == 640
    assert T.tpa_factor_elements_per_token(0, 128, 1, 1) == 0


def test_status_strings():
    for s, name in T.STATUS_NAMES.items():
        assert T.tpa_status_string(s).startswith(name)


def _fake_cache(**kw):
    args = dict(batch=2, capacity=64, heads=32, head_dim=128, r_k=1, r_v=1, dtype=T.TPA_BF16, reserved=0,
                rope_base=10000.0, a_k=0x10000, b_k=0x20000, a_v=0x30000, b_v=0x40000, seq_lens=0x50000)
    args.update(kw)
    return T.tpa_cache(**args)


def _decode(lib, c, **kw):
    a = dict(q=0x60000, q_pos=0x70000, scale=0.1, out=0x80000, max_len=64, splits=0, kernel=0, ws=None, ws_bytes=0)
    a.update(kw)
    return lib.tpa_decode_attention(ctypes.byref(c) if c is not None else None, a["q"], a["q_pos"],
                                    a["scale"], a["out"], a["max_len"], a["splits"], a["kernel"], a["ws"],
                                    a["ws_bytes"], None)


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 100, 3), ("heads", 33, 3), ("heads", 0, 3), ("r_k", 5, 3), ("r_v", 0, 3),
    ("dtype", 7, 3), ("batch", 0, 2), ("capacity", 0, 2), ("reserved", 1, 2), ("rope_base", 1.0, 2),
    ("a_k", 0, 1), ("seq_lens", 0, 1), ("b_v", 0x40008, 6),
])
def test_decode_rejects_bad_cache(field, value, status):
    lib = T.load_library()
    c = _fake_cache(**{field: value})
    assert _decode(lib, c) == status
    assert lib.tpa_last_error_message().decode() != ""


def test_bf16_heads_must_fill_16_bytes():
    lib = T.load_library()
    assert _decode(lib, _fake_cache(heads=4)) == 3          # 8 bytes of bf16
    assert _decode(lib, _fake_cache(heads=4, dtype=T.TPA_F32, head_dim=16), max_len=0) != 3


def test_decode_rejects_bad_arguments():
    lib = T.load_library()
    c = _fake_cache()
    assert _decode(lib, None) == 1
    assert _decode(lib, c, q=None) == 1
    assert _decode(lib, c, out=None) == 1
    assert _decode(lib, c, max_len=-1) == 2
    assert _decode(lib, c, max_len=65) == 4
    assert _decode(lib, c, splits=-2) == 2
    assert _decode(lib, c, kernel=9) == 2
    assert _decode(lib, c, scale=float("nan")) == 2
    assert _decode(lib, c, q=0x60004) == 6
    assert _decode(lib, _fake_cache(dtype=T.TPA_F32), kernel=T.TPA_KERNEL_TENSOR) == 3


def test_factored_decode_rejects_bad_arguments():
    lib = T.load_library()
    P = 0x90000

    def call(c=None, rq=6, a_q=P, b_q=P, kernel=0):
        c = _fake_cache() if c is None else c
        return lib.tpa_decode_attention_factored(ctypes.byref(c), rq, a_q, b_q, 0x70000, 0.1, 0x80000, 64, 0, kernel,
                                                 None, 0, None)

    assert call(rq=0) == 2
    assert call(rq=9) == 3
    assert call(a_q=None) == 1
    assert call(b_q=None) == 1
    assert call(b_q=P + 8) == 6
    assert call(a_q=P + 1) == 6
    assert call(c=_fake_cache(dtype=T.TPA_F32, heads=32, head_dim=128)) == 3   # tcgen05 kernel only
    assert call(c=_fake_cache(heads=16)) == 3
    assert call(c=_fake_cache(r_k=2, r_v=1)) == 3
    assert call(kernel=T.TPA_KERNEL_SIMT) == 3
    assert call(kernel=T.TPA_KERNEL_TENSOR_SYNC) == 3
    assert lib.tpa_last_error_message().decode() != ""


def test_decode_step_rejects_bad_arguments():
    lib = T.load_library()
    P = 0x90000

    def call(c=None, pos=0x70000, ak=P, bk=P, av=P, bv=P, rq=0, a_q=None, q=0x60000, advance=1, kernel=0):
        c = _fake_cache() if c is None else c
        return lib.tpa_decode_step(ctypes.byref(c), pos, ak, bk, av, bv, rq, a_q, q, 0.1, 0x80000, 64, advance, 0,
                                   kernel, None, 0, None)

    assert call(rq=-1) == 2
    assert call(advance=2) == 2
    assert call(pos=None) == 1
    assert call(q=None) == 1
    for k in ("ak", "bk", "av", "bv"):
        assert call(**{k: None}) == 1
        assert call(**{k: P + 4}) == 6
    assert call(rq=3, a_q=None) == 1
    assert call(rq=9, a_q=P) == 3
    assert call(c=_fake_cache(dtype=T.TPA_F32)) == 3   # tcgen05 kernel only
    assert call(c=_fake_cache(r_k=2, r_v=1)) == 3
    assert call(c=_fake_cache(batch=1025)) == 3
    assert call(kernel=T.TPA_KERNEL_SIMT) == 3
    assert call(kernel=T.TPA_KERNEL_TENSOR_SYNC) == 3
    assert lib.tpa_last_error_message().decode() != ""


def test_lse_decode_and_merge_reject_bad_arguments():
    lib = T.load_library()
    P = 0x90000
    c = _fake_cache()
    lse = lambda cc=c, lse_p=P, kernel=0: lib.tpa_decode_attention_lse(ctypes.byref(cc), 0x60000, 0x70000, 0.1,
                                                                        0x80000, lse_p, 64, 0, kernel, None, 0, None)
    assert lse(lse_p=None) == 1
    assert lse(lse_p=P + 2) == 6
    assert lse(kernel=T.TPA_KERNEL_SIMT) == 3
    assert lse(cc=_fake_cache(dtype=T.TPA_F32)) == 3
    merge = lambda n=2, rows=8, d=128, po=P, pl=P, o=0xA0000, lo=None: lib.tpa_merge_lse(n, rows, d, po, pl, o, lo, None)
    assert merge(n=0) == 2
    assert merge(rows=-1) == 2
    assert merge(d=130) == 3
    assert merge(d=2) == 3
    assert merge(rows=0, po=None, pl=None, o=None) == 0      # nothing to merge
    assert merge(po=None) == 1
    assert merge(o=None) == 1
    assert merge(po=P + 8) == 6
    assert merge(lo=P + 2) == 6


def test_stage_rejects_bad_arguments():
    lib = T.load_library()
    assert lib.tpa_stage_async(None, None, 0, None) == 0          # nothing to copy
    assert lib.tpa_stage_async(None, 0x90000, 16, None) == 1
    assert lib.tpa_stage_async(0x90000, None, 16, None) == 1
    with pytest.raises(ValueError):
        T.tpa_stage_async(torch.empty(4), torch.empty(4))          # src is not pinned


def test_step_plan_rejects_bad_arguments():
    lib = T.load_library()
    P = 0x90000

    def init(plan, c=None, rq=0, ak=P, stage=(None, None, 0), kernel=0):
        c = _fake_cache() if c is None else c
        return lib.tpa_step_plan_init(plan, ctypes.byref(c), 0x70000, ak, P, P, P, rq, None, 0x60000, 0.1, 0x80000,
                                      64, 1, 0, kernel, None, 0, *stage)

    plan = T.tpa_step_plan()
    assert lib.tpa_step_plan_run(None, None) == 1
    assert lib.tpa_step_plan_run(ctypes.byref(plan), None) == 2        # never initialised
    assert init(None) == 1
    assert init(ctypes.byref(plan), rq=-1) == 2
    assert init(ctypes.byref(plan), ak=None) == 1
    assert init(ctypes.byref(plan), ak=P + 4) == 6
    assert init(ctypes.byref(plan), stage=(None, 0xA0000, 64)) == 1
    assert init(ctypes.byref(plan), stage=(0xA0000, None, 64)) == 1
    assert init(ctypes.byref(plan), c=_fake_cache(dtype=T.TPA_F32)) == 3
    assert init(ctypes.byref(plan), kernel=T.TPA_KERNEL_SIMT) == 3
    assert lib.tpa_step_plan_run(ctypes.byref(plan), None) == 2        # a failed init leaves it unusable
    assert ctypes.sizeof(T.tpa_step_plan) == 2048


def test_append_rejects_bad_arguments():
    lib = T.load_library()
    c = _fake_cache()
    P = 0x90000
    assert lib.tpa_cache_append(ctypes.byref(c), -1, P, P, P, P, P, None) == 2
    assert lib.tpa_cache_append(ctypes.byref(c), 0, None, None, None, None, None, None) == 0   # no-op
    assert lib.tpa_cache_append(ctypes.byref(c), 3, None, P, P, P, P, None) == 1
    assert lib.tpa_cache_append(ctypes.byref(c), 3, P, P + 2, P, P, P, None) == 6


def test_prefill_rejects_bad_arguments():
    lib = T.load_library()
    c = _fake_cache()
    P = 0x90000

    def call(n=16, rq=6, ws=0xA0000, ws_bytes=1 << 40, kernel=0, cc=c):
        return lib.tpa_prefill_attention(ctypes.byref(cc), n, rq, P, P, P, 0.1, P, kernel, ws, ws_bytes, None)

    assert call(n=-1) == 2
    assert call(n=65) == 2
    assert call(rq=0) == 3
    assert call(rq=9) == 3
    assert call(n=0) == 0
    assert call(ws=None) == 5
    assert call(ws_bytes=16) == 5
    assert call(ws=0xA0010) == 6
    assert call(kernel=T.TPA_KERNEL_TENSOR, cc=_fake_cache(dtype=T.TPA_F32)) == 3


def test_workspace_sizes_follow_the_split_plan():
    lib = T.load_library()
    c = _fake_cache(capacity=1 << 19)
    # one split needs no workspace; more splits need (m, l) and o per split and head
    assert lib.tpa_decode_workspace_size(ctypes.byref(c), 100, 1, T.TPA_KERNEL_SIMT) == 0
    n = lib.tpa_decode_workspace_size(ctypes.byref(c), 1 << 19, 8, T.TPA_KERNEL_SIMT)
    parts = 2 * 8 * 32
    assert n >= parts * (2 + 128) * 4
    assert lib.tpa_decode_default_splits(ctypes.byref(c), 1 << 19, T.TPA_KERNEL_SIMT) >= 1


def test_selftest_rejects_bad_limits():
    lib = T.load_library()
    assert lib.tpa_selftest_wait_timeout(0, None) == 2
    assert lib.tpa_selftest_wait_timeout(10_000_000_001, None) == 2
    assert lib.tpa_last_error_message().decode() != ""


def test_prefill_workspace_sizes():
    """The tensor-core prefill's workspace: fp16 copies of the B_K and B_V planes and the
    chunk's rotated B_Q rank rows, the chunk padded to whole 32-query blocks (no dense query); the
    CUDA-core prefill's: dense fp32 queries."""
    lib = T.load_library()
    r256 = lambda n: (n + 255) // 256 * 256
    for B, cap, r, n, rq in ((4, 4096, 2, 4096, 6), (3, 1000, 1, 77, 1), (1, 64, 2, 5, 8)):
        c = _fake_cache(batch=B, capacity=cap, r_k=r, r_v=r)
        want = 2 * r256(B * cap * r * 128 * 2) + r256(B * ((n + 31) // 32 * 32) * rq * 128 * 2)
        assert lib.tpa_prefill_workspace_size(ctypes.byref(c), n, rq, T.TPA_KERNEL_AUTO) == want
        assert lib.tpa_prefill_workspace_size(ctypes.byref(c), n, rq, T.TPA_KERNEL_SIMT) == r256(B * n * 32 * 128 * 4)
    # the prefill workload: 42 MB instead of the 268 MB of dense fp32 queries
    c = _fake_cache(batch=4, capacity=4096, r_k=2, r_v=2)
    assert lib.tpa_prefill_workspace_size(ctypes.byref(c), 4096, 6, T.TPA_KERNEL_AUTO) == 2 * 8388608 + 25165824
