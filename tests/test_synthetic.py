"""Seeded input generators: shapes, determinism and distributions (no GPU)."""
import numpy as np
import torch

from factorized_kv_cache_b200 import synthetic as S


def test_decode_shapes_and_determinism():
    w = S.WORKLOADS["decode_b32_var32k"]
    a = S.decode_inputs(w, batch=3, length=64, min_length=16)
    b = S.decode_inputs(w, batch=3, length=64, min_length=16)
    assert a["a_k"].shape == (3, 64, 2, 32) and a["a_k"].dtype == torch.bfloat16
    assert a["b_k"].shape == (3, 64, 2, 128)
    assert a["a_v"].shape == (3, 64, 2, 32) and a["b_v"].shape == (3, 64, 2, 128)
    assert a["q"].shape == (3, 32, 128)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    L = a["lengths"].numpy()
    assert ((L >= 16) & (L <= 64)).all()
    assert np.array_equal(a["q_pos"].numpy(), L)
    assert np.array_equal(a["positions"][1].numpy(), np.arange(64))


def test_decode_distributions():
    w = S.WORKLOADS["decode_b8_l8k"]
    x = S.decode_inputs(w, batch=2, length=4096)
    assert abs(x["a_k"].float().std().item() - 1.0) < 0.01
    assert abs(x["b_k"].float().std().item() * np.sqrt(128) - 1.0) < 0.01
    assert abs(x["q"].float().std().item() - 1.0) < 0.02
    t = S.WORKLOADS["decode_tiny_f32"]
    y = S.decode_inputs(t)
    assert y["a_k"].dtype == torch.float32 and y["a_k"].shape == (1, 64, 1, 4)
    assert int(y["q_pos"][0]) == 64


def test_prefill_shapes():
    w = S.WORKLOADS["prefill_b4_t4k"]
    x = S.prefill_inputs(w, batch=1, tokens=32)
    assert x["a_q"].shape == (1, 32, 6, 32) and x["b_q"].shape == (1, 32, 6, 128)
    assert x["a_k"].shape == (1, 32, 2, 32) and x["b_v"].shape == (1, 32, 2, 128)
    # x ~ N(0,1) width 2048 through W ~ N(0, 1/2048): unit-variance factors
    assert abs(x["b_q"].float().std().item() - 1.0) < 0.1


def test_cache_bytes_of_workloads():
    # (R_K+R_V)(h+d_h) elements per token, bf16
    w = S.WORKLOADS["decode_long_512k"]
    per_tok = (w.r_k + w.r_v) * (w.heads + w.head_dim) * 2
    assert per_tok * w.length == 335_544_320
