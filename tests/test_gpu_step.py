"""GPU parity of tpa_decode_step (append the generated token and attend with its
query, fused) against the oracle's decode_step, and against the two-call path
(tpa_cache_append, then tpa_decode_attention) for what the cache holds."""
import ctypes
import numpy as np
import pytest
import torch

import oracle.tpa_oracle as O
from factorized_kv_cache_b200 import synthetic as S
from factorized_kv_cache_b200 import tpa as T
from tests.gpu_cases import DEV, build_decode_cache, readback
from tests.parity_util import TOL, assert_rows_close, default_scale, f64

pytestmark = pytest.mark.gpu

BF16 = TOL[torch.bfloat16]


def _token(w, batch, seed, r_q=0):
    """The generated token's factors (the workload's value distributions) and its query."""
    g = S.rng(seed, 23)
    R, h, d = w.r_k, w.heads, w.head_dim
    tok = {
        "a_k": g.standard_normal((batch, R, h), dtype=np.float32),
        "b_k": g.standard_normal((batch, R, d), dtype=np.float32) / np.float32(np.sqrt(d)),
        "a_v": g.standard_normal((batch, R, h), dtype=np.float32),
        "b_v": g.standard_normal((batch, R, d), dtype=np.float32) / np.float32(np.sqrt(d)),
    }
    if r_q == 0:
        tok["q"] = g.standard_normal((batch, h, d), dtype=np.float32)
    else:
        tok["a_q"] = g.standard_normal((batch, r_q, h), dtype=np.float32)
        tok["b_q"] = g.standard_normal((batch, r_q, d), dtype=np.float32) * np.float32(np.sqrt(r_q))
    return {k: S.to_storage(v, "bf16").to(DEV) for k, v in tok.items()}


def _step(cache, tok, pos, **kw):
    qkw = {"q": tok["q"]} if "q" in tok else {"a_q": tok["a_q"], "b_q": tok["b_q"]}
    return T.tpa_decode_step(cache, pos, tok["a_k"], tok["b_k"], tok["a_v"], tok["b_v"], **qkw, **kw)


def _oracle(cpu, lengths, tok, pos, w, b, heads=None):
    L = int(lengths[b])
    sel = slice(None) if heads is None else list(heads)
    qkw = {"q": f64(tok["q"][b])[sel]} if "q" in tok else {"a_q": f64(tok["a_q"][b])[:, sel], "b_q": f64(tok["b_q"][b])}
    o, row = O.decode_step(cpu["a_k"][b, :L][:, :, sel], cpu["b_k"][b, :L], cpu["a_v"][b, :L][:, :, sel],
                           cpu["b_v"][b, :L], f64(tok["a_k"][b])[:, sel], f64(tok["b_k"][b]),
                           f64(tok["a_v"][b])[:, sel], f64(tok["b_v"][b]), float(pos[b]),
                           default_scale(w.head_dim), w.rope_base, storage="bf16", **qkw)
    return o, row


def _same_as_append(cache, before, tok, pos, lengths):
    """The slot the step filled holds exactly what tpa_cache_append writes for the token."""
    ref = T.TpaCache(*(t.clone() for t in before), rope_base=cache.rope_base)
    T.tpa_cache_append(ref, pos[:, None].contiguous(), tok["a_k"][:, None].contiguous(),
                       tok["b_k"][:, None].contiguous(), tok["a_v"][:, None].contiguous(),
                       tok["b_v"][:, None].contiguous())
    for b, L in enumerate(lengths):
        if L >= cache.capacity:
            continue
        for name in ("a_k", "b_k", "a_v", "b_v"):
            assert torch.equal(getattr(cache, name)[b, L], getattr(ref, name)[b, L]), (name, b)


@pytest.mark.parametrize("rank", [1, 2])
@pytest.mark.parametrize("r_q", [0, 6])
@pytest.mark.parametrize("splits", [0, 1, 5, 300])
def test_step_ragged(rank, r_q, splits):
    """Ragged lengths (empty, one token, tile edges, several thousand) over partitions that make
    whole-CTA sequences, shared ones and idle CTAs; the output against the oracle's step, the
    stored row against tpa_cache_append, the lengths advanced by one."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step", r_k=rank, r_v=rank, seed=70 + rank)
    lengths = [1000, 0, 1, 127, 128, 4000, 129, 333]
    cache, x, _, _ = build_decode_cache(w, batch=8, length=4001, lengths=lengths)
    before = [t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)]
    tok = _token(w, 8, 80 + rank + r_q, r_q)
    pos = torch.tensor(lengths, dtype=torch.int32, device=DEV) + 7
    out = _step(cache, tok, pos, max_len=4000, num_splits=splits)
    torch.cuda.synchronize()
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens.cpu(), torch.tensor(lengths, dtype=torch.int32) + 1)
    _same_as_append(cache, before, tok, pos, lengths)
    cpu = readback(T.TpaCache(*before, rope_base=cache.rope_base))
    got = f64(out)
    for b in range(8):
        ref, row = _oracle(cpu, lengths, tok, pos.cpu(), w, b)
        assert_rows_close(got[b], ref, BF16, f"step R={rank} r_q={r_q} splits={splits} b={b}")
        assert (np.abs(f64(cache.b_k[b, lengths[b]]) - row) <= 2.0 ** -7 * np.abs(row) + 1e-6).all()


def test_step_without_advance_overwrites_the_same_slot():
    """advance=False: the lengths stay, so a second step replaces the first step's token."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_fixed", seed=74)
    lengths = [700, 0, 2500, 64]
    cache, x, _, _ = build_decode_cache(w, batch=4, length=2600, lengths=lengths)
    before = [t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)]
    pos = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    _step(cache, _token(w, 4, 90), pos, max_len=2600, advance=False)
    tok = _token(w, 4, 91)
    out = _step(cache, tok, pos, max_len=2600, advance=False)
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens.cpu(), torch.tensor(lengths, dtype=torch.int32))
    _same_as_append(cache, before, tok, pos, lengths)
    cpu = readback(T.TpaCache(*before, rope_base=cache.rope_base))
    for b in range(4):
        ref, _ = _oracle(cpu, lengths, tok, pos.cpu(), w, b)
        assert_rows_close(f64(out[b]), ref, BF16, f"fixed-length step b={b}")


def test_generation_chain():
    """Six steps back to back on one stream, each attending every token the earlier steps
    stored (the next split kernel reads the slot and the length the previous merge wrote)."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_chain", seed=75)
    lengths = [300, 0, 127, 1000]
    cache, x, _, _ = build_decode_cache(w, batch=4, length=1010, lengths=lengths)
    cpu = readback(cache)
    toks, outs = [], []
    for k in range(6):
        tok = _token(w, 4, 100 + k, r_q=3 if k % 2 else 0)
        pos = cache.seq_lens.clone()
        toks.append((tok, pos.cpu()))
        outs.append(_step(cache, tok, pos, max_len=1010).clone())
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens.cpu(), torch.tensor(lengths, dtype=torch.int32) + 6)
    scale = default_scale(w.head_dim)
    for b in range(4):
        L = lengths[b]
        ak, bk, av, bv = cpu["a_k"][b, :L], cpu["b_k"][b, :L], cpu["a_v"][b, :L], cpu["b_v"][b, :L]
        for k, ((tok, pos), out) in enumerate(zip(toks, outs)):
            qkw = {"q": f64(tok["q"][b])} if "q" in tok else {"a_q": f64(tok["a_q"][b]), "b_q": f64(tok["b_q"][b])}
            ref, row = O.decode_step(ak, bk, av, bv, f64(tok["a_k"][b]), f64(tok["b_k"][b]), f64(tok["a_v"][b]),
                                     f64(tok["b_v"][b]), float(pos[b]), scale, w.rope_base, storage="bf16", **qkw)
            assert_rows_close(f64(out[b]), ref, BF16, f"chain step {k} b={b}")
            ak = np.concatenate([ak, f64(tok["a_k"][b])[None]])
            bk = np.concatenate([bk, row[None]])
            av = np.concatenate([av, f64(tok["a_v"][b])[None]])
            bv = np.concatenate([bv, f64(tok["b_v"][b])[None]])


def test_full_cache_is_reported_and_not_attended():
    """A sequence already at capacity: its token is neither stored nor attended (the output is
    the plain decode), its length stays, and the overflow bit is set; the others step normally."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_full", seed=76)
    cap = 512
    lengths = [cap, 100, cap, 0]
    cache, x, q, _ = build_decode_cache(w, batch=4, length=cap, lengths=lengths)
    before = [t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)]
    tok = _token(w, 4, 110)
    pos = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    out = _step(cache, tok, pos, max_len=cap)
    assert T.tpa_read_device_error() == T.TPA_DEVERR_APPEND_OVERFLOW
    assert cache.seq_lens.cpu().tolist() == [cap, 101, cap, 1]
    cpu = readback(T.TpaCache(*before, rope_base=cache.rope_base))
    scale = default_scale(w.head_dim)
    for b in range(4):
        if lengths[b] == cap:
            ref = O.decode_attention(cpu["a_k"][b], cpu["b_k"][b], cpu["a_v"][b], cpu["b_v"][b], f64(tok["q"][b]),
                                     float(pos[b]), scale, w.rope_base)
        else:
            ref, _ = _oracle(cpu, lengths, tok, pos.cpu(), w, b)
        assert_rows_close(f64(out[b]), ref, BF16, f"full-cache step b={b}")


def test_step_workload_full_size():
    """The decode workload at full size (B=8, cached length 8191 + the step's token = 8192
    attended), in the launch configuration the benchmark times (default grid, advance=False);
    the oracle on 6 heads of every sequence."""
    w = S.WORKLOADS["decode_b8_l8k"]
    lengths = [w.length - 1] * 8
    cache, x, _, _ = build_decode_cache(w, batch=8, length=w.length, lengths=lengths)
    before = [t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)]
    tok = _token(w, 8, 120)
    pos = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    out = _step(cache, tok, pos, max_len=w.length, advance=False)
    assert T.tpa_read_device_error() == 0
    _same_as_append(cache, before, tok, pos, lengths)
    heads = [0, 5, 13, 21, 30, 31]
    cpu = readback(T.TpaCache(*before, rope_base=cache.rope_base))
    for b in range(8):
        ref, _ = _oracle(cpu, lengths, tok, pos.cpu(), w, b, heads=heads)
        assert_rows_close(f64(out[b])[heads], ref, BF16, f"full-size step b={b}")


def test_step_equals_append_then_decode():
    """The fused step and the two-call path (tpa_cache_append, then tpa_decode_attention over
    L + 1 tokens) agree to the merge's rounding, and leave identical caches and lengths."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_vs_two_calls", seed=77)
    lengths = [2000, 5, 0, 3000, 128, 1]
    cache, x, _, _ = build_decode_cache(w, batch=6, length=3001, lengths=lengths)
    twin = T.TpaCache(*(t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)),
                      rope_base=cache.rope_base)
    tok = _token(w, 6, 130)
    pos = cache.seq_lens.clone()
    fused = _step(cache, tok, pos, max_len=3001)
    T.tpa_cache_append(twin, pos[:, None].contiguous(), tok["a_k"][:, None].contiguous(),
                       tok["b_k"][:, None].contiguous(), tok["a_v"][:, None].contiguous(),
                       tok["b_v"][:, None].contiguous())
    two = T.tpa_decode_attention(twin, tok["q"], pos, max_len=3001)
    assert T.tpa_read_device_error() == 0
    for name in ("a_k", "b_k", "a_v", "b_v", "seq_lens"):
        a, b = getattr(cache, name), getattr(twin, name)
        if name == "seq_lens":
            assert torch.equal(a, b)
            continue
        for s, L in enumerate(lengths):
            assert torch.equal(a[s, :L + 1], b[s, :L + 1]), (name, s)
    assert_rows_close(f64(fused), f64(two), 5e-4, "fused vs two calls")


def test_plan_matches_the_call():
    """DecodeStepPlan (arguments bound once) launches exactly what tpa_decode_step launches:
    three generation steps with new contents in the bound buffers give identical outputs,
    caches and lengths."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_plan", seed=78)
    lengths = [900, 3, 0, 1500]
    cache, x, _, _ = build_decode_cache(w, batch=4, length=1600, lengths=lengths)
    twin = T.TpaCache(*(t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)),
                      rope_base=cache.rope_base)
    buf = _token(w, 4, 140)
    pos = torch.empty(4, dtype=torch.int32, device=DEV)
    out = torch.empty(4, w.heads, w.head_dim, dtype=torch.float32, device=DEV)
    plan = T.DecodeStepPlan(cache, pos, buf["a_k"], buf["b_k"], buf["a_v"], buf["b_v"], out, q=buf["q"],
                            max_len=1600)
    for k in range(3):
        tok = _token(w, 4, 141 + k)
        for name in tok:
            buf[name].copy_(tok[name])
        pos.copy_(cache.seq_lens)
        plan()
        ref = _step(twin, tok, twin.seq_lens.clone(), max_len=1600)
        assert torch.equal(out, ref), k
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens, twin.seq_lens)
    for name in ("a_k", "b_k", "a_v", "b_v"):
        for b, L in enumerate(lengths):
            assert torch.equal(getattr(cache, name)[b, :L + 3], getattr(twin, name)[b, :L + 3])


def test_step_and_lse_at_maximum_batch():
    """1024 sequences (empty ones among them): the fused step against the oracle on a sample,
    and the lse decode of the stepped cache against the oracle's lse."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_max_batch", seed=132)
    g = np.random.default_rng(132)
    lengths = g.integers(0, 200, size=1024)
    lengths[::101] = 0
    cache, x, _, _ = build_decode_cache(w, batch=1024, length=201, lengths=lengths.tolist(), nan_tail=False)
    before = [t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)]
    tok = _token(w, 1024, 133)
    pos = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    out = _step(cache, tok, pos, max_len=201)
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens.cpu(), torch.tensor(lengths, dtype=torch.int32) + 1)
    sample = sorted(set(g.choice(1024, 32, replace=False).tolist()) | {0, 101, 1023})
    cpu = readback(T.TpaCache(*before, rope_base=cache.rope_base), sample)
    for n, b in enumerate(sample):
        L = int(lengths[b])
        ref, _ = O.decode_step(cpu["a_k"][n, :L], cpu["b_k"][n, :L], cpu["a_v"][n, :L], cpu["b_v"][n, :L],
                               f64(tok["a_k"][b]), f64(tok["b_k"][b]), f64(tok["a_v"][b]), f64(tok["b_v"][b]),
                               float(pos[b]), default_scale(w.head_dim), w.rope_base, q=f64(tok["q"][b]),
                               storage="bf16")
        assert_rows_close(f64(out[b]), ref, BF16, f"max-batch step b={b}")
    o2, lse = T.tpa_decode_attention_lse(cache, tok["q"], pos, max_len=201)
    cpu2 = readback(cache, sample)
    for n, b in enumerate(sample):
        L = int(lengths[b]) + 1
        o, l = O.decode_attention_lse(cpu2["a_k"][n, :L], cpu2["b_k"][n, :L], cpu2["a_v"][n, :L], cpu2["b_v"][n, :L],
                                      f64(tok["q"][b]), float(pos[b]), default_scale(w.head_dim), w.rope_base)
        assert np.abs(f64(lse[b]) - l).max() <= BF16, b
        assert_rows_close(f64(o2[b]), o, BF16, f"max-batch lse decode b={b}")


@pytest.mark.parametrize("rank", [1, 2])
def test_step_advance_over_many_merge_waves(rank):
    """256 sequences whose lengths sit on tile edges, advanced by the step.  The merge grid runs
    in several waves, and the head-0 CTAs of the first wave advance every length (each by a
    whole new tile) before later waves start: every merge CTA must still use the partition and
    the lengths the split kernel used, and merge exactly the partials it wrote."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_waves", r_k=rank, r_v=rank, seed=140 + rank)
    g = np.random.default_rng(140 + rank)
    lengths = g.choice([128, 256, 384], size=256)
    lengths[::37] = 0
    cache, x, _, _ = build_decode_cache(w, batch=256, length=400, lengths=lengths.tolist(), nan_tail=False)
    before = [t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)]
    tok = _token(w, 256, 141 + rank)
    pos = torch.tensor(lengths, dtype=torch.int32, device=DEV)
    out = _step(cache, tok, pos, max_len=400)
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens.cpu(), torch.tensor(lengths, dtype=torch.int32) + 1)
    _same_as_append(cache, before, tok, pos, lengths.tolist())
    sample = sorted(set(g.choice(256, 24, replace=False).tolist()) | {0, 1, 254, 255})
    cpu = readback(T.TpaCache(*before, rope_base=cache.rope_base), sample)
    for n, b in enumerate(sample):
        L = int(lengths[b])
        ref, _ = O.decode_step(cpu["a_k"][n, :L], cpu["b_k"][n, :L], cpu["a_v"][n, :L], cpu["b_v"][n, :L],
                               f64(tok["a_k"][b]), f64(tok["b_k"][b]), f64(tok["a_v"][b]), f64(tok["b_v"][b]),
                               float(pos[b]), default_scale(w.head_dim), w.rope_base, q=f64(tok["q"][b]),
                               storage="bf16")
        assert_rows_close(f64(out[b]), ref, BF16, f"many-wave step R={rank} b={b}")


def test_plan_graph_copies_in_steps_and_copies_out():
    """DecodeStepPlan.graph(): each replay copies the host inputs in, steps (advancing the
    lengths) and copies the output back; the same as the plain calls on a twin cache."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_graph", seed=79)
    lengths = [500, 0, 1200]
    cache, x, _, _ = build_decode_cache(w, batch=3, length=1300, lengths=lengths)
    twin = T.TpaCache(*(t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)),
                      rope_base=cache.rope_base)
    names = ("a_k", "b_k", "a_v", "b_v", "q")
    toks = [_token(w, 3, 150 + k) for k in range(3)]
    sizes = [toks[0][k].numel() for k in names] + [3]
    host_in = torch.empty(sum(sizes) * 4, dtype=torch.uint8).pin_memory()
    dev_in = torch.empty_like(host_in, device=DEV)
    views, off = {}, 0
    for k in names:
        nb = toks[0][k].numel() * 2
        views[k] = dev_in[off:off + nb].view(torch.bfloat16).view(toks[0][k].shape)
        off += (nb + 255) // 256 * 256
    views["pos"] = dev_in[off:off + 12].view(torch.int32)
    out = torch.empty(3, w.heads, w.head_dim, dtype=torch.float32, device=DEV)
    host_out = torch.empty(3, w.heads, w.head_dim, dtype=torch.float32).pin_memory()
    plan = T.DecodeStepPlan(cache, views["pos"], views["a_k"], views["b_k"], views["a_v"], views["b_v"], out,
                            q=views["q"], max_len=1300)
    staging = torch.empty_like(dev_in)
    g = None
    for k, tok in enumerate(toks):
        pos = twin.seq_lens.clone()
        for name in names:                      # the step's inputs, laid out in the staging buffer
            staging_view = staging[views[name].data_ptr() - dev_in.data_ptr():][:tok[name].numel() * 2]
            staging_view.copy_(tok[name].view(-1).view(torch.uint8))
        staging[views["pos"].data_ptr() - dev_in.data_ptr():][:12].copy_(pos.view(torch.uint8))
        host_in.copy_(staging.cpu())
        if g is None:
            g = plan.graph(host_in, dev_in, host_out)   # the capture's first run is step 0
        else:
            g.replay()
        torch.cuda.synchronize()
        ref = _step(twin, tok, pos, max_len=1300)
        assert torch.equal(host_out, ref.cpu()), k
    assert T.tpa_read_device_error() == 0
    assert torch.equal(cache.seq_lens, twin.seq_lens)


def test_plan_writes_its_output_to_pinned_host_memory():
    """DecodeStepPlan with a pinned host ``out``: the kernels write the output to the host
    directly; it equals the step with a device output."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_host_out", seed=83)
    lengths = [2100, 0, 64, 1]
    cache, x, _, _ = build_decode_cache(w, batch=4, length=2200, lengths=lengths)
    twin = T.TpaCache(*(t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)),
                      rope_base=cache.rope_base)
    tok = _token(w, 4, 160)
    pos = cache.seq_lens.clone()
    host_out = torch.full((4, w.heads, w.head_dim), float("nan"), dtype=torch.float32).pin_memory()
    plan = T.DecodeStepPlan(cache, pos, tok["a_k"], tok["b_k"], tok["a_v"], tok["b_v"], host_out, q=tok["q"],
                            max_len=2200)
    plan()
    torch.cuda.synchronize()
    ref = _step(twin, tok, pos.clone(), max_len=2200)
    assert T.tpa_read_device_error() == 0
    assert torch.equal(host_out, ref.cpu())
    with pytest.raises(ValueError):
        T.DecodeStepPlan(cache, pos, tok["a_k"], tok["b_k"], tok["a_v"], tok["b_v"],
                         torch.empty(4, w.heads, w.head_dim), q=tok["q"])   # pageable host memory


def test_plan_stages_its_inputs_from_pinned_host_memory():
    """DecodeStepPlan with ``stage=(host_in, dev_in)``: every call copies the packed inputs from
    pinned host memory before the step, so new host contents reach the kernels; each step equals
    the step on device inputs."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="step_staged", seed=84)
    lengths = [900, 0, 128, 5]
    cache, x, _, _ = build_decode_cache(w, batch=4, length=1000, lengths=lengths)
    twin = T.TpaCache(*(t.clone() for t in (cache.a_k, cache.b_k, cache.a_v, cache.b_v, cache.seq_lens)),
                      rope_base=cache.rope_base)
    names = ("q_pos", "a_k", "b_k", "a_v", "b_v", "q")
    first = dict(_token(w, 4, 170), q_pos=cache.seq_lens.clone())
    layout, off = [], 0
    for n in names:
        nb = first[n].numel() * first[n].element_size()
        layout.append((n, off, nb))
        off += (nb + 255) // 256 * 256
    host_in = torch.zeros(off, dtype=torch.uint8).pin_memory()
    dev_in = torch.zeros(off, dtype=torch.uint8, device=DEV)
    views = {n: dev_in[o:o + nb].view(first[n].dtype).view(first[n].shape) for n, o, nb in layout}
    out = torch.empty(4, w.heads, w.head_dim, dtype=torch.float32, device=DEV)
    plan = T.DecodeStepPlan(cache, views["q_pos"], views["a_k"], views["b_k"], views["a_v"], views["b_v"], out,
                            q=views["q"], max_len=1000, stage=(host_in, dev_in))
    for k in range(3):
        tok = dict(_token(w, 4, 170 + k), q_pos=twin.seq_lens.clone())
        for n, o, nb in layout:
            host_in[o:o + nb].copy_(tok[n].cpu().contiguous().view(-1).view(torch.uint8))
        got = plan().clone()
        ref = _step(twin, tok, tok["q_pos"], max_len=1000)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), k
        assert torch.equal(cache.seq_lens, twin.seq_lens), k
    assert T.tpa_read_device_error() == 0
    with pytest.raises(ValueError):
        T.DecodeStepPlan(cache, views["q_pos"], views["a_k"], views["b_k"], views["a_v"], views["b_v"], out,
                         q=views["q"], stage=(torch.zeros(off, dtype=torch.uint8), dev_in))   # pageable host memory
    # the C entry point checks the copy's ends itself (a C caller has no binding to check them):
    # pageable host memory as the source, or host memory as the destination, is refused
    lib = T.load_library()
    c = cache.struct()
    pageable = torch.zeros(off, dtype=torch.uint8)

    nws = int(lib.tpa_decode_workspace_size(ctypes.byref(c), 1000, 0, 0))
    ws = T.workspace(nws, DEV)

    def c_init(dst, src):
        p = T.tpa_step_plan()
        return lib.tpa_step_plan_init(ctypes.byref(p), ctypes.byref(c), T._ptr(views["q_pos"]), T._ptr(views["a_k"]),
                                      T._ptr(views["b_k"]), T._ptr(views["a_v"]), T._ptr(views["b_v"]), 0, None,
                                      T._ptr(views["q"]), 0.1, T._ptr(out), 1000, 1, 0, 0, T._ptr(ws), nws,
                                      T._ptr(dst), T._ptr(src), off)
    assert c_init(dev_in, pageable) == 3      # TPA_ERR_UNSUPPORTED
    assert c_init(host_in, host_in) == 3
    assert c_init(dev_in, host_in) == T.TPA_OK


@pytest.mark.parametrize("lengths", [[60000], [40001, 1], [0, 30000]])
@pytest.mark.parametrize("grid", [0, 300])
@pytest.mark.parametrize("r_q", [0, 6])
def test_small_batch_merge(lengths, grid, r_q):
    """A batch of one or two sequences, each split over many CTAs: the merge then runs 1024
    threads a CTA and loads every partial in one pass (with 300 CTAs, more partials than one
    pass holds).  The plain decode with its log-sum-exp and the fused step against the oracle."""
    w = S.WORKLOADS["decode_b8_l8k"].replace(name="small_batch", seed=91)
    B, cap = len(lengths), max(lengths) + 2
    cache, x, q, q_pos = build_decode_cache(w, batch=B, length=cap, lengths=lengths)
    cpu = readback(cache)
    scale = default_scale(w.head_dim)
    if r_q == 0:
        out, lse = T.tpa_decode_attention_lse(cache, q, q_pos, max_len=cap, num_splits=grid)
        for b, L in enumerate(lengths):
            ref, ref_lse = O.decode_attention_lse(cpu["a_k"][b, :L], cpu["b_k"][b, :L], cpu["a_v"][b, :L],
                                                  cpu["b_v"][b, :L], f64(q[b]), float(q_pos[b]), scale,
                                                  w.rope_base)
            if L:
                assert_rows_close(f64(out[b]), ref, BF16, f"decode b={b}")
                # an absolute error e in the log-sum-exp is a relative error e in the softmax's sum
                assert np.abs(f64(lse[b]) - ref_lse).max() <= BF16, f"lse b={b}"
            else:
                assert torch.count_nonzero(out[b]) == 0 and torch.isneginf(lse[b]).all()
    tok = _token(w, B, 92, r_q)
    pos = cache.seq_lens.clone()
    got = f64(_step(cache, tok, pos, max_len=cap, num_splits=grid))
    for b in range(B):
        ref, _ = _oracle(cpu, lengths, tok, pos.cpu(), w, b)
        assert_rows_close(got[b], ref, BF16, f"step b={b}")
    assert T.tpa_read_device_error() == 0
