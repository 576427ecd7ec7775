#!/usr/bin/env python
"""Benchmark of TPA attention over a factorized KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--kernel auto|simt|tensor]

One step of a decode workload is one generation step of the whole batch: the
newest token's factors are written into the cache (RoPE on B_K at its
position) and its query attends every cached token (query RoPE, factor
scores, online softmax, rank-R value updates, split-KV log-sum-exp merge).
The cache keeps a fixed length: the newest token is rewritten in place each
step, so every step attends exactly sum_b L_b tokens.

One step of the prefill workload writes the prompt's factors and runs the
causal prefill over them.

The default workload is decode_b32_var32k (B=32, R=2, lengths uniform in
[16384, 32768]), the largest decode that fits one GPU.  On one GPU the same run
also times the long-context decode (decode_long_512k, the fused step) and the
causal prefill (prefill_b4_t4k) and adds them to the line as ``long_context``
and ``prefill``, each with its own roofline and clock record (``--extras``).
The CPU oracle baseline runs on rank 0 at N=1 only.

Rank 0 prints one JSON line.  Under torchrun every rank runs its own batch on
its own GPU (weak scaling, no collective on the data path); the time is the
maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cached tokens attended/sec (TPA decode) + achieved HBM GB/s vs peak, 1×B200"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# --------------------------------------------------------------------------- helpers
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0}, "fallback"


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


TRAFFIC_SOURCE = ("not measured in this run: dram__bytes_read.sum + dram__bytes_write.sum of one launch of the "
                  "dominant kernel from a committed ncu capture (profiles/ncu_traffic.json), reported only while "
                  "the hash of the kernel's sources matches the captured one (null otherwise)")


def ncu_traffic(workload: str, kernel_sources):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_sha") != source_sha(kernel_sources):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), sm_max=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hw_th=parts[6], sw_th=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hw_th", "hw_thermal_slowdown"),
                              ("sw_th", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        loaded = [r["sm"] for r in rows if r["power"] > 200.0] or [r["sm"] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r["sm_max"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "power_w_max": max(r["power"] for r in rows)}


# --------------------------------------------------------------------------- CPU oracle runs
def _oracle_task(args):
    """One decode over a slice of a sequence with the float64 oracle, RoPE on B_K
    included (runs in a spawned worker)."""
    import oracle.tpa_oracle as O
    a_k, b_k, a_v, b_v, positions, q, q_pos, scale, base = args
    f = lambda a: np.asarray(a, dtype=np.float64)
    O.decode_attention_from_unrotated(f(a_k), f(b_k), f(a_v), f(b_v), positions, f(q), q_pos, scale, base)
    return a_k.shape[0]


def _decode_tasks(host, w, n_tasks, slice_tokens):
    """Oracle tasks cycling over the workload's sequences, `slice_tokens` tokens each."""
    B = host["a_k"].shape[0]
    tasks = []
    scale = 1.0 / math.sqrt(w.head_dim)
    for t in range(n_tasks):
        b = t % B
        L = int(host["lengths"][b])
        n = min(L, slice_tokens)
        s0 = (t // B * n) % max(1, L - n + 1)
        tasks.append((host["a_k"][b, s0:s0 + n], host["b_k"][b, s0:s0 + n], host["a_v"][b, s0:s0 + n],
                      host["b_v"][b, s0:s0 + n], np.arange(s0, s0 + n), host["q"][b], float(host["q_pos"][b]),
                      scale, w.rope_base))
    return tasks


def cpu_oracle_rate(host, w, target_s: float, workers: int):
    """Cached tokens attended per second by the float64 oracle on `workers` host cores."""
    slice_tokens = 4096
    t0 = time.perf_counter()
    n1 = _oracle_task(_decode_tasks(host, w, 1, slice_tokens)[0])
    per_token = (time.perf_counter() - t0) / n1
    per_task = per_token * min(slice_tokens, int(host["lengths"].max()))
    n_tasks = max(workers, int(target_s * workers / max(per_task, 1e-6)))
    n_tasks = (n_tasks + workers - 1) // workers * workers
    tasks = _decode_tasks(host, w, n_tasks, slice_tokens)
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers) as pool:
        pool.map(_oracle_task, tasks[:workers])          # import + warm
        t0 = time.perf_counter()
        done = sum(pool.map(_oracle_task, tasks, chunksize=1))
        dt = time.perf_counter() - t0
    return done / dt, dict(tokens=done, seconds=dt, tasks=len(tasks), slice_tokens=slice_tokens)


# --------------------------------------------------------------------------- decode bench
def rank_workload(w, rank):
    """The workload rank `rank` runs: the same shapes, its own seed (rank 0 keeps the workload's)."""
    return w.replace(seed=w.seed + 1000 * rank) if rank else w


def max_over_ranks(x: float, world: int, dev) -> float:
    """Maximum of a per-rank number (a time) over all ranks; x itself on one rank."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def decode_host_inputs(w, rank):
    from factorized_kv_cache_b200 import synthetic as S
    return S.decode_inputs(rank_workload(w, rank))


def run_ours_decode(args, w, rank, world, dev, with_e2e=True):
    import torch
    import torch.distributed as dist
    from factorized_kv_cache_b200 import synthetic as S
    from factorized_kv_cache_b200 import tpa as T

    kernel = {"auto": T.TPA_KERNEL_AUTO, "simt": T.TPA_KERNEL_SIMT, "tensor": T.TPA_KERNEL_TENSOR,
              "tensor_sync": T.TPA_KERNEL_TENSOR_SYNC}[args.kernel]
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    esize = 4 if w.dtype == "f32" else 2
    x = decode_host_inputs(w, rank)
    B, cap = x["a_k"].shape[:2]
    lengths = x["lengths"].numpy().astype(np.int64)
    per_tok = (w.r_k + w.r_v) * (w.heads + w.head_dim) * esize
    cache_bytes = B * cap * per_tok
    copies = 1 if cache_bytes >= 2 * L2_BYTES else int(math.ceil(2 * L2_BYTES / cache_bytes)) + 1

    # The step generates one token per sequence: its factors and query come from the workload's
    # newest token (slot L_b - 1, position L_b - 1).  Fused (tpa_decode_step): the cache holds
    # L_b - 1 tokens and the step stores the token and attends all L_b (advance=False, so every
    # step rewrites the same slot).  Two calls: the cache holds L_b tokens, tpa_cache_write_slots
    # rewrites slot L_b - 1, then tpa_decode_attention attends all L_b.
    fused = args.step == "fused" and kernel in (T.TPA_KERNEL_AUTO, T.TPA_KERNEL_TENSOR) and w.dtype == "bf16"
    if fused and lengths.min() < 1:
        raise ValueError("the fused step needs every sequence to hold its newest token")
    # copy 0 from the seeded inputs through the product append path, the rest cloned
    c0 = T.TpaCache.allocate(B, cap, w.heads, w.head_dim, w.r_k, w.r_v, dtype=dt, rope_base=w.rope_base, device=dev)
    T.tpa_cache_append(c0, x["positions"].to(dev), x["a_k"].to(dev), x["b_k"].to(dev), x["a_v"].to(dev),
                       x["b_v"].to(dev))
    c0.seq_lens.copy_(torch.from_numpy((lengths - 1 if fused else lengths).astype(np.int32)).to(dev))
    caches = [c0] + [T.TpaCache(c0.a_k.clone(), c0.b_k.clone(), c0.a_v.clone(), c0.b_v.clone(), c0.seq_lens.clone(),
                                w.rope_base) for _ in range(copies - 1)]
    newest = torch.from_numpy((lengths - 1).clip(min=0).astype(np.int32))[:, None]
    sel = (torch.arange(B), torch.from_numpy((lengths - 1).clip(min=0)))
    inputs = {}   # the step's device inputs, by name; the e2e leg copies them from one pinned buffer
    if fused:
        for k in ("a_k", "b_k", "a_v", "b_v"):
            inputs[k] = x[k][sel].contiguous().to(dev)                 # [B, R, h | d_h]
    else:
        for k in ("a_k", "b_k", "a_v", "b_v"):
            inputs[k] = x[k][sel][:, None].contiguous().to(dev)        # [B, 1, R, h | d_h]
        inputs["slots"] = newest.to(dev)
        inputs["pos2"] = newest.to(dev)
    inputs["q_pos"] = newest[:, 0].contiguous().to(dev)
    rq = args.query_rank
    if rq > 0:
        # the query in TPA form: A_Q ~ N(0,1), B_Q ~ N(0, R_Q), so the summed query has unit variance
        g = S.rng(rank_workload(w, rank).seed, 23)
        inputs["a_q"] = S.to_storage(g.standard_normal((B, rq, w.heads), dtype=np.float32), w.dtype).to(dev)
        inputs["b_q"] = S.to_storage(g.standard_normal((B, rq, w.head_dim), dtype=np.float32) *
                                     np.float32(math.sqrt(rq)), w.dtype).to(dev)
        query_bytes = B * rq * (w.heads + w.head_dim) * esize
    else:
        inputs["q"] = x["q"].to(dev)
        query_bytes = B * w.heads * w.head_dim * esize
    out = torch.empty(B, w.heads, w.head_dim, dtype=torch.float32, device=dev)
    splits = T.tpa_decode_default_splits(c0, cap, kernel)
    ws = T.workspace(T.tpa_decode_workspace_size(c0, cap, 0, kernel), dev)
    tokens_per_step = int(lengths.sum())

    def step(c, v=inputs):
        qkw = {"a_q": v["a_q"], "b_q": v["b_q"]} if rq > 0 else {"q": v["q"]}
        if fused:
            T.tpa_decode_step(caches[c], v["q_pos"], v["a_k"], v["b_k"], v["a_v"], v["b_v"], **qkw, out=out,
                              max_len=cap, advance=False, kernel=kernel, workspace_buf=ws)
            return
        T.tpa_cache_write_slots(caches[c], v["slots"], v["pos2"], v["a_k"], v["b_k"], v["a_v"], v["b_v"])
        if rq > 0:
            T.tpa_decode_attention_factored(caches[c], v["a_q"], v["b_q"], v["q_pos"], out=out, max_len=cap,
                                            kernel=kernel, workspace_buf=ws)
        else:
            T.tpa_decode_attention(caches[c], v["q"], v["q_pos"], out=out, max_len=cap, kernel=kernel,
                                   workspace_buf=ws)

    def decode_call(c):
        """The call the roofline times: the fused step, or the decode of the two-call step."""
        if fused:
            step(c)
        elif rq > 0:
            T.tpa_decode_attention_factored(caches[c], inputs["a_q"], inputs["b_q"], inputs["q_pos"], out=out,
                                            max_len=cap, kernel=kernel, workspace_buf=ws)
        else:
            T.tpa_decode_attention(caches[c], inputs["q"], inputs["q_pos"], out=out, max_len=cap, kernel=kernel,
                                   workspace_buf=ws)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for c in range(copies):     # eager run first (loads the module, checks arguments)
            step(c)
    torch.cuda.synchronize(dev)
    # one graph per cache copy for the whole step; for the kernel roofline, one graph of n_calls
    # decode calls cycling over the copies, so that the per-graph launch cost is not charged to the kernel
    gs = []
    for c in range(copies):
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1, stream=stream):
            step(c)
        gs.append(g1)
    # the timed steps replay graphs of `copies` consecutive steps (one per cache copy), so that
    # the steps follow each other as a decode loop captured in CUDA graphs would
    gm = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gm, stream=stream):
        for c in range(copies):
            step(c)
    n_calls = copies * max(1, math.ceil(4 / copies))
    gd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gd, stream=stream):
        for k in range(n_calls):
            decode_call(k % copies)
    torch.cuda.synchronize(dev)
    if T.tpa_read_device_error() != 0:
        raise RuntimeError("device error word set after set-up")

    K, W = args.steps, args.warmup
    reps = max(1, K // n_calls)
    with torch.cuda.stream(stream):
        for k in range(W):
            gs[k % copies].replay()
        gm.replay()
        gd.replay()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        full, rest = divmod(K, copies)
        for _ in range(full):
            gm.replay()
        for k in range(rest):
            gs[k].replay()
        t_end.record(stream)
        # the decode call alone, n_calls back to back per graph, for the roofline
        for r in range(reps):
            ev[r][0].record(stream)
            gd.replay()
            ev[r][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    elapsed_ms = t_start.elapsed_time(t_end)
    decode_ms = [a.elapsed_time(b) / n_calls for a, b in ev]
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    if T.tpa_read_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    e2e = run_decode_e2e(args, K, W, B, w, inputs, fused, rq, caches, copies, cap, kernel, ws, out, step, stream,
                         world, dev, tokens_per_step) if with_e2e else None
    return _decode_result(args, w, world, K, W, B, lengths, tokens_per_step, per_tok, fused, query_bytes, rq,
                          kernel, splits, copies, cache_bytes, elapsed_ms, decode_ms, n_calls, clk, e2e), x, lengths


def run_decode_e2e(args, K, W, B, w, inputs, fused, rq, caches, copies, cap, kernel, ws, out, step, stream, world,
                   dev, tokens_per_step):
    """The decode step end to end through the public API with host buffers."""
    import torch
    import torch.distributed as dist
    from factorized_kv_cache_b200 import tpa as T
    # e2e through the public API with host buffers: every step copies its inputs from one pinned
    # host buffer (one H2D copy) and reads the output back (one D2H copy), then synchronises
    layout, off = [], 0
    for k2, v in inputs.items():
        nb = v.numel() * v.element_size()
        layout.append((k2, off, nb, v))
        off += (nb + 255) // 256 * 256
    host_in = torch.empty(off, dtype=torch.uint8).pin_memory()
    dev_in = torch.empty(off, dtype=torch.uint8, device=dev)
    views = {}
    for k2, o, nb, v in layout:
        host_in[o:o + nb].copy_(v.cpu().contiguous().view(-1).view(torch.uint8))
        views[k2] = dev_in[o:o + nb].view(v.dtype).view(v.shape)
    host_out = torch.empty(B, w.heads, w.head_dim, dtype=torch.float32).pin_memory()
    h2d = sum(nb for _, _, nb, _ in layout)
    d2h = host_out.numel() * 4
    e2e_steps = max(1, min(K, 2000))

    if fused:
        # a generation loop binds its buffers once (T.DecodeStepPlan) and calls it every step: the
        # plan copies the packed inputs from the pinned host buffer, then runs the step, whose
        # output goes to pinned host memory that the kernels write directly (the device-to-host
        # transfer of the result, with no copy to launch)
        v = views
        qkw = {"a_q": v["a_q"], "b_q": v["b_q"]} if rq > 0 else {"q": v["q"]}
        plans = [T.DecodeStepPlan(caches[c], v["q_pos"], v["a_k"], v["b_k"], v["a_v"], v["b_v"], host_out, **qkw,
                                  max_len=cap, advance=False, kernel=kernel, workspace_buf=ws,
                                  stage=(host_in, dev_in)) for c in range(copies)]

    def e2e_step(c):
        if fused:
            plans[c](stream)
        else:
            with torch.cuda.stream(stream):
                dev_in.copy_(host_in, non_blocking=True)
                step(c, views)
                host_out.copy_(out, non_blocking=True)
        stream.synchronize()

    for k in range(min(W, 10)):
        e2e_step(k % copies)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for k in range(e2e_steps):
        e2e_step(k % copies)
    e2e_s = time.perf_counter() - t0
    e2e_s = max_over_ranks(e2e_s, world, dev)
    return {"value": world * tokens_per_step * e2e_steps / e2e_s, "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}


def _decode_result(args, w, world, K, W, B, lengths, tokens_per_step, per_tok, fused, query_bytes, rq, kernel,
                   splits, copies, cache_bytes, elapsed_ms, decode_ms, n_calls, clk, e2e):
    from factorized_kv_cache_b200 import tpa as T
    launches_per_step = 2 if fused else 1 + 1 + (1 if splits > 1 else 0)
    # factor bytes of every attended token (cached, or the step's own read from its inputs), the
    # step's token stored (fused), the query and the fp32 output
    bytes_per_decode = tokens_per_step * per_tok + (B * per_tok if fused else 0) + query_bytes + \
        B * w.heads * w.head_dim * 4
    mean_decode_s = statistics.mean(decode_ms) / 1e3
    peaks, kind = measured_peaks()
    achieved = bytes_per_decode / mean_decode_s / 1e9
    # the dominant kernel's source and the headers it includes (the traffic figure is reused
    # only while all of them are unchanged)
    hdrs = ["factorized_kv_cache_b200/csrc/device_common.cuh", "factorized_kv_cache_b200/csrc/ptx_sm100.cuh"]
    if kernel == T.TPA_KERNEL_SIMT or w.dtype == "f32":
        kernel_src = ["factorized_kv_cache_b200/csrc/attention_simt.cu"] + hdrs
    elif kernel == T.TPA_KERNEL_TENSOR_SYNC:
        kernel_src = ["factorized_kv_cache_b200/csrc/decode_tensor.cu",
                      "factorized_kv_cache_b200/csrc/decode_common.cuh"] + hdrs
    else:
        kernel_src = ["factorized_kv_cache_b200/csrc/decode_umma.cu",
                      "factorized_kv_cache_b200/csrc/decode_common.cuh"] + hdrs
    kernel_src = [p for p in kernel_src if os.path.exists(os.path.join(ROOT, p))]
    res = {
        "metric": METRIC,
        "value": world * tokens_per_step * K / (elapsed_ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": elapsed_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded Philox normals; A~N(0,1), B~N(0,1/d_h), q~N(0,1))",
        "config": {
            "workload": w.name, "batch": B, "seq_len": int(lengths.max()), "seq_len_min": int(lengths.min()),
            "heads": w.heads, "head_dim": w.head_dim, "r_k": w.r_k, "r_v": w.r_v,
            "tokens_attended_per_step": tokens_per_step, "kernel": args.kernel, "splits": splits,
            "query": "dense" if rq == 0 else f"TPA factors, R_Q={rq}",
            "step": ("tpa_decode_step: split kernel over the L-1 cached tokens + merge that stores the newest "
                     "token (RoPE on B_K) and joins it" if fused else
                     "write newest token (RoPE on B_K) + decode attention (+ LSE merge)") +
                    f"; timed as CUDA graphs of {copies} consecutive steps (one per cache copy)",
            "l2": (f"inputs larger than L2: {copies} cache copies rotated ({copies * cache_bytes / 2**20:.0f} MiB "
                   f"> 126 MiB L2)" if copies > 1 else f"inputs larger than L2 ({cache_bytes / 2**20:.0f} MiB)"),
            "parallelism": f"dp{world} (independent batches, no collective)",
        },
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": ncu_traffic(w.name, kernel_src) if kernel_src else None,
            "traffic_source": TRAFFIC_SOURCE, "peak_kind": kind,
            "kernel": ("fused step call" if fused else "decode attention call") +
                      " (split kernel + merge), timed right after the K timed steps on the same stream: graphs of "
                      "back-to-back decode calls over the same cache copies, CUDA events around each graph",
            "calls_per_graph": n_calls,
            "algorithmic_bytes_per_launch": bytes_per_decode, "mean_launch_us": mean_decode_s * 1e6,
        },
        "gpu_launches": K * launches_per_step,
        "clocks": clk,
    }
    if e2e is not None:
        res["e2e"] = e2e
    return res


def run_ours_decode_sharded(args, w, rank, world, dev):
    """Strong scaling of one batch: rank r holds, for every sequence, the token range
    token_range(L_b, world, r) at the tokens' global positions, decodes it with
    tpa_decode_attention_lse, and the ranks all-gather (out, lse) and merge them with
    tpa_merge_lse, so every rank ends with the output of the whole range."""
    import torch
    import torch.distributed as dist
    from factorized_kv_cache_b200 import sharded
    from factorized_kv_cache_b200 import tpa as T

    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    esize = 4 if w.dtype == "f32" else 2
    x = decode_host_inputs(w, 0)                 # the same batch on every rank
    B, cap = x["a_k"].shape[:2]
    lengths = x["lengths"].numpy().astype(np.int64)
    ranges = [sharded.token_range(int(L), world, rank) for L in lengths]
    shard_lens = np.array([e - s for s, e in ranges], dtype=np.int64)
    scap = max(1, int(shard_lens.max()))
    # tokens [s_b, s_b + scap) of each sequence (indices past the sequence clamp to its last
    # slot: they sit past the shard's length and are never attended)
    idx = np.stack([np.minimum(np.arange(scap) + s, cap - 1) for s, _ in ranges])
    rows = torch.arange(B)[:, None]
    tix = torch.from_numpy(idx)
    per_tok = (w.r_k + w.r_v) * (w.heads + w.head_dim) * esize
    shard_bytes = B * scap * per_tok
    copies = 1 if shard_bytes >= 2 * L2_BYTES else int(math.ceil(2 * L2_BYTES / shard_bytes)) + 1
    c0 = T.TpaCache.allocate(B, scap, w.heads, w.head_dim, w.r_k, w.r_v, dtype=dt, rope_base=w.rope_base, device=dev)
    T.tpa_cache_append(c0, x["positions"][rows, tix].contiguous().to(dev),
                       *(x[k][rows, tix].contiguous().to(dev) for k in ("a_k", "b_k", "a_v", "b_v")))
    c0.seq_lens.copy_(torch.from_numpy(shard_lens.astype(np.int32)).to(dev))
    caches = [c0] + [T.TpaCache(c0.a_k.clone(), c0.b_k.clone(), c0.a_v.clone(), c0.b_v.clone(), c0.seq_lens.clone(),
                                w.rope_base) for _ in range(copies - 1)]
    q = x["q"].to(dev)
    q_pos = x["q_pos"].to(dev)
    out = torch.empty(B, w.heads, w.head_dim, dtype=torch.float32, device=dev)
    lse = torch.empty(B, w.heads, dtype=torch.float32, device=dev)
    res = torch.empty_like(out)
    res_lse = torch.empty_like(lse)
    ws = T.workspace(T.tpa_decode_workspace_size(c0, scap, 0, T.TPA_KERNEL_AUTO), dev)

    def local(c, qv=q):
        T.tpa_decode_attention_lse(caches[c], qv, q_pos, out=out, lse=lse, max_len=scap, workspace_buf=ws)

    def exchange_merge():
        if world > 1:
            parts_out, parts_lse = sharded.all_gather_partials(out, lse)
        else:
            parts_out, parts_lse = out[None], lse[None]
        T.tpa_merge_lse(parts_out, parts_lse, out=res, lse_out=res_lse)

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for c in range(copies):
            local(c)
            exchange_merge()
    torch.cuda.synchronize(dev)
    gl = []
    for c in range(copies):
        g1 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1, stream=stream):
            local(c)
        gl.append(g1)
    n_calls = copies * max(1, math.ceil(4 / copies))
    gd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gd, stream=stream):
        for k in range(n_calls):
            local(k % copies)
    torch.cuda.synchronize(dev)
    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for k in range(W):
            gl[k % copies].replay()
            exchange_merge()
        gd.replay()
    torch.cuda.synchronize(dev)
    if T.tpa_read_device_error() != 0:
        raise RuntimeError("device error word set after set-up")
    reps = max(1, K // n_calls)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for k in range(K):
            gl[(W + k) % copies].replay()
            exchange_merge()
        t_end.record(stream)
        for r in range(reps):
            ev[r][0].record(stream)
            gd.replay()
            ev[r][1].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    local_s = statistics.mean(a.elapsed_time(b) / n_calls for a, b in ev) / 1e3
    if T.tpa_read_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    # e2e: the query from pinned host memory, the merged output back, every step
    host_q = x["q"].pin_memory()
    host_out = torch.empty(B, w.heads, w.head_dim, dtype=torch.float32).pin_memory()
    dev_q = torch.empty_like(q)
    e2e_steps = max(1, min(K, 500))

    def e2e_step(c):
        with torch.cuda.stream(stream):
            dev_q.copy_(host_q, non_blocking=True)
            local(c, dev_q)
            exchange_merge()
            host_out.copy_(res, non_blocking=True)
        stream.synchronize()

    for k in range(min(W, 10)):
        e2e_step(k % copies)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for k in range(e2e_steps):
        e2e_step(k % copies)
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev)

    tokens = int(lengths.sum())
    local_bytes = int(shard_lens.sum()) * per_tok + B * w.heads * w.head_dim * (esize + 4) + B * w.heads * 4
    peaks, kind = measured_peaks()
    achieved = local_bytes / local_s / 1e9
    res_json = {
        "metric": METRIC,
        "value": tokens * K / (elapsed_ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": elapsed_ms / K,
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded Philox normals; A~N(0,1), B~N(0,1/d_h), q~N(0,1))",
        "config": {
            "workload": w.name, "batch": B, "seq_len": int(lengths.max()), "heads": w.heads, "head_dim": w.head_dim,
            "r_k": w.r_k, "r_v": w.r_v, "tokens_attended_per_step": tokens,
            "shard": f"token ranges over {world} rank(s); this rank holds {int(shard_lens.sum())} tokens",
            "step": "tpa_decode_attention_lse on the local range (one CUDA graph) + all-gather of (out, lse) + "
                    "tpa_merge_lse",
            "l2": (f"inputs larger than L2: {copies} cache copies rotated" if copies > 1 else
                   f"inputs larger than L2 ({shard_bytes / 2**20:.0f} MiB)"),
            "parallelism": f"token-sharded x{world} (one all-gather per step)",
        },
        "roofline": {
            "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_kind": kind,
            "kernel": "local decode call with lse (split kernel + merge), graphs of back-to-back calls",
            "calls_per_graph": n_calls, "algorithmic_bytes_per_launch": local_bytes,
            "mean_launch_us": local_s * 1e6,
        },
        "e2e": {"value": tokens * e2e_steps / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": q.numel() * esize,
                "d2h_bytes_per_step": host_out.numel() * 4, "steps": e2e_steps},
        "gpu_launches": K * 3,
        "clocks": clk,
    }
    return res_json, x, lengths


def _host_arrays(x, lengths):
    host = {k: x[k].float().numpy() for k in ("a_k", "b_k", "a_v", "b_v", "q")}
    host["lengths"] = lengths
    host["q_pos"] = (lengths - 1).clip(min=0)
    return host


def add_cpu_baseline(res, x, w, lengths, target_s):
    host = _host_arrays(x, lengths)
    host["lengths"] = lengths
    host["q_pos"] = (lengths - 1).clip(min=0)
    workers = max(1, min(os.cpu_count() or 1, 16))
    rate, info = cpu_oracle_rate(host, w, target_s, workers)
    res["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": workers, "kind": "oracle",
                           "sample": f"{info['tasks']} decode slices of <= {info['slice_tokens']} cached tokens "
                                     f"(all {w.heads} heads) of this workload, float64 oracle, "
                                     f"{info['seconds']:.1f} s on {workers} spawned processes"}


def run_reference_prefill(args, w):
    """Reference arm for the prefill workload: the float64 oracle on sampled query rows."""
    workers = max(1, min(os.cpu_count() or 1, 16))
    K, W = args.steps, args.warmup
    budget = 150.0 / max(1, K + W)
    rows_per_task = 8
    n_fn = lambda per_task: max(1, min(workers, int(budget * workers / max(per_task, 1e-6))))
    done, dt, n = _prefill_rate(w, workers, n_fn, rows_per_task, steps=K, warm_steps=W)
    value = done / dt
    sample = (f"each step: {n} oracle prefills of {rows_per_task} random query rows of sequence 0 (all heads, "
              f"full causal prefix) of {w.name}, float64 oracle on {workers} spawned processes")
    return {
        "impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": K,
        "warmup": W, "ms_per_step": dt / max(1, K) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.tokens, "heads": w.heads,
                   "head_dim": w.head_dim, "r_q": w.r_q, "r_k": w.r_k, "r_v": w.r_v},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args, w):
    """The float64 CPU oracle as the reference arm (host cores only)."""
    from factorized_kv_cache_b200 import synthetic as S
    if isinstance(w, S.PrefillWorkload):
        return run_reference_prefill(args, w)
    x = decode_host_inputs(w, 0)
    lengths = x["lengths"].numpy().astype(np.int64)
    host = _host_arrays(x, lengths)
    workers = max(1, min(os.cpu_count() or 1, 16))
    K, W = args.steps, args.warmup
    budget = 150.0 / max(1, K + W)
    slice_tokens = 4096
    t0 = time.perf_counter()
    _oracle_task(_decode_tasks(host, w, 1, slice_tokens)[0])
    per_task = time.perf_counter() - t0
    tasks_per_step = max(1, min(workers, int(budget * workers / max(per_task, 1e-6))))
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers) as pool:
        for k in range(W):
            pool.map(_oracle_task, _decode_tasks(host, w, tasks_per_step, slice_tokens))
        t0 = time.perf_counter()
        done = 0
        for k in range(K):
            done += sum(pool.map(_oracle_task, _decode_tasks(host, w, tasks_per_step, slice_tokens)))
        dt = time.perf_counter() - t0
    value = done / dt
    sample = (f"each step: {tasks_per_step} decode slices of <= {slice_tokens} cached tokens (all heads) of "
              f"{w.name}, float64 oracle on {workers} spawned processes")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1, "steps": K,
        "warmup": W, "ms_per_step": dt / max(1, K) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": int(x["a_k"].shape[0]), "seq_len": int(lengths.max()),
                   "heads": w.heads, "head_dim": w.head_dim, "r_k": w.r_k, "r_v": w.r_v},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": workers, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------------- prefill bench
PREFILL_METRIC = "causal prefill query tokens/sec (TPA, R_Q-factorized queries) + tensor TFLOP/s vs peak, 1×B200"


_PF = {}


def _prefill_worker_init(w):
    """Spawned worker: regenerate sequence 0 of the prefill workload from its seed.

    The hidden states and projections come from fixed Philox streams, so
    batch=1 reproduces sequence 0 of the full batch exactly."""
    from factorized_kv_cache_b200 import synthetic as S
    x = S.prefill_inputs(w, batch=1)
    _PF.update({k: x[k][0].double().numpy() for k in ("a_q", "b_q", "a_k", "b_k", "a_v", "b_v")})
    _PF["w"] = w


def _prefill_oracle_task(rows):
    """Oracle prefill of some query rows of sequence 0 (all heads, full causal prefix, RoPE)."""
    import oracle.tpa_oracle as O
    w = _PF["w"]
    L = _PF["a_k"].shape[0]
    pos = np.arange(L)
    O.prefill_attention(_PF["a_k"], O.append_rope(_PF["b_k"], pos, w.rope_base, "bf16"), _PF["a_v"], _PF["b_v"],
                        _PF["a_q"], _PF["b_q"], pos, 1.0 / math.sqrt(w.head_dim), w.rope_base, rows=rows)
    return len(rows)


def _prefill_rate(w, workers, n_tasks_fn, rows_per_task, steps=1, warm_steps=0):
    """Run oracle prefill tasks on a spawned pool; returns (rows done, seconds, tasks per step)."""
    g = np.random.default_rng(0)
    draw = lambda n: [np.sort(g.integers(0, w.tokens, rows_per_task)) for _ in range(n)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers, initializer=_prefill_worker_init, initargs=(w,)) as pool:
        t0 = time.perf_counter()
        pool.map(_prefill_oracle_task, draw(workers), chunksize=1)      # calibration, one task per worker
        per_task = (time.perf_counter() - t0)
        n = n_tasks_fn(per_task)
        for _ in range(warm_steps):
            pool.map(_prefill_oracle_task, draw(n), chunksize=1)
        done = 0
        t0 = time.perf_counter()
        for _ in range(steps):
            done += sum(pool.map(_prefill_oracle_task, draw(n), chunksize=1))
        dt = time.perf_counter() - t0
    return done, dt, n


def run_ours_prefill(args, w, rank, world, dev):
    import torch
    import torch.distributed as dist
    from factorized_kv_cache_b200 import synthetic as S
    from factorized_kv_cache_b200 import tpa as T

    kernel = {"auto": T.TPA_KERNEL_AUTO, "simt": T.TPA_KERNEL_SIMT, "tensor": T.TPA_KERNEL_TENSOR,
              "tensor_sync": T.TPA_KERNEL_TENSOR_SYNC}[args.kernel]
    ww = rank_workload(w, rank)
    x = S.prefill_inputs(ww)
    B, Tn = w.batch, w.tokens
    cache = T.TpaCache.allocate(B, Tn, w.heads, w.head_dim, w.r_k, w.r_v, dtype=torch.bfloat16,
                                rope_base=w.rope_base, device=dev)
    cache.seq_lens.fill_(Tn)
    d = {k: x[k].to(dev) for k in ("a_q", "b_q", "a_k", "b_k", "a_v", "b_v", "positions")}
    slots = d["positions"]
    out = torch.empty(B, Tn, w.heads, w.head_dim, dtype=torch.float32, device=dev)
    ws = T.workspace(T.tpa_prefill_workspace_size(cache, Tn, w.r_q, kernel), dev)

    def write():
        T.tpa_cache_write_slots(cache, slots, d["positions"], d["a_k"], d["b_k"], d["a_v"], d["b_v"])

    def prefill():
        T.tpa_prefill_attention(cache, d["a_q"], d["b_q"], d["positions"], out=out, kernel=kernel, workspace_buf=ws)

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        write()
        prefill()
    torch.cuda.synchronize(dev)
    gw, gp = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw, stream=stream):
        write()
    with torch.cuda.graph(gp, stream=stream):
        prefill()
    torch.cuda.synchronize(dev)
    if T.tpa_read_device_error() != 0:
        raise RuntimeError("device error word set after set-up")
    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for _ in range(W):
            gw.replay()
            gp.replay()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for k in range(K):
            gw.replay()
            ev[k][0].record(stream)
            gp.replay()
            ev[k][1].record(stream)
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    elapsed_ms = t_start.elapsed_time(t_end)
    pre_ms = [a.elapsed_time(b) for a, b in ev]
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    if T.tpa_read_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    # e2e: host factors and queries in, output back, through the public API
    host = {k: x[k].pin_memory() for k in ("a_q", "b_q", "a_k", "b_k", "a_v", "b_v", "positions")}
    host_out = torch.empty_like(out, device="cpu").pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host_out.numel() * 4
    e2e_steps = max(1, min(K, 20))

    def e2e_step():
        with torch.cuda.stream(stream):
            for k2, v in host.items():
                d[k2].copy_(v, non_blocking=True)
            T.tpa_cache_write_slots(cache, d["positions"], d["positions"], d["a_k"], d["b_k"], d["a_v"], d["b_v"],
                                    stream=stream)
            T.tpa_prefill_attention(cache, d["a_q"], d["b_q"], d["positions"], out=out, kernel=kernel,
                                    workspace_buf=ws, stream=stream)
            host_out.copy_(out, non_blocking=True)
        stream.synchronize()

    e2e_step()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        e2e_step()
    e2e_s = max_over_ranks(time.perf_counter() - t0, world, dev)

    pairs = B * Tn * (Tn + 1) // 2
    # algorithmic flops per causal (query, key) pair, counted with the scores formed on the rank
    # factors (B_Q . B_K^T, R_Q R_K dot products of d_h shared by all heads) and the value
    # contraction per head (R_V rank-one updates of d_h); the dense per-head count (a d_h dot
    # product per head and rank of the key, plus the same value term) is reported beside it
    flops = pairs * (2 * w.r_q * w.r_k * w.head_dim + 2 * w.heads * w.r_v * w.head_dim)
    flops_dense = pairs * w.heads * 2 * w.head_dim * (w.r_k + w.r_v)
    mean_s = statistics.mean(pre_ms) / 1e3
    peaks, kind = measured_peaks()
    achieved = flops / mean_s / 1e12
    tensor = kernel != T.TPA_KERNEL_SIMT
    src = ["factorized_kv_cache_b200/csrc/prefill_tensor.cu"] if tensor else ["factorized_kv_cache_b200/csrc/attention_simt.cu"]
    res = {
        "metric": PREFILL_METRIC, "value": world * B * Tn * K / (elapsed_ms / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (x~N(0,1) width 2048, factors x W with W~N(0,1/2048))",
        "config": {"workload": w.name, "batch": B, "seq_len": Tn, "heads": w.heads, "head_dim": w.head_dim,
                   "r_q": w.r_q, "r_k": w.r_k, "r_v": w.r_v, "kernel": args.kernel,
                   "step": "write prompt factors (RoPE on B_K) + causal prefill, CUDA graphs",
                   "l2": f"inputs larger than L2 (the {out.numel() * 4 / 1e6:.0f} MB fp32 output and "
                         f"{(ws.numel() if ws is not None else 0) / 1e6:.0f} MB of workspace per step)",
                   "parallelism": f"dp{world} (independent batches, no collective)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "traffic": ncu_traffic(w.name, src), "peak_kind": kind + " (bf16 burst)",
                     "kernel": "prefill attention call",
                     "algorithmic_flops_per_launch": flops,
                     "flops_count": "rank-factor scores (2 R_Q R_K d_h per pair) + per-head values (2 h R_V d_h "
                                    "per pair), causal pairs only",
                     "dense_equivalent_flops_per_launch": flops_dense,
                     "dense_equivalent_tflops": flops_dense / mean_s / 1e12,
                     "mean_launch_us": mean_s * 1e6},
        "e2e": {"value": world * B * Tn * e2e_steps / e2e_s, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps},
        "gpu_launches": K * 3,
        "clocks": clk,
    }
    return res, x


def add_prefill_cpu_baseline(res, x, w, target_s):
    workers = max(1, min(os.cpu_count() or 1, 16))
    rows_per_task = 16
    n_fn = lambda per_task: max(workers, int(target_s * workers / max(per_task, 1e-6)) // workers * workers)
    done, dt, n = _prefill_rate(w, workers, n_fn, rows_per_task)
    res["cpu_baseline"] = {"value": done / dt, "unit": "tokens/s", "cores": workers, "kind": "oracle",
                           "sample": f"{n} oracle prefills of {rows_per_task} random query rows of sequence 0 "
                                     f"(all heads, full causal prefix, RoPE included) of {w.name}; {dt:.1f} s on "
                                     f"{workers} spawned processes"}


DEFAULT_WORKLOAD = "decode_b32_var32k"   # the largest single-GPU decode workload


def add_extras(args, res, dev):
    """Two more workloads timed in the same run on one GPU, each with its own roofline and clock
    record: the long-context decode (one sequence of 524288 tokens, the fused step) and the
    causal prefill (its own metric: query tokens/s and tensor TFLOP/s)."""
    import gc
    import torch
    from factorized_kv_cache_b200 import synthetic as S
    gc.collect()
    torch.cuda.empty_cache()
    keep = ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config", "roofline", "e2e", "gpu_launches",
            "clocks")
    wl = S.WORKLOADS["decode_long_512k"]
    r_long, x, _ = run_ours_decode(args, wl, 0, 1, dev)
    del x
    res["long_context"] = dict({"metric": METRIC}, **{k: r_long[k] for k in keep if k in r_long})
    gc.collect()
    torch.cuda.empty_cache()
    wp = S.WORKLOADS["prefill_b4_t4k"]
    pargs = argparse.Namespace(**vars(args))
    pargs.steps = max(3, min(args.steps, 10))
    r_pre, x = run_ours_prefill(pargs, wp, 0, 1, dev)
    del x
    if args.cpu_seconds > 0:
        add_prefill_cpu_baseline(r_pre, None, wp, min(args.cpu_seconds, 8.0))
    res["prefill"] = dict({"metric": PREFILL_METRIC}, **{k: r_pre[k] for k in keep + ("cpu_baseline",)
                                                         if k in r_pre})
    gc.collect()
    torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=["decode_tiny_f32", "decode_b8_l8k", "decode_b32_var32k", "prefill_b4_t4k",
                             "decode_long_512k"])
    ap.add_argument("--kernel", choices=["auto", "simt", "tensor", "tensor_sync"], default="auto")
    ap.add_argument("--query-rank", type=int, default=0,
                    help="decode workloads: 0 = dense query; R_Q > 0 = query given as TPA factors A_Q, B_Q")
    ap.add_argument("--step", choices=["fused", "two_call"], default="fused",
                    help="decode step: tpa_decode_step (tcgen05 path), or tpa_cache_write_slots + decode")
    ap.add_argument("--shard-tokens", action="store_true",
                    help="decode workloads: split every sequence's token range across the ranks (strong scaling)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU oracle sample length (0: skip)")
    ap.add_argument("--extras", choices=["auto", "on", "off"], default="auto",
                    help="one GPU: also time the long-context decode and the causal prefill in the same run "
                         "(auto: with the default workload)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling smaller cases)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the workload's length / prompt tokens")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from factorized_kv_cache_b200 import synthetic as S
    w = S.WORKLOADS[args.workload]
    if args.batch > 0:
        w = w.replace(batch=args.batch)
    if args.seq_len > 0:
        if isinstance(w, S.PrefillWorkload):
            w = w.replace(tokens=args.seq_len)
        else:
            w = w.replace(length=args.seq_len, min_length=min(w.min_length, args.seq_len))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    try:
        if isinstance(w, S.PrefillWorkload):
            res, x = run_ours_prefill(args, w, rank, world, dev)
            if rank == 0 and world == 1 and args.cpu_seconds > 0:
                add_prefill_cpu_baseline(res, x, w, args.cpu_seconds)
        elif args.shard_tokens:
            res, x, lengths = run_ours_decode_sharded(args, w, rank, world, dev)
            if rank == 0 and world == 1 and args.cpu_seconds > 0:
                add_cpu_baseline(res, x, w, lengths, args.cpu_seconds)
        else:
            res, x, lengths = run_ours_decode(args, w, rank, world, dev)
            if rank == 0 and world == 1 and args.cpu_seconds > 0:
                add_cpu_baseline(res, x, w, lengths, args.cpu_seconds)
            del x
            extras = args.extras == "on" or (args.extras == "auto" and args.workload == DEFAULT_WORKLOAD and
                                             args.batch == 0 and args.seq_len == 0)
            if extras and world == 1:
                add_extras(args, res, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
