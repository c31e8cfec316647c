#!/usr/bin/env python3
"""Benchmark of the InfLLM-V2 sparse-attention prefill path on B200.

One step = the whole prefill hot path over one 131072-token sequence
(h_q=32, h_kv=2, d=128, |I|=96): pool K (stage-1 and coarse windows),
compressed scores with the LSE approximation and the fused group sum,
max-pool + top-k block selection, block-sparse attention.  Inputs are
seeded synthetic tensors (inputs/gen.py), resident in HBM before the timed
region; the working set (Q 1 GiB, S_shared 4.3 GB) is larger than L2, so no
extra flush is needed between steps.

Output: one JSON line (rank 0).  `value` is tokens/s over all ranks;
`e2e` repeats the measurement through the public API with the inputs copied
from pinned host memory and the output copied back inside the timed region
(pipelined over two buffer sets; the serial figure rides along);
`roofline` describes the dominant kernel; `step_roofline` the whole step
against the sum of its steps' bounds; `decode` the 16 x 131072 decode step
(µs/step, fraction of HBM); `varlen` the packed 131072-token dense/sparse
switch workload (tokens/s, dense and sparse time, the dense kernel's
roofline); `cpu_baseline` times the fp64 oracle on a bounded sample of rows
on all host cores the process may use, and on one core.

`--impl reference` times the oracle alone (the reference arm for this build:
there is no installable reference implementation; the pages carry no code).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "128K prefill attn tokens/s (select+sparse) & decode µs/step; % of roofline"
WORKLOAD = "prefill_128k"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- work counts
def visible_counts(n: int, n_init: int = 1, n_local: int = 32, top_k: int = 63):
    """Per query position t of an n-token sequence: visible C1 windows, C2
    windows, sparse keys (|I| blocks of 64; the query's own block is the
    only partial one) and, of those, the keys of the shared blocks (init and
    local, the query's own block among them) and of the top-k blocks."""
    t = np.arange(n, dtype=np.int64)
    n1 = np.where(t >= 31, (t - 31) // 16 + 1, 0)
    n2 = np.where(t >= 127, (t - 127) // 64 + 1, 0)
    b_t = t // 64
    nsel = np.minimum(n_init + n_local + top_k, b_t + 1)
    keys = (nsel - 1) * 64 + (t % 64) + 1
    i_hi = np.minimum(n_init, b_t + 1)
    l_start = np.maximum(i_hi, b_t - n_local + 1)
    nshared = i_hi + np.maximum(0, b_t - l_start + 1)
    shared_keys = (nshared - 1) * 64 + (t % 64) + 1
    topk_keys = keys - shared_keys
    return n1, n2, keys, shared_keys, topk_keys


def algorithmic_work(n: int, h_q: int, h_kv: int, d: int):
    n1, n2, keys, shared_keys, topk_keys = visible_counts(n)
    G = h_q // h_kv
    ld = ((n - 32) // 16 + 1 + 3) // 4 * 4
    w = {}
    # compress: read K, write both pooled key sets
    w["compress_bytes"] = n * h_kv * d * 2 + h_kv * (int(n1[-1]) + int(n2[-1])) * d * 2
    # scores: 2d flop per (head, token, visible window) for both passes; one exp each
    w["score_flops"] = 2 * d * h_q * int(n1.sum() + n2.sum())
    w["score_exps"] = h_q * int(n1.sum() + n2.sum())
    w["score_bytes"] = n * h_q * d * 2 + 4 * h_kv * int(n1.sum())
    # top-k: read the visible part of S_shared, write the block lists
    w["topk_bytes"] = 4 * h_kv * int(n1.sum()) + 4 * h_kv * n * 96
    # the pooled form: one (max, last window) pair per group of four visible windows
    groups = (n1 + 3) // 4
    w["score_bytes_pooled"] = n * h_q * d * 2 + 8 * h_kv * int(groups.sum())
    w["topk_bytes_pooled"] = 8 * h_kv * int(groups.sum()) + 4 * h_kv * n * 96
    # sparse attention: QK^T and PV over the visible selected keys
    w["sparse_flops"] = 4 * d * h_q * int(keys.sum())
    w["sparse_exps"] = h_q * int(keys.sum())
    # K and V rows the attention must bring to the SMs (algorithmic): the
    # top-k blocks of every (token, group), and the shared init and local
    # blocks once per 64-token query block and group (they are the same for
    # every token of the block)
    def shared_blocks_at(b0):
        i_hi = np.minimum(1, b0 + 1)
        return i_hi + np.maximum(0, b0 - np.maximum(i_hi, b0 - 31) + 1)
    qb = np.arange(0, (n + 63) // 64)
    w["sparse_topk_gather_bytes"] = h_kv * 2 * d * 2 * int(topk_keys.sum())
    w["sparse_shared_gather_bytes"] = h_kv * 2 * d * 2 * 64 * int(shared_blocks_at(qb).sum())
    w["sparse_gather_bytes"] = w["sparse_topk_gather_bytes"] + w["sparse_shared_gather_bytes"]
    # what the kernels move for the shared blocks: the LOCAL form reads them
    # once per CTA of two 128-row query tiles, 256/G tokens (re-reads counted
    # apart from the algorithmic bytes)
    t0 = np.arange(0, n, max(1, 256 // G))
    w["sparse_shared_gather_bytes_kernel"] = h_kv * 2 * d * 2 * 64 * int(shared_blocks_at(t0 // 64).sum())
    w["ld"] = ld
    return w


# ---------------------------------------------------------------- L2 gather probe
def measure_l2_gather(T, torch, K, V, stream, target_bytes: float = 8e9, reps: int = 3) -> dict:
    """Best L2 -> SM gather bandwidth (GB/s) over the probe's producer counts:
    random pairs of 64-key blocks of K and V of one kv group (the first
    2048 blocks, 67 MB: L2-resident), 192 KB in flight per SM."""
    nsm = torch.cuda.get_device_properties(K.device).multi_processor_count
    nblk = min(2048, K.shape[0] // 64)
    out = {}
    for prod in (1, 2, 3, 6):
        tiles = max(1, int(target_bytes / (nsm * prod * 32768)))
        T.infllm2_probe_l2_gather(K, V, nblk, tiles, prod, stream)
        best = None
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            T.infllm2_probe_l2_gather(K, V, nblk, tiles, prod, stream)
            b.record(stream)
            b.synchronize()
            ms = a.elapsed_time(b)
            best = ms if best is None else min(best, ms)
        out[f"producers_{prod}"] = nsm * prod * tiles * 32768 / (best / 1e3) / 1e9
    return {"GB/s": max(out.values()), "variants": out, "footprint_MB": 2 * nblk * 64 * K.shape[1] * 256 / 1e6}


# ---------------------------------------------------------------- ranks
def max_over_ranks(x: float, device) -> float:
    """Largest value of x over all ranks (the job's time is its slowest
    rank's).  Single process: x itself."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self):
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        sel = []
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            sel = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "50", *sel],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a moment to start: wait for its first sample so the
        # timed region that follows is covered from its start
        t0 = time.time()
        while time.time() - t0 < 10.0:
            with open(self.path) as f:
                if f.read().count("\n") >= 1:
                    break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle baseline
def oracle_sequence(w, data, lse: str = "approx"):
    """The fp64 oracle's sequence object (inputs converted, keys pooled) and
    the seconds that took."""
    from oracle import infllm2_oracle as O
    p = O.Params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k, lse_mode=lse)
    t0 = time.perf_counter()
    seq = O.Sequence1(O.to_f64(data["Q"]), O.to_f64(data["K"]), O.to_f64(data["V"]), p)
    return seq, time.perf_counter() - t0


def oracle_rows(seq, rows: int, seed: int) -> float:
    """Scores, selection and sparse attention of the oracle for `rows`
    uniformly sampled (token, group) rows; returns the seconds taken."""
    rng = np.random.default_rng(seed)
    t1 = time.perf_counter()
    for _ in range(rows):
        t = int(rng.integers(0, seq.n))
        g = int(rng.integers(0, seq.h_kv))
        seq.sparse_out(t, g, seq.select(t, g))
    return time.perf_counter() - t1


def oracle_sample(w, data, seconds: float, lse: str = "approx", threads: int = 1, seq=None):
    """Time the fp64 oracle with NumPy/BLAS limited to `threads` threads:
    pooling of the whole sequence, then rows sampled until ~`seconds`.
    Returns tokens/s extrapolated to all rows of the sequence, the rows done,
    the seconds spent, and the sequence object (reusable)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=threads):
        if seq is None:
            seq, t_pool = oracle_sequence(w, data, lse)
        else:
            seq, t_pool = seq
        rows, t_rows, seed = 0, 0.0, 123
        while t_rows < seconds:
            t_rows += oracle_rows(seq, 8, seed)
            rows += 8
            seed += 1
    per_row = t_rows / max(rows, 1)
    total_s = t_pool + per_row * seq.n * seq.h_kv
    return seq.n / total_s, rows, t_pool + t_rows, (seq, t_pool)


def cpu_baseline_entry(w, data, seconds: float, lse: str) -> dict:
    """The oracle on every host core the process may use (BLAS threads =
    len(sched_getaffinity)) and on one core, half of `seconds` each."""
    ncores = len(os.sched_getaffinity(0))
    tok_n, rows_n, secs_n, seq = oracle_sample(w, data, seconds / 2, lse, threads=ncores)
    tok_1, rows_1, secs_1, _ = oracle_sample(w, data, seconds / 2, lse, threads=1, seq=seq)
    return {"value": tok_n, "unit": "tokens/s", "cores": ncores, "kind": "oracle",
            "sample": f"fp64 oracle, NumPy/BLAS threads = {ncores}: pooling of the whole {w.seqlen}-token sequence "
                      f"({seq[1]:.1f} s) + {rows_n} uniformly sampled (token, group) rows ({secs_n:.1f} s in all), "
                      f"extrapolated to all {w.seqlen * w.h_kv} rows",
            "extrapolated": True,
            "one_core": {"value": tok_1, "unit": "tokens/s", "cores": 1,
                         "sample": f"same, 1 thread: {rows_1} rows ({secs_1 - seq[1]:.1f} s) + the same pooling"}}


# ---------------------------------------------------------------- decode
def decode_bytes_per_step(prefix: int, steps: int, batch: int, h_kv: int, d: int) -> float:
    """Algorithmic HBM bytes of one decode step (averaged over the timed
    steps): the visible pooled keys of both kinds and the K/V rows of the
    visible selected keys, per sequence and kv group."""
    tot = 0.0
    for i in range(steps):
        t = prefix + i
        n1 = (t - 31) // 16 + 1
        n2 = (t - 127) // 64 + 1
        b_t = t // 64
        keys = (min(96, b_t + 1) - 1) * 64 + (t % 64) + 1
        tot += batch * h_kv * (n1 * d * 2 + n2 * d * 2 + keys * 2 * d * 2)
    return tot / steps


def bench_layer(T, gen, torch, dev, reps: int = 3, decode_steps: int = 8):
    """One attention layer with random bf16 weights: the q/k/v and output
    projections (cuBLAS GEMMs through torch) around the attention, with this
    library's sparse attention and with a dense attention (torch SDPA on a
    fused backend: a library kernel, the baseline).  Time to first token of a
    131072-token prefill and time per output token of a 16 x 131072 decode, at
    the bench workload's heads (32 query, 2 kv, d = 128, hidden 4096).  No norm
    or positional encoding: the layers differ only in the attention."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    backends = [SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION]
    w = gen.WORKLOADS["prefill_128k"]
    n, hq, hkv, d = w.seqlen, w.h_q, w.h_kv, w.d
    hidden = hq * d
    gen_t = torch.Generator(device=dev).manual_seed(1234)

    def rand(*shape, scale=1.0):
        return (torch.randn(*shape, generator=gen_t, device=dev) * scale).to(torch.bfloat16)

    Wq, Wk = rand(hidden, hq * d, scale=hidden ** -0.5), rand(hidden, hkv * d, scale=hidden ** -0.5)
    Wv, Wo = rand(hidden, hkv * d, scale=hidden ** -0.5), rand(hq * d, hidden, scale=(hq * d) ** -0.5)
    p = T.default_params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k)

    def timed(fn, n_iter=1, before=None):
        fn()                                   # warm-up
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            if before is not None:
                before()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(n_iter):
                fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / n_iter)
        return statistics.median(ts)

    res = {"workload": {"prefill": f"1 x {n}", "decode": f"16 x {n} cache"}, "hidden": hidden, "h_q": hq,
           "h_kv": hkv, "d": d, "n_sel": w.n_sel, "weights": "random bf16 (no norm, no positional encoding)",
           "dense": "torch scaled_dot_product_attention, cuDNN / flash / efficient backend"}
    # ---- prefill: time to first token of one layer
    x = rand(n, hidden)
    cu = torch.tensor([0, n], dtype=torch.int32, device=dev)
    vl = T.make_varlen([n], cu, p)
    Kc1 = torch.empty(hkv, vl.total_c1, d, dtype=torch.bfloat16, device=dev)
    Kc2 = torch.empty(hkv, vl.total_c2, d, dtype=torch.bfloat16, device=dev)
    ld = T.infllm2_scores_ld(vl, p)
    S = torch.empty(hkv, n, ld, dtype=torch.float32, device=dev)
    idx = torch.empty(hkv, n, p.n_sel, dtype=torch.int32, device=dev)
    o = torch.empty(n, hq, d, dtype=torch.bfloat16, device=dev)
    sws = torch.empty(T.infllm2_sparse_workspace_bytes(vl, hq), dtype=torch.uint8, device=dev)

    def sparse_prefill():
        q = (x @ Wq).view(n, hq, d)
        k = (x @ Wk).view(n, hkv, d)
        v = (x @ Wv).view(n, hkv, d)
        T.infllm2_compress_k(k, vl, Kc1, Kc2, p)
        T.infllm2_shared_scores(q, Kc1, Kc2, vl, hkv, S, ld, p)
        T.infllm2_topk_blocks(S, ld, vl, hkv, idx, p)
        T.infllm2_sparse_attn(q, k, v, idx, vl, o, p, workspace=sws)
        return o.view(n, hidden) @ Wo

    def dense_prefill():
        q = (x @ Wq).view(1, n, hq, d).transpose(1, 2)
        k = (x @ Wk).view(1, n, hkv, d).transpose(1, 2)
        v = (x @ Wv).view(1, n, hkv, d).transpose(1, 2)
        with sdpa_kernel(backends):
            a = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        return a.transpose(1, 2).reshape(n, hidden) @ Wo

    res["ttft_ms"] = {"sparse": timed(sparse_prefill)}
    try:
        res["ttft_ms"]["dense"] = timed(dense_prefill)
        res["ttft_speedup"] = res["ttft_ms"]["dense"] / res["ttft_ms"]["sparse"]
    except RuntimeError as e:                  # no fused SDPA backend for this shape
        res["ttft_ms"]["dense"] = None
        res["dense_error"] = str(e).splitlines()[0][:200]
    del x, Kc1, Kc2, S, idx, o, sws
    torch.cuda.empty_cache()
    # ---- decode: time per output token of one layer
    batch, cap = 16, n + decode_steps + 1
    k_cache = rand(batch, cap, hkv, d)
    v_cache = rand(batch, cap, hkv, d)
    kc1 = torch.empty(batch, hkv, T.window_count(cap, 32, 16), d, dtype=torch.bfloat16, device=dev)
    kc2 = torch.empty(batch, hkv, T.window_count(cap, 128, 64), d, dtype=torch.bfloat16, device=dev)
    seq_len = torch.full((batch,), n, dtype=torch.int32, device=dev)
    st = T.make_decode_state(k_cache, v_cache, kc1, kc2, seq_len, hq)
    ws = torch.empty(T.infllm2_decode_workspace_bytes(st, p), dtype=torch.uint8, device=dev)
    od = torch.empty(batch, hq, d, dtype=torch.bfloat16, device=dev)
    T.infllm2_decode_build_caches(st, p)
    xd = rand(batch, hidden)

    def sparse_decode():
        q = (xd @ Wq).view(batch, hq, d)
        kn = (xd @ Wk).view(batch, hkv, d)
        vn = (xd @ Wv).view(batch, hkv, d)
        T.infllm2_decode_step(st, q, kn, vn, od, ws, p)
        return od.view(batch, hidden) @ Wo

    def reset():
        seq_len.fill_(n)

    res["tpot_us"] = {"sparse": 1e3 * timed(sparse_decode, decode_steps, before=reset)}
    reset()
    del k_cache, v_cache, kc1, kc2, ws
    torch.cuda.empty_cache()
    kd = rand(batch, hkv, n, d)                # the dense cache, laid out for SDPA
    vd = rand(batch, hkv, n, d)

    def dense_decode():
        q = (xd @ Wq).view(batch, hq, 1, d)
        with sdpa_kernel(backends):
            a = F.scaled_dot_product_attention(q, kd, vd, enable_gqa=True)
        return a.reshape(batch, hidden) @ Wo

    try:
        res["tpot_us"]["dense"] = 1e3 * timed(dense_decode, decode_steps)
        res["tpot_speedup"] = res["tpot_us"]["dense"] / res["tpot_us"]["sparse"]
    except RuntimeError as e:
        res["tpot_us"]["dense"] = None
        res["dense_decode_error"] = str(e).splitlines()[0][:200]
    res["device_status"] = T.infllm2_get_device_status()
    return res


def bench_decode(T, gen, torch, dev, graph_steps: int = 64, reps: int = 3, batch: int = 0):
    """µs per decode step of the 16 x 131072 workload, steps replayed from a
    CUDA graph of `graph_steps` consecutive steps (inputs staged on device).
    `batch` > 0 runs fewer sequences (a smaller case for profiling)."""
    w = gen.WORKLOADS["decode_16x128k"]
    prefix, steps, batch = w.seqlen, graph_steps, (batch or w.batch)
    cap = prefix + steps
    p = T.default_params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k)
    k_cache = torch.empty(batch, cap, w.h_kv, w.d, dtype=torch.bfloat16, device=dev)
    v_cache = torch.empty_like(k_cache)
    q_all = torch.empty(steps, batch, w.h_q, w.d, dtype=torch.bfloat16, device=dev)
    kn_all = torch.empty(steps, batch, w.h_kv, w.d, dtype=torch.bfloat16, device=dev)
    vn_all = torch.empty_like(kn_all)
    for b in range(batch):
        one = gen.make_decode_sequence(w, b, prefix, steps)
        k_cache[b] = one["K"].to(dev)
        v_cache[b] = one["V"].to(dev)
        q_all[:, b] = one["q_steps"].to(dev)
        kn_all[:, b] = one["K"][prefix:].to(dev)
        vn_all[:, b] = one["V"][prefix:].to(dev)
    kc1 = torch.empty(batch, w.h_kv, T.window_count(cap, 32, 16), w.d, dtype=torch.bfloat16, device=dev)
    kc2 = torch.empty(batch, w.h_kv, T.window_count(cap, 128, 64), w.d, dtype=torch.bfloat16, device=dev)
    seq_len = torch.full((batch,), prefix, dtype=torch.int32, device=dev)
    st = T.make_decode_state(k_cache, v_cache, kc1, kc2, seq_len, w.h_q)
    ws = torch.empty(T.infllm2_decode_workspace_bytes(st, p), dtype=torch.uint8, device=dev)
    out = torch.empty(batch, w.h_q, w.d, dtype=torch.bfloat16, device=dev)
    T.infllm2_decode_build_caches(st, p)
    stream = torch.cuda.Stream()
    prefix_t = torch.full((batch,), prefix, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    # one eager pass (warm-up, and the first call on the device)
    with torch.cuda.stream(stream):
        for i in range(steps):
            T.infllm2_decode_step(st, q_all[i], kn_all[i], vn_all[i], out, ws, p, stream)
        seq_len.copy_(prefix_t)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            T.infllm2_decode_step(st, q_all[i], kn_all[i], vn_all[i], out, ws, p, stream)
    times = []
    for _ in range(reps + 1):
        seq_len.copy_(prefix_t)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):          # replay and both events on the same stream
            a.record(stream)
            g.replay()
            b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    status = T.infllm2_get_device_status()
    ms = statistics.median(times[1:])
    us = 1e3 * ms / steps
    byts = decode_bytes_per_step(prefix, steps, batch, w.h_kv, w.d)
    del g
    return {"workload": w.name, "us_per_step": us, "graph_steps": steps, "batch": batch, "cache": prefix,
            "launches_per_step": 3, "bytes_per_step": byts, "achieved_GB/s": byts / (us / 1e6) / 1e9,
            "device_status": status}


def bench_varlen(T, gen, torch, dev, hbm: float, tflops_burst: float, reps: int = 5, warmup: int = 3,
                 sm_mhz: float = 1965.0) -> dict:
    """The dense/sparse switch on the packed 131072-token varlen workload:
    sequences of at most 8192 tokens run the dense causal kernel (one call
    over their packed batch), the others the sparse path (pool, scores,
    top-k, sparse attention over their packed batch).  tokens/s = all packed
    tokens / (dense time + sparse time), CUDA events on one stream."""
    w = gen.WORKLOADS["varlen_128k"]
    data = gen.make_prefill(w)
    p = T.default_params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k)
    lens = list(data["lens"])
    cu = data["cu_seqlens"].tolist()
    dense_ids = [i for i, n in enumerate(lens) if n <= p.dense_threshold]
    sparse_ids = [i for i, n in enumerate(lens) if n > p.dense_threshold]

    def sub(ids):
        parts = {k: torch.cat([data[k][cu[i]:cu[i + 1]] for i in ids]).to(dev) for k in ("Q", "K", "V")}
        ls = [lens[i] for i in ids]
        c = torch.tensor([0] + list(np.cumsum(ls)), dtype=torch.int32, device=dev)
        return parts, ls, c

    stream = torch.cuda.current_stream()
    dq, dl, dc = sub(dense_ids)
    dvl = T.make_varlen(dl, dc, p)
    dout = torch.empty(dvl.total, w.h_q, w.d, dtype=torch.bfloat16, device=dev)
    sq, sl, sc = sub(sparse_ids)
    svl = T.make_varlen(sl, sc, p)
    Kc1 = torch.empty(w.h_kv, svl.total_c1, w.d, dtype=torch.bfloat16, device=dev)
    Kc2 = torch.empty(w.h_kv, svl.total_c2, w.d, dtype=torch.bfloat16, device=dev)
    ld = T.infllm2_scores_ld(svl, p)
    S = torch.empty(w.h_kv, svl.total, ld, dtype=torch.float32, device=dev)
    idx = torch.empty(w.h_kv, svl.total, p.n_sel, dtype=torch.int32, device=dev)
    sout = torch.empty(svl.total, w.h_q, w.d, dtype=torch.bfloat16, device=dev)
    sws = torch.empty(T.infllm2_sparse_workspace_bytes(svl, w.h_q), dtype=torch.uint8, device=dev)

    def step(ev=None):
        if ev is not None: ev[0].record(stream)
        T.infllm2_dense_attn(dq["Q"], dq["K"], dq["V"], dvl, dout, p, stream)
        if ev is not None: ev[1].record(stream)
        T.infllm2_compress_k(sq["K"], svl, Kc1, Kc2, p, stream)
        T.infllm2_shared_scores(sq["Q"], Kc1, Kc2, svl, w.h_kv, S, ld, p, stream)
        T.infllm2_topk_blocks(S, ld, svl, w.h_kv, idx, p, stream)
        T.infllm2_sparse_attn(sq["Q"], sq["K"], sq["V"], idx, svl, sout, p, stream, workspace=sws)
        if ev is not None: ev[2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for k in range(reps):
        step(evs[k])
    torch.cuda.synchronize()
    t_dense = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    t_sparse = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    # the dense kernel's roofline: 4 d h_q flop and h_q exps per causal (t, u <= t) pair
    pairs = sum(n * (n + 1) // 2 for n in dl)
    flops = 4 * w.d * w.h_q * pairs
    exps = w.h_q * pairs
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu = 16.0 * nsm * sm_mhz * 1e6
    t_tensor, t_sfu = flops / (tflops_burst * 1e12), exps / sfu
    dense_roof = {"bound": "tensor" if t_tensor >= t_sfu else "sfu", "flops": flops, "exps": exps,
                  "achieved_TFLOP/s": flops / (t_dense / 1e3) / 1e12, "peak_TFLOP/s": tflops_burst,
                  "frac_tensor": flops / (t_dense / 1e3) / 1e12 / tflops_burst,
                  "roofline_ms": 1e3 * max(t_tensor, t_sfu), "frac": 1e3 * max(t_tensor, t_sfu) / t_dense,
                  "peak_source": "MEASURED_PEAKS bf16 burst; ex2 at 16 per SM per clock"}
    total = dvl.total + svl.total
    status = T.infllm2_get_device_status()
    return {"workload": w.name, "tokens": total, "sequences": len(lens), "dense_sequences": len(dense_ids),
            "sparse_sequences": len(sparse_ids), "dense_tokens": dvl.total, "sparse_tokens": svl.total,
            "ms_per_step": t_dense + t_sparse, "dense_ms": t_dense, "sparse_ms": t_sparse,
            "tokens/s": total / ((t_dense + t_sparse) / 1e3), "dense_kernel_roofline": dense_roof,
            "steps": reps, "warmup": warmup, "device_status": status}


def bench_backward(T, gen, torch, dev, w, data, p, Q, K, V, idx, out, sws, vl, stream, reps: int = 3,
                   warmup: int = 2, tflops: float = 1694.5) -> dict:
    """The backward of the block-sparse attention on the bench workload (the
    forward's lists, output and row log-sum-exps from the timed step): dQ, dK,
    dV in fp32.  ms per backward call, CUDA events on the launching stream."""
    total = vl.total
    lse = sws[: total * w.h_q * 4].view(torch.float32).view(total, w.h_q)
    dout = gen.make_grad_out(total, w.h_q, w.d, 7).to(dev)
    ws = torch.empty(T.infllm2_sparse_backward_workspace_bytes(vl, w.h_q, w.h_kv, p), dtype=torch.uint8, device=dev)
    dQ = torch.empty(total, w.h_q, w.d, dtype=torch.float32, device=dev)
    dK = torch.empty(total, w.h_kv, w.d, dtype=torch.float32, device=dev)
    dV = torch.empty_like(dK)

    def step():
        T.infllm2_sparse_attn_backward(Q, K, V, out, dout, lse, idx, vl, dQ, dK, dV, ws, p, stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        b.synchronize()
        ts.append(a.elapsed_time(b))
    ms = statistics.median(ts)
    # contractions: dQ pass 3 products and dK/dV pass 4 products of 2 d flop
    # per (row, attended key): S, dP, dQ / S, dP, dV, dK
    n1, n2, keys, shared_keys, topk_keys = visible_counts(w.seqlen, w.n_init, w.n_local, w.top_k)
    flops = (3 + 4) * 2 * w.d * w.h_q * int(keys.sum())
    status = T.infllm2_get_device_status()
    del ws, dQ, dK, dV, dout
    return {"workload": w.name, "ms": ms, "tokens/s": total / (ms / 1e3), "launches": 8,
            "flops": flops, "TFLOP/s": flops / (ms / 1e3) / 1e12, "frac_tensor": flops / (ms / 1e3) / 1e12 / tflops,
            "peak_source": "MEASURED_PEAKS bf16 burst", "outputs": "dQ, dK, dV fp32", "device_status": status}


# ---------------------------------------------------------------- main
def config_of(w, args, world: int) -> dict:
    return {"workload": w.name, "seq_len": w.seqlen, "h_q": w.h_q, "h_kv": w.h_kv, "d": w.d,
            "n_sel": w.n_sel, "lse": args.lse, "pool": args.pool,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "working set larger than L2 (Q 1 GiB; S_shared 4.3 GB, or its pooled pairs 2.2 GB); no extra flush"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed varlen dense/sparse switch workload")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward (dQ, dK, dV) timing")
    ap.add_argument("--decode-only", action="store_true", help="time only the decode workload (for profiling)")
    ap.add_argument("--layer", action="store_true",
                    help="time one attention layer with random weights: sparse vs dense TTFT (128K prefill) and "
                         "TPOT (16 x 128K decode)")
    ap.add_argument("--decode-steps", type=int, default=64)
    ap.add_argument("--decode-batch", type=int, default=0, help="sequences of the decode case (0: the workload's 16)")
    ap.add_argument("--pool", default="s_shared", choices=["fused", "s_shared"],
                    help="fused: the score kernel writes the max-pool's (max, last window) pairs; s_shared: it writes "
                         "S_shared and the selection pools it")
    ap.add_argument("--lse", default="approx", choices=["approx", "exact"],
                    help="LSE of the scoring step: the coarse approximation (default) or the exact two-pass form")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from inputs import gen
    w = gen.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        # The oracle as it stands, on the host cores.  One step is a bounded
        # sample of the workload: R uniformly sampled (token, group) rows
        # (scores, selection, attention); the pooling of the whole sequence is
        # timed once before the steps.  `value` extrapolates the per-row time
        # to every row of the sequence plus the pooling; `ms_per_step` is the
        # wall time of one sample step as actually run.
        from threadpoolctl import threadpool_limits
        ncores = len(os.sched_getaffinity(0))
        data = gen.make_prefill(w)
        with threadpool_limits(limits=ncores):
            seq, t_pool = oracle_sequence(w, data, args.lse)
            probe = oracle_rows(seq, 8, 7) / 8
            R = max(8, int(args.cpu_seconds / max(1, args.steps) / max(probe, 1e-4)))
            for k in range(args.warmup):
                oracle_rows(seq, max(1, R // 8), 1000 + k)
            times = [oracle_rows(seq, R, 2000 + k) for k in range(args.steps)]
        per_row = sum(times) / (R * args.steps)
        tok_s = seq.n / (t_pool + per_row * seq.n * seq.h_kv)
        sample = (f"fp64 oracle, NumPy/BLAS threads = {ncores}: {args.steps} steps of {R} uniformly sampled "
                  f"(token, group) rows (warm-up steps of {max(1, R // 8)} rows), pooling of the whole "
                  f"{w.seqlen}-token sequence timed once ({t_pool:.1f} s); extrapolated to all "
                  f"{seq.n * seq.h_kv} rows")
        line = {
            "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
            "extrapolated": True, "rows_per_step": R, "ms_per_full_step_extrapolated": 1e3 * w.seqlen / tok_s,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) Q,V; K with per-block offsets)",
            "config": config_of(w, args, 1),
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": ncores, "kind": "oracle", "sample": sample,
                             "extrapolated": True},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    import trainable_block_sparse_pool_b200 as T

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    T.lib()

    if args.layer:
        clocks = ClockSampler()
        clocks.start()
        res = bench_layer(T, gen, torch, dev)
        res["clocks"] = clocks.stop()
        if rank == 0:
            print(json.dumps({"layer": res}), flush=True)
        return

    if args.decode_only:
        dd = bench_decode(T, gen, torch, dev, graph_steps=args.decode_steps, batch=args.decode_batch)
        if rank == 0:
            print(json.dumps({"decode": dd}), flush=True)
        return

    data = gen.make_prefill(w)
    p = T.default_params(n_init=w.n_init, n_local=w.n_local, top_k=w.top_k,
                         lse_mode=T.LSE_EXACT if args.lse == "exact" else T.LSE_APPROX)
    Q, K, V = data["Q"].to(dev), data["K"].to(dev), data["V"].to(dev)
    cu = data["cu_seqlens"].to(dev)
    vl = T.make_varlen(data["lens"], cu, p)
    Kc1 = torch.empty(w.h_kv, vl.total_c1, w.d, dtype=torch.bfloat16, device=dev)
    Kc2 = torch.empty(w.h_kv, vl.total_c2, w.d, dtype=torch.bfloat16, device=dev)
    fused = args.pool == "fused"
    ld = T.infllm2_pooled_ld(vl, p) if fused else T.infllm2_scores_ld(vl, p)
    S = torch.empty(w.h_kv, vl.total, ld, dtype=torch.float32, device=dev)   # pairs or S_shared
    idx = torch.empty(w.h_kv, vl.total, p.n_sel, dtype=torch.int32, device=dev)
    out = torch.empty(vl.total, w.h_q, w.d, dtype=torch.bfloat16, device=dev)
    sws = torch.empty(T.infllm2_sparse_workspace_bytes(vl, w.h_q), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    kernels = ["compress", "scores", "topk", "sparse"]

    def step(ev=None, bufs=None):
        q, k, v, o = bufs if bufs is not None else (Q, K, V, out)
        if ev is not None: ev[0].record(stream)
        T.infllm2_compress_k(k, vl, Kc1, Kc2, p, stream)
        if ev is not None: ev[1].record(stream)
        if fused:
            T.infllm2_pooled_scores(q, Kc1, Kc2, vl, w.h_kv, S, ld, p, stream)
        else:
            T.infllm2_shared_scores(q, Kc1, Kc2, vl, w.h_kv, S, ld, p, stream)
        if ev is not None: ev[2].record(stream)
        if fused:
            T.infllm2_topk_blocks_pooled(S, ld, vl, w.h_kv, idx, p, stream)
        else:
            T.infllm2_topk_blocks(S, ld, vl, w.h_kv, idx, p, stream)
        if ev is not None: ev[3].record(stream)
        T.infllm2_sparse_attn(q, k, v, idx, vl, o, p, stream, workspace=sws)
        if ev is not None: ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if T.infllm2_get_device_status() != 0:
        raise RuntimeError("device status after warm-up: %d" % T.infllm2_get_device_status())

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    clocks = ClockSampler()
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    per_kernel = {nm: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs) for i, nm in enumerate(kernels)}
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    tokens = w.seqlen * world
    value = tokens / (ms_per_step / 1e3)
    status = T.infllm2_get_device_status()

    # ---- e2e through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        Qh, Kh, Vh = data["Q"].pin_memory(), data["K"].pin_memory(), data["V"].pin_memory()
        outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            Q.copy_(Qh, non_blocking=True); K.copy_(Kh, non_blocking=True); V.copy_(Vh, non_blocking=True)
            step()
            outh.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        serial_ms = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        h2d = sum(x.numel() * x.element_size() for x in (Qh, Kh, Vh))
        d2h = outh.numel() * outh.element_size()

        # Pipelined: two sets of device inputs and outputs, the uploads on one
        # stream and the downloads on another, so the copies of steps k+1 and
        # k-1 run under the kernels of step k.  Every step still copies its own
        # Q, K, V in from pinned host memory and its output back, inside the
        # timed region.
        sets = [(Q, K, V, out), (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(out))]
        outs_h = [outh, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def run_pipelined(n):
            for kk in range(n):
                bsel = kk & 1
                q, k, v, o = sets[bsel]
                if kk >= 2:
                    up.wait_event(ev_done[bsel])       # step kk-2 has finished reading this set
                with torch.cuda.stream(up):
                    q.copy_(Qh, non_blocking=True); k.copy_(Kh, non_blocking=True); v.copy_(Vh, non_blocking=True)
                    ev_in[bsel].record(up)
                stream.wait_event(ev_in[bsel])
                if kk >= 2:
                    stream.wait_event(ev_out[bsel])    # step kk-2's output has been read back
                step(bufs=sets[bsel])
                ev_done[bsel].record(stream)
                down.wait_event(ev_done[bsel])
                with torch.cuda.stream(down):
                    outs_h[bsel].copy_(o, non_blocking=True)
                    ev_out[bsel].record(down)
            for e in ev_out:
                stream.wait_event(e)

        run_pipelined(4)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        up.wait_event(a); down.wait_event(a)
        run_pipelined(args.steps)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / args.steps, dev)
        e2e = {"value": tokens / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "pipelined": "two buffer sets; uploads and downloads on their own streams overlap the kernels of "
                            "the neighbouring steps",
               "serial": {"value": tokens / (serial_ms / 1e3), "unit": "tokens/s", "ms_per_step": serial_ms}}

    # ---- L2 -> SM gather bandwidth with the attention's tile shape (this run)
    l2 = measure_l2_gather(T, torch, K, V, stream)

    # ---- roofline of the dominant kernel
    hbm, tflops, tflops_sus, src = _peaks()
    work = algorithmic_work(w.seqlen, w.h_q, w.h_kv, w.d)
    if fused:
        work["score_bytes"], work["topk_bytes"] = work["score_bytes_pooled"], work["topk_bytes_pooled"]
    dom = max(per_kernel, key=per_kernel.get)
    if dom == "sparse":
        # the attention is bound by moving the selected K/V rows from L2 to
        # the SMs: algorithmic bytes = the top-k blocks per (token, group) +
        # the shared init/local blocks once per 64-token query block and group
        ach = work["sparse_gather_bytes"] / (per_kernel["sparse"] / 1e3) / 1e9
        tflop = work["sparse_flops"] / (per_kernel["sparse"] / 1e3) / 1e12
        roof = {"kernel": "sparse_attn (top-k gather + shared init/local tiles)", "bound": "l2", "achieved": ach,
                "peak": l2["GB/s"], "unit": "GB/s", "frac": ach / l2["GB/s"], "traffic": None,
                "algorithmic_bytes": work["sparse_gather_bytes"],
                "kernel_gather_bytes": work["sparse_topk_gather_bytes"] + work["sparse_shared_gather_bytes_kernel"],
                "peak_source": "L2 -> SM gather bandwidth measured in this run by the library's own probe "
                               "(infllm2_probe_l2_gather, same tile shape); no driver-measured L2 figure exists",
                "tensor": {"achieved": tflop, "peak": tflops, "unit": "TFLOP/s", "frac": tflop / tflops,
                           "peak_source": f"{src} bf16 burst (MEASURED_PEAKS)"},
                "hbm_traffic_note": "DRAM bytes come from ncu captures, summarised under profiles/"}
    elif dom == "scores":
        ach = work["score_flops"] / (per_kernel["scores"] / 1e3) / 1e12
        roof = {"kernel": "shared_scores", "bound": "tensor", "achieved": ach, "peak": tflops, "unit": "TFLOP/s",
                "frac": ach / tflops, "traffic": None, "peak_source": f"{src} bf16 burst"}
    else:
        b = work[f"{dom}_bytes"]
        ach = b / (per_kernel[dom] / 1e3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                "traffic": None, "peak_source": f"{src} HBM copy"}

    # ---- the whole step against the sum of its steps' rooflines (each step's
    # time bound = the slowest of tensor, SFU exp, HBM and L2-gather time)
    sm_mhz = (clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0) if isinstance(clk, dict) else 1965.0
    nsm = torch.cuda.get_device_properties(dev).multi_processor_count
    sfu = 16.0 * nsm * sm_mhz * 1e6            # ex2 per second: 16 per SM per clock
    tens = tflops_sus * 1e12                   # a long step: the sustained GEMM figure
    bw = hbm * 1e9
    l2bw = l2["GB/s"] * 1e9
    t_roof = {
        "compress": work["compress_bytes"] / bw,
        "scores": max(work["score_flops"] / tens, work["score_exps"] / sfu, work["score_bytes"] / bw),
        "topk": work["topk_bytes"] / bw,
        "sparse": max(work["sparse_flops"] / tens, work["sparse_exps"] / sfu, work["sparse_gather_bytes"] / l2bw),
    }
    step_roof = {"roofline_ms": {k: v * 1e3 for k, v in t_roof.items()},
                 "measured_ms": dict(per_kernel),
                 "frac": sum(t_roof.values()) * 1e3 / ms_per_step,
                 "peaks": {"tensor_TFLOP/s": tflops_sus, "sfu_Gexp/s": sfu / 1e9, "hbm_GB/s": hbm,
                           "l2_gather_GB/s": l2["GB/s"], "sm_mhz": sm_mhz}}

    kern_detail = {}
    for nm in kernels:
        ms = per_kernel[nm]
        d_ = {"ms": ms}
        if nm == "compress":
            d_["GB/s"] = work["compress_bytes"] / (ms / 1e3) / 1e9
        elif nm == "scores":
            d_["TFLOP/s"] = work["score_flops"] / (ms / 1e3) / 1e12
            d_["Gexp/s"] = work["score_exps"] / (ms / 1e3) / 1e9
        elif nm == "topk":
            d_["GB/s"] = work["topk_bytes"] / (ms / 1e3) / 1e9
        elif nm == "sparse":
            d_["TFLOP/s"] = work["sparse_flops"] / (ms / 1e3) / 1e12
            d_["gather_GB/s"] = work["sparse_gather_bytes"] / (ms / 1e3) / 1e9
        kern_detail[nm] = d_

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) Q,V; K with per-block offsets)",
        "config": config_of(w, args, world),
        "e2e": e2e,
        "gpu_launches": (len(kernels) + 2) * args.steps,   # the sparse call is three launches (list check, top-k, local)
        "kernels": kern_detail,
        "roofline": roof,
        "step_roofline": step_roof,
        "l2_gather_probe": l2,
        "clocks": clk,
        "device_status": status,
    }
    if not args.no_decode:
        dd = bench_decode(T, gen, torch, dev, graph_steps=args.decode_steps)
        dd["peak_GB/s"] = hbm
        dd["frac"] = dd["achieved_GB/s"] / hbm
        dd["bound"] = "hbm"
        line["decode"] = dd
    if not args.no_backward:
        line["backward"] = bench_backward(T, gen, torch, dev, w, data, p, Q, K, V, idx, out, sws, vl, stream,
                                          tflops=tflops)
    if not args.no_varlen:
        line["varlen"] = bench_varlen(T, gen, torch, dev, hbm, tflops, sm_mhz=sm_mhz)
        line["gpu_launches_varlen_step"] = 7   # dense; compress, scores, top-k, sparse (three launches)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_entry(w, data, args.cpu_seconds, args.lse)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
