#!/usr/bin/env python
"""Benchmark: batched multi-agent decode over packed low-bit KV caches.

Headline workload (the largest decode configuration that fits one GPU; one
step = one decode token for every agent): variable-length decode in
Gemma-3-12B shape, 6 agents x 48 layers, 16 query / 8 KV heads, head_dim 256,
packed lengths per agent drawn from {4K, 8K, 16K, 32K}, 4-bit group-64 codes
plus a full 256-token bf16 recent window, K outlier channels x10.  Per layer
the step runs kvq_append_decode_attn over that layer's views: the new token
enters the window, the oldest window token is quantized into the packed part,
and attention runs over the result.  The 48 calls of a step are replayed from
one CUDA graph; the per-step working set (11 GB) is far larger than L2, so no
flush is needed between steps.

Measured beside it, each with the same fields (step, dominant kernel
roofline, one call over all views, end to end through the C ABI, CPU oracle,
clocks):
  llama8b   10 agents x 32 layers, Llama-3.1-8B shape, 4096 packed 4-bit
            tokens + 128-token window per view;
  qwen32b   8 agents x 64 layers, Qwen3-32B shape, 64 q / 8 kv heads,
            packed lengths in [8K, 16K], per-(agent, layer) widths
            {2, 3, 4, 8} with mean 3 bits, 128-token window;
and the bulk handoff codec (quantize then dequantize one agent's 32-layer x
8-head x 32768-token x 128 K and V cache, 4-bit).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--legs gemma12b,llama8b,qwen32b] [--skip-codec] [--skip-cpu]

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import csv
import ctypes
import io
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn packed-KV GB/s & tokens/s/agent, % of HBM peak; quantize GB/s"
HEADLINE = "gemma12b"
WORKLOADS = {
    "gemma12b": ("variable-length decode, Gemma-3-12B shape: 6 agents x 48 layers, 16 q / 8 kv heads, head_dim 256, "
                 "packed lengths per agent drawn from {4096, 8192, 16384, 32768}, 4-bit group-64 codes + 256-token "
                 "bf16 window per view, K outlier channels x10, one decode token per agent per step"),
    "llama8b": ("batched multi-agent decode, Llama-3.1-8B shape: 10 agents x 32 layers, 32 q / 8 kv heads, "
                "head_dim 128, 4096 packed 4-bit group-64 tokens + 128-token bf16 window per view, "
                "one decode token per agent per step"),
    "qwen32b": ("mixed-precision multi-agent decode, Qwen3-32B shape: 8 agents x 64 layers, 64 q / 8 kv heads, "
                "head_dim 128, packed lengths uniform in [8192, 16384], per-(agent, layer) widths {2, 3, 4, 8} with "
                "mean 3 bits, group-64 codes + 128-token bf16 window, K outlier channels x10, one decode token per "
                "agent per step"),
}
# the profile summary of each workload's dominant kernel (ncu DRAM bytes per launch)
PROFILES = {"gemma12b": "decode_attn_layer_gemma12b.md", "llama8b": "decode_attn_layer_llama8b.md",
            "qwen32b": "decode_attn_layer_qwen32b.md"}


def workload(key, rank=0):
    from quantized_kv_cache_dequantize_b200 import workloads as wl
    # every rank holds its own agents (weak scaling): the same shapes, other draws
    if key == "gemma12b":
        return wl.varlen_gemma12b(seed=4 + 1000 * rank)
    if key == "llama8b":
        return wl.decode_llama8b(seed=3 + 1000 * rank)
    return wl.mixed_qwen32b(seed=5 + 1000 * rank)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# ------------------------------------------------------------- byte counts --

def view_attn_bytes(H, Hq, D, n_p, n_w, bits):
    """Algorithmic bytes of attention over one view: packed K and V codes and
    their scale/min, bf16 window K and V, bf16 q in, fp32 out."""
    rb = D // 8 * bits
    return H * (n_p * (2 * rb + 2 * (D // 64) * 8) + n_w * 2 * D * 2) + Hq * D * 2 + Hq * D * 4


def attn_bytes(n_views, Hkv, Hq, D, n_p, n_w, bits):
    """n_views identical views (kept for callers that count a uniform workload)."""
    return n_views * view_attn_bytes(Hkv, Hq, D, n_p, n_w, bits)


def views_attn_bytes(views, Hq):
    return sum(view_attn_bytes(v.n_kv_heads, Hq, v.head_dim, v.n_packed, v.n_window, v.bits) for v in views)


def view_append_bytes(H, D, bits):
    """kvq_append with a full window: read the new K/V token and the flushed
    window row, write the packed row (+ scale/min) and the window row."""
    rb = D // 8 * bits
    return 2 * H * (D * 2 + D * 2 + rb + (D // 64) * 8 + D * 2)


def views_append_bytes(views):
    return sum(view_append_bytes(v.n_kv_heads, v.head_dim, v.bits) for v in views)


def append_bytes(n_views, Hkv, D, bits):
    return n_views * view_append_bytes(Hkv, D, bits)


def launches_per_call(views):
    """Kernel launches of one kvq_append_decode_attn over these views: the
    append grids (128 views each) and one attention grid per width group of
    up to 96 views."""
    from collections import Counter
    n_app = -(-len(views) // 128)
    groups = Counter(v.bits for v in views if v.n_packed > 0)
    return n_app + sum(-(-c // 96) for c in groups.values())


# ------------------------------------------------------------ clock sampler --

class ClockSampler:
    """nvidia-smi samples (every 20 ms) of the SM clock, power and throttle
    reasons, each with its timestamp; mark() brackets the timed region and
    summary() keeps the samples inside it (the nearest three when the region
    is shorter than the sampling interval)."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def __exit__(self, *exc):
        self.out = ""
        time.sleep(0.05)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    @staticmethod
    def _num(x):
        try:
            return float(x)
        except ValueError:
            return None

    def summary(self):
        import datetime
        if not getattr(self, "out", ""):
            return None
        rows = []
        for r in csv.reader(io.StringIO(self.out)):
            r = [c.strip() for c in r]
            if len(r) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, r))
        if not rows:
            return None
        where = "inside the timed region"
        if self.t0 is not None and self.t1 is not None:
            inside = [x for x in rows if self.t0 <= x[0] <= self.t1]
            if not inside:
                mid = 0.5 * (self.t0 + self.t1)
                inside = sorted(rows, key=lambda x: abs(x[0] - mid))[:3]
                where = "nearest to the timed region (shorter than the sampling interval)"
            rows = inside
        sm = [v for v in (self._num(r[2]) for _, r in rows) if v is not None]
        mx = max((v for v in (self._num(r[3]) for _, r in rows) if v is not None), default=None)
        pw = [v for v in (self._num(r[4]) for _, r in rows) if v is not None]
        reasons = set()
        for _, r in rows:
            for name, val in zip(self.REASONS, r[6:10]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(rows), "samples_are": where,
                "power_w": float(np.median(pw)) if pw else None}


# ------------------------------------------------------------------ helpers --

def ev_pair():
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def kernel_source_sha():
    """sha256 of the decode-attention kernel sources (ties ncu counters to a kernel version)."""
    import hashlib
    h = hashlib.sha256()
    for f in ("kvq_attn.cuh", "kvq_ptx.cuh"):
        with open(os.path.join(ROOT, "quantized_kv_cache_dequantize_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(key):
    """DRAM bytes per launch of a workload's per-layer decode-attention call
    from its committed ncu summary, if that was taken on the current kernel
    source."""
    path = os.path.join(ROOT, "profiles", PROFILES[key])
    try:
        vals = {}
        for line in open(path):
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
        if vals.get("kernel_source_sha256") == kernel_source_sha():
            return float(vals["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


def time_graph(graph, stream, warmup, steps, clk=None):
    """Mean device time of one replay (CUDA events on the replay stream); clk
    (a ClockSampler) is marked around the timed replays."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            graph.replay()
        stream.synchronize()
        e0, e1 = ev_pair()
        if clk is not None:
            clk.mark(True)
        e0.record(stream)
        for _ in range(steps):
            graph.replay()
        e1.record(stream)
    stream.synchronize()
    if clk is not None:
        clk.mark(False)
    return e0.elapsed_time(e1) / 1e3 / steps


# ------------------------------------------------------------ oracle timing --

def _prepare_oracle_views(w, views_idx, device, threads=1):
    """Oracle inputs of some views (quantized by the oracle itself, on host
    threads; untimed): list of (q bits, bits, kc, ks, vc, vs, kw, vw, bytes)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    from quantized_kv_cache_dequantize_b200 import cache as kcache, workloads as wl
    q_all = kcache.decode_queries(w, device=device)
    raw = []
    for (a, l) in views_idx:
        k, v, head = kcache.view_inputs(w, a, l, device=device)
        raw.append((a, l, wl.bf16_bits(k), wl.bf16_bits(v), wl.bf16_bits(q_all[a * w.n_layers + l])))

    def prep(item):
        a, l, kb, vb, qv = item
        n_p = w.view_len(a)
        bits = w.view_bits(a, l)
        kc, ks = oracle.quantize(kb[:, :n_p], bits)
        vc, vs = oracle.quantize(vb[:, :n_p], bits)
        nb = view_attn_bytes(w.n_kv_heads, w.n_q_heads, w.head_dim, n_p, w.window, bits)
        return (qv, bits, kc, ks, vc, vs, np.ascontiguousarray(kb[:, n_p:]), np.ascontiguousarray(vb[:, n_p:]), nb)

    with ThreadPoolExecutor(max(1, threads)) as pool:
        return list(pool.map(prep, raw))


def oracle_sample(w, views_idx, device="cuda"):
    """Time the fp64 CPU oracle on some views of a decode workload, one
    thread.  Returns (seconds of attention, algorithmic bytes of those views)."""
    import oracle
    prepared = _prepare_oracle_views(w, views_idx, device, threads=len(os.sched_getaffinity(0)))
    secs, nbytes = 0.0, 0
    for (qv, bits, kc, ks, vc, vs, kw, vw, nb) in prepared:
        t0 = time.perf_counter()
        oracle.decode_attn(qv, bits, kc, ks, vc, vs, kw, vw, w.softmax_scale)
        secs += time.perf_counter() - t0
        nbytes += nb
    return secs, nbytes


def oracle_threaded(w, views_idx, device="cuda"):
    """The same oracle attention as oracle_sample, split into one call per
    (view, KV head) and spread over every host core this process may use
    (the C oracle runs outside the GIL).  Returns (seconds, bytes, threads)."""
    from concurrent.futures import ThreadPoolExecutor

    import oracle
    threads = max(1, len(os.sched_getaffinity(0)))
    prepared = _prepare_oracle_views(w, views_idx, device, threads=threads)
    G = w.n_q_heads // w.n_kv_heads
    jobs, nbytes = [], 0
    for (qv, bits, kc, ks, vc, vs, kw, vw, nb) in prepared:
        for hk in range(w.n_kv_heads):
            h = slice(hk, hk + 1)
            jobs.append((qv[hk * G:(hk + 1) * G], bits, kc[h], ks[h], vc[h], vs[h], kw[h], vw[h]))
        nbytes += nb
    with ThreadPoolExecutor(threads) as pool:
        t0 = time.perf_counter()
        list(pool.map(lambda j: oracle.decode_attn(*j, w.softmax_scale), jobs))
        secs = time.perf_counter() - t0
    return secs, nbytes, threads


def cpu_sample_views(key, w):
    """The bounded sample of a workload the CPU oracle is timed on."""
    if key == "gemma12b":
        return [(a, 0) for a in range(w.n_agents)], "every agent at layer 0 (6 views, 4K-32K packed tokens)"
    if key == "llama8b":
        v = [(a, l) for l in range(0, 32, 8) for a in range(0, 10, 3)][:12]
        return v, "12 (agent, layer) views (8 kv heads x 4224 tokens each)"
    return [(a, 0) for a in range(w.n_agents)], "every agent at layer 0 (8 views, 8K-16K packed tokens, their widths)"


def cpu_baseline(key, w, device):
    views, desc = cpu_sample_views(key, w)
    secs, nb = oracle_sample(w, views, device)
    cpu = {"value": nb / secs / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{desc} of the decode workload, fp64 oracle attention, single thread, "
                     f"{secs:.1f} s of attention"}
    # the same oracle split over (view, KV head) on all host cores: context
    # only, so a failure here never costs the line
    try:
        tsecs, tnb, threads = oracle_threaded(w, views, device)
        cpu["threaded"] = {"value": tnb / tsecs / 1e9, "unit": "GB/s", "cores": threads,
                           "kind": "oracle, one call per (view, KV head) on host threads"}
    except Exception as e:  # noqa: BLE001
        cpu["threaded"] = {"error": f"{type(e).__name__}: {e}"}
    return cpu


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, as it stands, on the host cores, over
    the headline workload: each step one whole (agent, layer) view."""
    if rank != 0:
        return
    import oracle
    w = workload(HEADLINE)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    order = [(s % w.n_agents, (s // w.n_agents) % w.n_layers) for s in range(args.warmup + args.steps)]
    prepared = _prepare_oracle_views(w, order, dev, threads=len(os.sched_getaffinity(0)))
    secs, nbytes = 0.0, 0
    for s, (qv, bits, kc, ks, vc, vs, kw, vw, nb) in enumerate(prepared):
        t0 = time.perf_counter()
        oracle.decode_attn(qv, bits, kc, ks, vc, vs, kw, vw, w.softmax_scale)
        if s >= args.warmup:
            secs += time.perf_counter() - t0
            nbytes += nb
    gbs = nbytes / secs / 1e9
    sample = (f"one whole (agent, layer) view per step, agents in turn ({w.n_kv_heads} kv heads x 4K-32K packed "
              f"+ {w.window} window tokens), fp64 oracle attention, single thread")
    line = {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOADS[HEADLINE]},
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- ours ---

def decode_leg(key, args, rank, world, local, peak, peak_kind):
    """Every measurement of one decode workload; returns its record."""
    import quantized_kv_cache_dequantize_b200 as kvq
    from quantized_kv_cache_dequantize_b200 import cache as kcache, dist as kdist
    dev = torch.device("cuda", torch.cuda.current_device())
    w = workload(key, rank)
    L, A, H, Hq, D = w.n_layers, w.n_agents, w.n_kv_heads, w.n_q_heads, w.head_dim
    scale = w.softmax_scale
    # room for every append of this leg: two untimed steps at capture, the
    # eager end-to-end loop's warm-up and timed steps
    pool = kcache.build_decode(w, dev, extra_packed=2 * (args.warmup + args.steps) + 8)
    layer_views = [[pool.views[a * L + l] for a in range(A)] for l in range(L)]

    def layer_major(t):  # [A*L, ...] agent-major -> [L, A, ...]
        return t.view(A, L, *t.shape[1:]).transpose(0, 1).contiguous()

    q = layer_major(kcache.decode_queries(w, device=dev))
    kn, vn = (layer_major(t) for t in kcache.decode_new_tokens(w, device=dev))
    out = torch.empty((L, A, Hq, D), dtype=torch.float32, device=dev)
    # per layer: a workspace for the fused step, one for attention alone (the
    # views grow during the leg: twice the size they need now)
    ws_step = [torch.zeros(2 * kvq.step_workspace_size(lv, Hq) + (1 << 20), dtype=torch.uint8, device=dev)
               for lv in layer_views]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()

    def step():
        for l in range(L):
            kvq.append_decode_attn(layer_views[l], kn[l], vn[l], q[l], scale, out=out[l], workspace=ws_step[l],
                                   stream=stream)

    # capture one step in a graph; host view counters advance at capture, so
    # the graph replays the same (full-window) append + attend each time
    with torch.cuda.stream(stream):
        step()  # eager warm-up of every code path
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    stream.synchronize()
    all_views = [v for lv in layer_views for v in lv]
    bytes_step = views_attn_bytes(all_views, Hq) + views_append_bytes(all_views)
    launches_step = sum(launches_per_call(lv) for lv in layer_views)
    kdist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_step = time_graph(graph, stream, args.warmup, args.steps, clk)
    kdist.barrier()
    t_step = kdist.max_over_ranks(t_step)
    value = kdist.aggregate_throughput(bytes_step, world, t_step) / 1e9

    # dominant kernel: the attention grid(s) of one kvq_decode_attn per layer
    # (split-K combine included), the layers' calls replayed from one graph so
    # that host launch cost stays out of the device timing
    ws_attn = [kvq.new_workspace(lv, Hq, device=dev) for lv in layer_views]

    def attn_layers():
        for l in range(L):
            kvq.decode_attn(layer_views[l], q[l], scale, out=out[l], workspace=ws_attn[l], stream=stream)

    with torch.cuda.stream(stream):
        attn_layers()
    stream.synchronize()
    g_attn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_attn, stream=stream):
        attn_layers()
    t_attn = time_graph(g_attn, stream, args.warmup, args.steps) / L
    del g_attn
    attn_layer_bytes = views_attn_bytes(all_views, Hq) / L
    attn_gbs = attn_layer_bytes / t_attn / 1e9
    bits_set = sorted({v.bits for v in all_views})

    # one call over all views (graph-replayed)
    q_all = q.view(L * A, Hq, D)
    out_all = out.view(L * A, Hq, D)
    ws_all = kvq.new_workspace(all_views, Hq, device=dev)
    with torch.cuda.stream(stream):
        kvq.decode_attn(all_views, q_all, scale, out=out_all, workspace=ws_all, stream=stream)
    stream.synchronize()
    g_all = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all, stream=stream):
        kvq.decode_attn(all_views, q_all, scale, out=out_all, workspace=ws_all, stream=stream)
    t_all = time_graph(g_all, stream, max(3, args.warmup), args.steps)
    del g_all, ws_all
    all_gbs = views_attn_bytes(all_views, Hq) / t_all / 1e9

    # end to end through the C ABI with host buffers.  Every step copies its
    # q and new K/V in from pinned host memory and its output back out; the
    # copies run on a second stream, double-buffered through device staging
    # tensors, so the next step's inputs arrive and the previous step's
    # output leaves while a step computes (a serving loop's pipelining).  The
    # timed region spans the first input copy to the last output copy.
    q_h = q.cpu().pin_memory()
    kn_h, vn_h = kn.cpu().pin_memory(), vn.cpu().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = q_h.numel() * 2 + kn_h.numel() * 2 + vn_h.numel() * 2
    d2h = out.numel() * 4
    stage_in = [(torch.empty_like(q), torch.empty_like(kn), torch.empty_like(vn)) for _ in range(2)]
    stage_out = [torch.empty_like(out) for _ in range(2)]
    cstream = torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]   # host -> stage b landed
    in_free = [torch.cuda.Event() for _ in range(2)]    # stage b copied into the step's inputs
    out_ready = [torch.cuda.Event() for _ in range(2)]  # step output copied into stage b
    out_free = [torch.cuda.Event() for _ in range(2)]   # stage b read back to the host

    def copy_in(b):
        cstream.wait_event(in_free[b])
        with torch.cuda.stream(cstream):
            for dst, src in zip(stage_in[b], (q_h, kn_h, vn_h)):
                dst.copy_(src, non_blocking=True)
            in_ready[b].record(cstream)

    def e2e_run(n, run_step):
        for b in range(2):
            in_free[b].record(stream)
            out_free[b].record(cstream)
        t0, t1 = ev_pair()
        t0.record(cstream)
        copy_in(0)
        for i in range(n):
            b = i % 2
            stream.wait_event(in_ready[b])
            with torch.cuda.stream(stream):
                for dst, src in zip((q, kn, vn), stage_in[b]):
                    dst.copy_(src)
                in_free[b].record(stream)
            if i + 1 < n:
                copy_in(1 - b)
            run_step()
            with torch.cuda.stream(stream):
                stream.wait_event(out_free[b])
                stage_out[b].copy_(out)
                out_ready[b].record(stream)
            cstream.wait_event(out_ready[b])
            with torch.cuda.stream(cstream):
                out_h[b].copy_(stage_out[b], non_blocking=True)
                out_free[b].record(cstream)
        stream.wait_stream(cstream)
        t1.record(stream)
        return t0, t1

    # (a) graph replay of the captured step (frozen view counters)
    def graph_step():
        with torch.cuda.stream(stream):
            graph.replay()

    e2e_run(args.warmup, graph_step)
    torch.cuda.synchronize()
    c0, c1 = e2e_run(args.steps, graph_step)
    torch.cuda.synchronize()
    t_e2e_graph = kdist.max_over_ranks(c0.elapsed_time(c1) / 1e3 / args.steps)
    del graph

    # (b) eager: every step calls kvq_append_decode_attn once per layer
    # through the C ABI, host planning included; the views grow by one token
    # per step (the host arrays are advanced by the library in place)
    lib = kvq.lib()
    arrs = [kvq._view_array(lv) for lv in layer_views]
    P = ctypes.c_void_p
    ptrs = [(P(kn[l].data_ptr()), P(vn[l].data_ptr()), P(q[l].data_ptr()), P(out[l].data_ptr()),
             P(ws_step[l].data_ptr()), ws_step[l].numel()) for l in range(L)]
    sp = P(stream.cuda_stream)
    fscale = ctypes.c_float(scale)

    def eager_step():
        for l in range(L):
            k_p, v_p, q_p, o_p, w_p, w_n = ptrs[l]
            st = lib.kvq_append_decode_attn(arrs[l], A, Hq, H, D, k_p, v_p, q_p, fscale, o_p, w_p, w_n, sp)
            if st != 0:
                raise kvq.KvqError(st, "kvq_append_decode_attn")

    e2e_run(args.warmup, eager_step)
    torch.cuda.synchronize()
    before = [arrs[l][i].n_packed for l in range(L) for i in range(A)]
    c0, c1 = e2e_run(args.steps, eager_step)
    torch.cuda.synchronize()
    t_e2e = kdist.max_over_ranks(c0.elapsed_time(c1) / 1e3 / args.steps)
    for l in range(L):  # keep the binding's views in step with the advanced arrays
        for i, v in enumerate(layer_views[l]):
            v.c.n_packed, v.c.n_window, v.c.window_head = arrs[l][i].n_packed, arrs[l][i].n_window, arrs[l][i].window_head
    grew = [arrs[l][i].n_packed for l in range(L) for i in range(A)]
    assert all(g - b == args.steps for g, b in zip(grew, before)), "eager steps did not advance the views"
    # bytes of the eager steps: the views grew by one packed token per step;
    # the mean over the timed steps is the mid-point's
    e2e_bytes = bytes_step + (args.steps - 1) / 2.0 * sum(
        2 * v.n_kv_heads * (v.head_dim // 8 * v.bits + v.head_dim // 64 * 8) for v in all_views)
    e2e_gbs = kdist.aggregate_throughput(e2e_bytes, world, t_e2e) / 1e9
    e2e_graph_gbs = kdist.aggregate_throughput(bytes_step, world, t_e2e_graph) / 1e9

    rec = {
        "workload": WORKLOADS[key], "value": value, "unit": "GB/s", "ms_per_step": t_step * 1e3,
        "bytes_per_step": bytes_step, "tokens_per_s_per_agent": 1.0 / t_step, "hbm_frac": value / world / peak,
        "config": {"agents_per_gpu": A, "layers": L, "n_q_heads": Hq, "n_kv_heads": H, "head_dim": D,
                   "packed_tokens": list(w.lengths), "window": w.window, "bits": bits_set,
                   "calls_per_step": "per layer: kvq_append_decode_attn (append grid + attention grid per width)",
                   "cuda_graph": True,
                   "l2": f"working set per step {bytes_step / 1e9:.2f} GB > 126 MB L2, no flush"},
        "roofline": {"bound": "hbm", "achieved": attn_gbs, "peak": peak, "unit": "GB/s",
                     "frac": attn_gbs / peak, "traffic": profiled_traffic(key),
                     "kernel": (f"decode_attn_kernel<{D // 64}, b>: one kvq_decode_attn per layer over its "
                                f"{A} views, widths {bits_set}"),
                     "bytes_per_launch": attn_layer_bytes, "launch_us": t_attn * 1e6,
                     "peak_kind": f"{peak_kind} (hbm_gbs), burst"},
        "all_views_one_call": {"gbs": all_gbs, "frac": all_gbs / peak, "ms": t_all * 1e3},
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": t_e2e * 1e3,
                "how": ("every step: q and the new K/V copied in from pinned host memory, one kvq_append_decode_attn "
                        "per layer through the C ABI (host planning included, the views grow by one token per "
                        "step), the output copied back; copies on a second stream, double-buffered")},
        "e2e_graph": {"value": e2e_graph_gbs, "unit": "GB/s", "ms_per_step": t_e2e_graph * 1e3,
                      "how": "the same copies around a replay of the captured step (view counters frozen)"},
        "gpu_launches_per_step": launches_step,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        rec["cpu_baseline"] = cpu_baseline(key, w, dev)
    del pool, ws_step, ws_attn, q, kn, vn, out, stage_in, stage_out
    torch.cuda.empty_cache()
    return rec


def codec_leg(args, local, peak):
    """Bulk handoff codec (quantize then dequantize), 4-bit."""
    import quantized_kv_cache_dequantize_b200 as kvq
    from quantized_kv_cache_dequantize_b200 import workloads as wl
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream()
    hw = wl.handoff_llama8b()
    H = hw.n_layers * hw.n_kv_heads
    gm = wl.generator(hw.seed)
    mask = torch.stack([wl.outlier_mask(gm, hw.n_kv_heads, hw.head_dim, hw.outlier_frac)
                        for _ in range(hw.n_layers)]).view(H, hw.head_dim)
    g = wl.generator(hw.seed, device=dev)
    kx, vx = wl.kv_pair(g, H, hw.n_tokens, hw.head_dim, mask, dev)
    rb = hw.head_dim // 8 * hw.bits
    kc = torch.empty((H, hw.n_tokens, rb), dtype=torch.uint8, device=dev)
    vc = torch.empty_like(kc)
    ks = torch.empty((H, hw.n_tokens, hw.head_dim // 64, 2), dtype=torch.float32, device=dev)
    vs = torch.empty_like(ks)
    ky, vy = torch.empty_like(kx), torch.empty_like(vx)
    n_el = 2 * H * hw.n_tokens * hw.head_dim
    codec_bytes = n_el * 2 + 2 * (kc.numel() + ks.numel() * 4)
    qt, dt = [], []
    torch.cuda.synchronize()  # the inputs come from the current stream; the timed stream starts after them
    with ClockSampler(local) as codec_clk, torch.cuda.stream(stream):
        for it in range(args.warmup + args.steps):
            if it == args.warmup:
                stream.synchronize()
                codec_clk.mark(True)
            a0, a1, a2 = torch.cuda.Event(True), torch.cuda.Event(True), torch.cuda.Event(True)
            a0.record(stream)
            kvq.quantize(kx, hw.bits, kc, ks, stream=stream)
            kvq.quantize(vx, hw.bits, vc, vs, stream=stream)
            a1.record(stream)
            kvq.dequantize(kc, ks, hw.n_tokens, hw.head_dim, hw.bits, out=ky, stream=stream)
            kvq.dequantize(vc, vs, hw.n_tokens, hw.head_dim, hw.bits, out=vy, stream=stream)
            a2.record(stream)
            if it >= args.warmup:
                qt.append((a0, a1))
                dt.append((a1, a2))
        stream.synchronize()
        codec_clk.mark(False)
    tq = float(np.mean([x.elapsed_time(y) for x, y in qt])) / 1e3
    td = float(np.mean([x.elapsed_time(y) for x, y in dt])) / 1e3
    rec = {"workload": "bulk cache handoff, Llama-3.1-8B shape: 32 layers x 8 kv heads x 32768 tokens x "
                       "128, K and V, 4-bit group-64, 1% K outlier channels x10",
           "bytes": codec_bytes,
           "quantize_gbs": codec_bytes / tq / 1e9, "quantize_ms": tq * 1e3,
           "quantize_frac": codec_bytes / tq / 1e9 / peak,
           "dequantize_gbs": codec_bytes / td / 1e9, "dequantize_ms": td * 1e3,
           "dequantize_frac": codec_bytes / td / 1e9 / peak,
           "clocks": codec_clk.summary()}
    del kx, vx, kc, vc, ks, vs, ky, vy
    torch.cuda.empty_cache()
    return rec


def run_ours(args, rank, world, local):
    peak, peak_kind = peaks()
    legs = [k for k in args.legs.split(",") if k]
    assert HEADLINE in legs, "the headline workload is always measured"
    recs = {k: decode_leg(k, args, rank, world, local, peak, peak_kind) for k in legs}
    codec = None if args.skip_codec else codec_leg(args, local, peak)
    if rank != 0:
        return
    h = recs[HEADLINE]
    line = {
        "metric": METRIC, "value": h["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": h["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict({"workload": h["workload"]}, **h["config"]),
        "tokens_per_s_per_agent": h["tokens_per_s_per_agent"],
        "hbm_frac": h["hbm_frac"],
        "roofline": h["roofline"],
        "all_views_one_call": h["all_views_one_call"],
        "e2e": h["e2e"],
        "e2e_graph": h["e2e_graph"],
        "cpu_baseline": h.get("cpu_baseline"),
        "gpu_launches": h["gpu_launches_per_step"] * args.steps,
        "clocks": h["clocks"],
        "workloads": {k: r for k, r in recs.items() if k != HEADLINE},
        "codec": codec,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--legs", default="gemma12b,llama8b,qwen32b")
    ap.add_argument("--skip-codec", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    from quantized_kv_cache_dequantize_b200 import dist as kdist
    rank, world, local = kdist.init_from_env()
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        kdist.shutdown()


if __name__ == "__main__":
    main()
