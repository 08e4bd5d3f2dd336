"""Small, fixed kernel cases for profilers (ncu) and quick timing.

    python -m quantized_kv_cache_dequantize_b200.profile_cases CASE [--reps N]

CASE:
  decode-layer   kvq_decode_attn over one layer of the batched decode
                 workload (10 agents, Llama-3.1-8B shape: 32 q / 8 kv heads,
                 head_dim 128, 4096 packed 4-bit tokens + 128-token window)
  decode-8layers the same over 8 layers (80 views) in one call
  quantize       kvq_quantize of 64 heads x 32768 tokens x 128 (bf16, 512 MiB)
  dequantize     kvq_dequantize of the same cache
  quantize-handoff / dequantize-handoff
                 the bulk handoff's K cache: 32 layers x 8 kv heads x 32768
                 tokens x 128 (2 GiB bf16), 1% outlier channels x10
  card-pack / card-unpack
                 kvq_card_pack of one agent's whole cache in Llama-3.1-8B
                 shape (32 layers x 8 kv heads, 32640 packed 4-bit tokens +
                 a full 128-token window), and kvq_card_unpack of that card
                 into fresh views
  decode-long    kvq_decode_attn over one layer of 10 agents with 32768
                 packed tokens each (+ 128-token window), Llama-3.1-8B shape
  sparse-layer / sparse-8layers / sparse-long
                 kvq_sparse_decode_attn over the views of decode-layer,
                 decode-8layers (top_k 512 of 4096 packed tokens per view and
                 KV head) and decode-long (top_k 2048 of 32768), + the window;
                 GB/s counts the bytes the path must read: all packed K codes
                 and scale/min (scoring), the selected rows' V codes and
                 scale/min, the window, q and out
  card-pack-decode
                 kvq_card_pack of every view of the batched decode workload
                 (10 agents x 32 layers, 4096 packed + 128 window)
  gemma-layer    kvq_decode_attn over one layer of the variable-length decode
                 workload in Gemma-3-12B shape (6 agents, 16 q / 8 kv heads,
                 head_dim 256, 4K-32K packed 4-bit tokens + 256-token window)
  qwen-layer     kvq_decode_attn over one layer of the mixed-precision decode
                 workload in Qwen3-32B shape (8 agents, 64 q / 8 kv heads,
                 head_dim 128, 8K-16K packed tokens at the layer's widths
                 {2, 3, 4, 8} + 128-token window)
Each case runs 3 warm-up calls, captures one call in a CUDA graph, replays
it once more and then --reps timed times, and prints the mean time per call
and the algorithmic GB/s.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import cache as kcache
from . import workloads as wl
from . import (card_info, card_pack, card_unpack, decode_attn, dequantize, new_workspace, quantize,
               sparse_decode_attn, sparse_workspace_size, views_for_card)


def _time(fn, reps):
    """Mean device time of one call: 3 eager warm-up calls, then the call
    captured in a CUDA graph and replayed `reps` times (host launch cost stays
    out of the timing).  The inputs were made on the current stream: it is
    drained first, so that the side stream never touches memory that work
    still queued there reads or writes (the allocator recycles blocks in
    the current stream's order only)."""
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        for _ in range(3):
            fn()
    st.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        fn()
    e0, e1 = torch.cuda.Event(True), torch.cuda.Event(True)
    with torch.cuda.stream(st):
        g.replay()
        e0.record(st)
        for _ in range(reps):
            g.replay()
        e1.record(st)
    st.synchronize()
    return e0.elapsed_time(e1) / reps / 1e3


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["decode-layer", "decode-8layers", "quantize", "dequantize", "quantize-handoff",
                                         "dequantize-handoff", "card-pack", "card-unpack", "card-pack-decode", "sparse-layer",
                                         "sparse-8layers", "decode-long", "sparse-long", "gemma-layer", "qwen-layer"])
    ap.add_argument("--reps", type=int, default=20)
    a = ap.parse_args(argv)
    dev = torch.device("cuda:0")
    if a.case.startswith("card"):
        w = (wl.decode_llama8b(n_agents=1, length=32768 - 128) if a.case != "card-pack-decode"
             else wl.decode_llama8b())
        pool = kcache.build_decode(w, dev)
        card = card_pack(pool.views)
        host = card.cpu()
        # bytes moved: every section read once and written once
        H, D = w.n_kv_heads, w.head_dim
        nbytes = 2 * sum(2 * H * (r["n_packed"] * (D * r["bits"] // 8 + D // 64 * 8) + r["n_window"] * D * 2)
                         for r in card_info(host)["views"])
        if a.case == "card-unpack":
            fresh = views_for_card(host, device=dev)
            t = _time(lambda: card_unpack(host, fresh, card=card, stream=torch.cuda.current_stream()), a.reps)
        else:
            t = _time(lambda: card_pack(pool.views, out=card, stream=torch.cuda.current_stream()), a.reps)
    elif a.case.startswith("sparse"):
        long = a.case == "sparse-long"
        w = wl.decode_llama8b(n_layers=8 if a.case == "sparse-8layers" else 1, length=32768 if long else 4096)
        top_k = 2048 if long else 512
        pool = kcache.build_decode(w, dev)
        q = kcache.decode_queries(w, device=dev)
        ws = torch.zeros(sparse_workspace_size(pool.views, w.n_q_heads, top_k), dtype=torch.uint8, device=dev)
        out = torch.empty((w.n_views, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
        t = _time(lambda: sparse_decode_attn(pool.views, q, w.softmax_scale, top_k, out=out, workspace=ws,
                                             stream=torch.cuda.current_stream()), a.reps)
        rb, ng = w.head_dim // 8 * 4, w.head_dim // 64
        n_p = w.view_len(0)
        nbytes = w.n_views * (w.n_kv_heads * (n_p * (rb + ng * 8) + top_k * (rb + ng * 8) + w.window * 4 * w.head_dim)
                              + w.n_q_heads * w.head_dim * 6)
    elif a.case in ("gemma-layer", "qwen-layer"):
        w = wl.varlen_gemma12b(n_layers=1) if a.case == "gemma-layer" else wl.mixed_qwen32b(n_layers=1)
        if a.case == "qwen-layer":
            # the first layer's widths of the 8 x 64 workload (its seeded allocation)
            full = wl.mixed_qwen32b()
            w = type(w)(**{**w.__dict__, "bits": tuple(full.view_bits(ag, 0) for ag in range(full.n_agents))})
        pool = kcache.build_decode(w, dev)
        q = kcache.decode_queries(w, device=dev)
        ws = new_workspace(pool.views, w.n_q_heads, device=dev)
        out = torch.empty((w.n_views, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
        t = _time(lambda: decode_attn(pool.views, q, w.softmax_scale, out=out, workspace=ws,
                                       stream=torch.cuda.current_stream()), a.reps)
        D = w.head_dim
        nbytes = sum(w.n_kv_heads * (w.view_len(ag) * (2 * D // 8 * w.view_bits(ag, 0) + 2 * (D // 64) * 8) +
                                     w.window * 4 * D) + w.n_q_heads * D * 6 for ag in range(w.n_agents))
    elif a.case.startswith("decode"):
        w = wl.decode_llama8b(n_layers=8 if a.case == "decode-8layers" else 1,
                              length=32768 if a.case == "decode-long" else 4096)
        pool = kcache.build_decode(w, dev)
        q = kcache.decode_queries(w, device=dev)
        ws = new_workspace(pool.views, w.n_q_heads, device=dev)
        out = torch.empty((w.n_views, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
        t = _time(lambda: decode_attn(pool.views, q, w.softmax_scale, out=out, workspace=ws,
                                       stream=torch.cuda.current_stream()), a.reps)
        rb = w.head_dim // 8 * 4
        nbytes = w.n_views * (w.n_kv_heads * (w.view_len(0) * (2 * rb + 2 * (w.head_dim // 64) * 8) +
                                              w.window * 4 * w.head_dim) + w.n_q_heads * w.head_dim * 6)
    else:
        if a.case.endswith("handoff"):
            hw = wl.handoff_llama8b()
            H, T, D = hw.n_layers * hw.n_kv_heads, hw.n_tokens, hw.head_dim
            gm = wl.generator(hw.seed)
            mask = torch.stack([wl.outlier_mask(gm, hw.n_kv_heads, D, hw.outlier_frac)
                                for _ in range(hw.n_layers)]).view(H, D)
            x = wl.normal_bf16(wl.generator(hw.seed, device=dev), (H, T, D), dev, mask)
        else:
            H, T, D = 64, 32768, 128
            x = wl.normal_bf16(wl.generator(2, device=dev), (H, T, D), dev)
        codes, sm = quantize(x, 4)
        y = torch.empty_like(x)
        nbytes = x.numel() * 2 + codes.numel() + sm.numel() * 4
        if a.case.startswith("quantize"):
            t = _time(lambda: quantize(x, 4, codes, sm, stream=torch.cuda.current_stream()), a.reps)
        else:
            t = _time(lambda: dequantize(codes, sm, T, D, 4, out=y, stream=torch.cuda.current_stream()), a.reps)
    print(f"{a.case}: {t * 1e6:.1f} us per call, {nbytes / t / 1e9:.0f} GB/s")


if __name__ == "__main__":
    main(sys.argv[1:])
