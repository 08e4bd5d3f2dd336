"""The three decode workloads at their full sizes, run as bench.py runs them:
one call per layer over that layer's views.  Every output is finite; sampled
views are checked against the fp64 oracle on copies of exactly the bf16 bytes
the GPU cache was built from (tolerance 2e-3 max-abs, 1e-3 relative L2 per
head).

- Llama-3.1-8B shape, 10 agents x 32 layers, 4096 packed 4-bit tokens + a
  128-token window: kvq_decode_attn per layer, then one kvq_append_decode_attn
  decode step per layer (the bench's step), checked against the oracle over
  the window model's placement after the append.
- Gemma-3-12B shape, 6 agents x 48 layers, head_dim 256, lengths from
  {4K, 8K, 16K, 32K}, 256-token window, K outlier channels.
- Qwen3-32B shape, 8 agents x 64 layers, 64 q / 8 kv heads, lengths in
  [8K, 16K], per-view widths {2, 3, 4, 8} with mean 3 bits.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import cache as kc, workloads as wl
from helpers import assert_close

pytestmark = pytest.mark.gpu


def layer_views(w, pool):
    L = w.n_layers
    return [[pool.views[a * L + l] for a in range(w.n_agents)] for l in range(L)]


def view_bytes(w, a, l):
    k, v, head = kc.view_inputs(w, a, l, "cuda")
    return wl.bf16_bits(k.cpu()), wl.bf16_bits(v.cpu()), head


def oracle_out(w, kb, vb, packed, window, q_bits, bits):
    """kb, vb: uint16 [H, n_tokens, D] of every token the view has seen."""
    kc_ = ks = vc = vs = kw = vw = None
    if packed:
        kc_, ks = oracle.quantize(np.ascontiguousarray(kb[:, packed]), bits)
        vc, vs = oracle.quantize(np.ascontiguousarray(vb[:, packed]), bits)
    if window:
        kw, vw = np.ascontiguousarray(kb[:, window]), np.ascontiguousarray(vb[:, window])
    return oracle.decode_attn(q_bits, bits, kc_, ks, vc, vs, kw, vw, w.softmax_scale)


def run_per_layer(w, pool, q):
    """kvq_decode_attn once per layer; returns fp32 [n_views, H_q, D] in view order."""
    L, A = w.n_layers, w.n_agents
    out = torch.empty((w.n_views, w.n_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
    for l, views in enumerate(layer_views(w, pool)):
        idx = [a * L + l for a in range(A)]
        o = kvq.decode_attn(views, q[idx].contiguous(), w.softmax_scale)
        out[idx] = o
    torch.cuda.synchronize()
    return out


def check_samples(w, out, q, samples):
    for a, l in samples:
        kb, vb, _ = view_bytes(w, a, l)
        n_p = w.view_len(a)
        i = a * w.n_layers + l
        ref = oracle_out(w, kb, vb, list(range(n_p)), list(range(n_p, n_p + w.window)),
                         wl.bf16_bits(q[i].cpu()), w.view_bits(a, l))
        assert_close(out[i].cpu().numpy().astype(np.float64), ref, f"{w.name} agent {a} layer {l}")


def test_llama8b_full_size(cuda_device):
    w = wl.decode_llama8b()
    pool = kc.build_decode(w, extra_packed=2)
    q = kc.decode_queries(w)
    out = run_per_layer(w, pool, q)
    assert bool(torch.isfinite(out).all())
    samples = [(0, 0), (9, 31), (4, 17)]
    check_samples(w, out, q, samples)

    # one decode step per layer, as the bench runs it
    kn, vn = kc.decode_new_tokens(w)
    L, A = w.n_layers, w.n_agents
    out2 = torch.empty_like(out)
    for l, views in enumerate(layer_views(w, pool)):
        idx = [a * L + l for a in range(A)]
        out2[idx] = kvq.append_decode_attn(views, kn[idx].contiguous(), vn[idx].contiguous(),
                                           q[idx].contiguous(), w.softmax_scale)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(out2).all())
    for a, l in samples:
        kb, vb, head = view_bytes(w, a, l)
        i = a * L + l
        n_p = w.view_len(a)
        kb = np.concatenate([kb, wl.bf16_bits(kn[i].cpu())[:, None]], axis=1)
        vb = np.concatenate([vb, wl.bf16_bits(vn[i].cpu())[:, None]], axis=1)
        m = oracle.WindowModel(w.window, range(n_p), range(n_p, n_p + w.window), head=head)
        m.append(n_p + w.window)
        assert pool.views[i].n_packed == len(m.packed) == n_p + 1
        ref = oracle_out(w, kb, vb, m.packed, m.window_logical(), wl.bf16_bits(q[i].cpu()), 4)
        assert_close(out2[i].cpu().numpy().astype(np.float64), ref, f"step, agent {a} layer {l}")


def test_gemma12b_full_size(cuda_device):
    w = wl.varlen_gemma12b()
    pool = kc.build_decode(w)
    q = kc.decode_queries(w)
    out = run_per_layer(w, pool, q)
    assert bool(torch.isfinite(out).all())
    # the longest and the shortest agent, first and last layer
    lens = [w.view_len(a) for a in range(w.n_agents)]
    lo, hi = int(np.argmin(lens)), int(np.argmax(lens))
    check_samples(w, out, q, [(hi, 0), (lo, w.n_layers - 1), (hi, 23)])


def test_qwen32b_mixed_bits_full_size(cuda_device):
    w = wl.mixed_qwen32b()
    pool = kc.build_decode(w)
    q = kc.decode_queries(w)
    out = run_per_layer(w, pool, q)
    assert bool(torch.isfinite(out).all())
    # one sampled view of each width
    samples, seen = [], set()
    for a in range(w.n_agents):
        for l in range(w.n_layers):
            b = w.view_bits(a, l)
            if b not in seen:
                seen.add(b)
                samples.append((a, l))
    assert seen == {2, 3, 4, 8}
    check_samples(w, out, q, samples)
