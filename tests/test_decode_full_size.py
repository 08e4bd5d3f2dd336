"""The three decode workloads at their full sizes, run as bench.py runs them:
one call per layer over that layer's views.  Outputs are checked against the
fp64 oracle on copies of exactly the bf16 bytes the GPU cache was built from
(tolerance 2e-3 max-abs, 1e-3 relative L2 per head), the oracle running on
host threads.

- Llama-3.1-8B shape, 10 agents x 32 layers, 4096 packed 4-bit tokens + a
  128-token window: kvq_decode_attn per layer, then one kvq_append_decode_attn
  decode step per layer (the bench's step), each of the 320 views checked in
  both, the step against the oracle over the window model's placement after
  the append.
- Gemma-3-12B shape, 6 agents x 48 layers, head_dim 256, lengths from
  {4K, 8K, 16K, 32K}, 256-token window, K outlier channels: every agent at the
  first, a middle and the last layer (18 views, the longest and the shortest
  agent among them).
- Qwen3-32B shape, 8 agents x 64 layers, 64 q / 8 kv heads, lengths in
  [8K, 16K], per-view widths {2, 3, 4, 8} with mean 3 bits: every agent at the
  first and the last layer, plus the first view of each width (at least 16
  views, every width among them).
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import cache as kc, workloads as wl
from helpers import OracleRunner, close_msg

pytestmark = pytest.mark.gpu


def layer_views(w, pool):
    L = w.n_layers
    return [[pool.views[a * L + l] for a in range(w.n_agents)] for l in range(L)]


def view_bytes(w, a, l):
    k, v, head = kc.view_inputs(w, a, l, "cuda")
    return wl.bf16_bits(k), wl.bf16_bits(v), head


def oracle_out(w, kb, vb, packed, window, q_bits, bits):
    """kb, vb: uint16 [H, n_tokens, D] of every token the view has seen;
    packed, window: token indices (window oldest first)."""
    kc_ = ks = vc = vs = kw = vw = None
    if len(packed):
        kc_, ks = oracle.quantize(np.ascontiguousarray(kb[:, packed]), bits)
        vc, vs = oracle.quantize(np.ascontiguousarray(vb[:, packed]), bits)
    if len(window):
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


def check_views(w, out, q, samples):
    """Every (agent, layer) in samples against the oracle; returns the count."""
    run = OracleRunner()
    out_h, q_h = out.cpu().numpy().astype(np.float64), q.cpu()

    def job(a, l, kb, vb):
        n_p = w.view_len(a)
        i = a * w.n_layers + l
        ref = oracle_out(w, kb, vb, np.arange(n_p), np.arange(n_p, n_p + w.window), wl.bf16_bits(q_h[i]),
                         w.view_bits(a, l))
        return close_msg(out_h[i], ref, f"{w.name} agent {a} layer {l}")

    for a, l in samples:
        kb, vb, _ = view_bytes(w, a, l)
        run.submit(job, a, l, kb, vb)
    return run.finish()


def test_llama8b_full_size(cuda_device):
    w = wl.decode_llama8b()
    L, A = w.n_layers, w.n_agents
    pool = kc.build_decode(w, extra_packed=2)
    q = kc.decode_queries(w)
    out = run_per_layer(w, pool, q)

    # one decode step per layer, as the bench runs it
    kn, vn = kc.decode_new_tokens(w)
    out2 = torch.empty_like(out)
    for l, views in enumerate(layer_views(w, pool)):
        idx = [a * L + l for a in range(A)]
        out2[idx] = kvq.append_decode_attn(views, kn[idx].contiguous(), vn[idx].contiguous(),
                                           q[idx].contiguous(), w.softmax_scale)
    torch.cuda.synchronize()
    assert all(v.n_packed == w.view_len(0) + 1 for v in pool.views)

    # every view, before and after the step, against the oracle
    run = OracleRunner()
    o1, o2 = out.cpu().numpy().astype(np.float64), out2.cpu().numpy().astype(np.float64)
    q_h, kn_h, vn_h = q.cpu(), kn.cpu(), vn.cpu()

    def job(a, l, kb, vb, head):
        i = a * L + l
        n_p = w.view_len(a)
        qb = wl.bf16_bits(q_h[i])
        ref = oracle_out(w, kb, vb, np.arange(n_p), np.arange(n_p, n_p + w.window), qb, 4)
        msg = close_msg(o1[i], ref, f"decode, agent {a} layer {l}")
        if msg:
            return msg
        kb2 = np.concatenate([kb, wl.bf16_bits(kn_h[i])[:, None]], axis=1)
        vb2 = np.concatenate([vb, wl.bf16_bits(vn_h[i])[:, None]], axis=1)
        m = oracle.WindowModel(w.window, range(n_p), range(n_p, n_p + w.window), head=head)
        m.append(n_p + w.window)
        if len(m.packed) != n_p + 1:
            return f"window model: {len(m.packed)} packed tokens after the step"
        ref2 = oracle_out(w, kb2, vb2, np.asarray(m.packed), np.asarray(m.window_logical()), qb, 4)
        return close_msg(o2[i], ref2, f"step, agent {a} layer {l}")

    for a in range(A):
        for l in range(L):
            kb, vb, head = view_bytes(w, a, l)
            run.submit(job, a, l, kb, vb, head)
    assert run.finish() == w.n_views


def test_gemma12b_full_size(cuda_device):
    w = wl.varlen_gemma12b()
    pool = kc.build_decode(w)
    q = kc.decode_queries(w)
    out = run_per_layer(w, pool, q)
    assert bool(torch.isfinite(out).all())
    lens = [w.view_len(a) for a in range(w.n_agents)]
    assert min(lens) < max(lens)
    samples = [(a, l) for a in range(w.n_agents) for l in (0, 23, w.n_layers - 1)]
    assert check_views(w, out, q, samples) == 3 * w.n_agents


def test_qwen32b_mixed_bits_full_size(cuda_device):
    w = wl.mixed_qwen32b()
    pool = kc.build_decode(w)
    q = kc.decode_queries(w)
    out = run_per_layer(w, pool, q)
    assert bool(torch.isfinite(out).all())
    samples = [(a, l) for a in range(w.n_agents) for l in (0, w.n_layers - 1)]
    seen = {w.view_bits(a, l) for a, l in samples}
    for a in range(w.n_agents):
        for l in range(w.n_layers):
            b = w.view_bits(a, l)
            if b not in seen:
                seen.add(b)
                samples.append((a, l))
    assert seen == {2, 3, 4, 8}
    assert check_views(w, out, q, samples) == len(samples) >= 16
