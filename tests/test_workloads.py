"""The seeded input recipe: every draw repeats bit for bit from its seed, and
the workloads have the sizes, length mixes and width counts they are
documented with (no arithmetic of the method is involved)."""
import math

import numpy as np
import torch

from quantized_kv_cache_dequantize_b200 import workloads as wl


def test_draws_repeat_from_their_seed():
    a = wl.normal_bf16(wl.generator(11), (3, 5, 64))
    b = wl.normal_bf16(wl.generator(11), (3, 5, 64))
    c = wl.normal_bf16(wl.generator(12), (3, 5, 64))
    assert a.dtype == torch.bfloat16 and torch.equal(a, b) and not torch.equal(a, c)
    m1 = wl.outlier_mask(wl.generator(4), 8, 128, 0.01)
    m2 = wl.outlier_mask(wl.generator(4), 8, 128, 0.01)
    assert torch.equal(m1, m2)


def test_outlier_masks():
    m = wl.outlier_mask(wl.generator(1), 8, 128, 0.01)
    assert int(m.sum()) == math.ceil(0.01 * 8 * 128)
    f = wl.outlier_mask(wl.generator(1), 2, 64, 0.0, first4=True)
    assert f[:, :4].all() and not f[:, 4:].any()
    # outlier channels of K are scaled by 10, V is not touched
    k, v = wl.kv_pair(wl.generator(2), 2, 300, 64, f)
    ks, vs = k.float().abs().mean(dim=1), v.float().abs().mean(dim=1)
    assert (ks[:, :4].mean() / ks[:, 4:].mean()) > 6 and abs(vs[:, :4].mean() / vs[:, 4:].mean() - 1) < 0.3


def test_workload_shapes():
    t = wl.tiny()
    assert (t.n_views, t.n_q_heads, t.n_kv_heads, t.head_dim, t.window, t.lengths, t.bits) == \
        (1, 4, 2, 64, 0, (256,), (4,))
    d = wl.decode_llama8b()
    assert (d.n_agents, d.n_layers, d.n_q_heads, d.n_kv_heads, d.head_dim, d.window) == (10, 32, 32, 8, 128, 128)
    assert set(d.lengths) == {4096} and set(d.bits) == {4}
    g = wl.varlen_gemma12b()
    assert (g.n_agents, g.n_layers, g.n_q_heads, g.n_kv_heads, g.head_dim, g.window) == (6, 48, 16, 8, 256, 256)
    assert set(g.lengths) <= {4096, 8192, 16384, 32768}
    q = wl.mixed_qwen32b()
    assert (q.n_agents, q.n_layers, q.n_q_heads, q.n_kv_heads, q.head_dim, q.window) == (8, 64, 64, 8, 128, 128)
    assert all(8192 <= n <= 16384 for n in q.lengths)
    counts = {b: q.bits.count(b) for b in (2, 3, 4, 8)}
    assert counts == {8: 32, 4: 96, 3: 128, 2: 256}
    assert np.mean(q.bits) == 3.0
    h = wl.handoff_llama8b()
    assert (h.n_layers, h.n_kv_heads, h.n_tokens, h.head_dim, h.bits, h.outlier_frac) == (32, 8, 32768, 128, 4, 0.01)
