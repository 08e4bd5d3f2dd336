"""kvq_append_decode_attn (one decode step: append, then attend, in one call)
against kvq_append followed by kvq_decode_attn on an identical copy of the
views: every step's output and the final cache contents are bitwise equal, and
attention after the steps matches the fp64 oracle over the window model's
token placement."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from helpers import assert_close
from test_append import setup_views

pytestmark = pytest.mark.gpu

TENSORS = ("k_codes", "v_codes", "k_scalemin", "v_scalemin", "k_window", "v_window")


def run_steps(configs, H, Hq, D, n_steps, device, seed=4242, scale=0.1):
    a, _, _, _ = setup_views(configs, H, D, device)
    b, models, tk, tv = setup_views(configs, H, D, device)
    g = wl.generator(seed)
    for step in range(n_steps):
        kn = wl.normal_bf16(g, (len(a), H, D)).to(device)
        vn = wl.normal_bf16(g, (len(a), H, D)).to(device)
        q = wl.normal_bf16(g, (len(a), Hq, D)).to(device)
        kvq.append(a, kn, vn)
        out_a = kvq.decode_attn(a, q, scale)
        out_b = kvq.append_decode_attn(b, kn, vn, q, scale)
        torch.cuda.synchronize()
        assert torch.equal(out_a, out_b), f"step {step}"
        for i, m in enumerate(models):
            tok = len(tk[i])
            tk[i].append(wl.bf16_bits(kn[i].cpu()))
            tv[i].append(wl.bf16_bits(vn[i].cpu()))
            m.append(tok)
        for va, vb in zip(a, b):
            assert (va.n_packed, va.n_window, va.window_head) == (vb.n_packed, vb.n_window, vb.window_head)
    for i, (va, vb) in enumerate(zip(a, b)):
        for name in TENSORS:
            assert torch.equal(getattr(va, name), getattr(vb, name)), f"view {i} {name}"
    return b, models, tk, tv, q, out_b


def test_fused_step_equals_append_then_attend(cuda_device):
    """Full rings that flush, rings filling up, no ring, a 1-slot ring, and a
    long packed part cut into several chunks (the flushed row lands in the
    last one); then the oracle over the model's placement."""
    H, Hq, D = 4, 16, 128
    configs = [(4, 8, 3000, 8, 3, 3100), (2, 8, 0, 5, 5, 64), (3, 0, 7, 0, 0, 64), (8, 1, 1, 1, 0, 64),
               (4, 16, 33, 16, 15, 64), (4, 64, 1000, 64, 0, 1100)]
    views, models, tk, tv, q, out = run_steps(configs, H, Hq, D, 20, cuda_device)
    out = out.cpu().numpy().astype(np.float64)
    for i, (view, m) in enumerate(zip(views, models)):
        bits = view.bits
        kc = ks = vc = vs = kw = vw = None
        if m.packed:
            kc, ks = oracle.quantize(np.stack([tk[i][t] for t in m.packed], 1), bits)
            vc, vs = oracle.quantize(np.stack([tv[i][t] for t in m.packed], 1), bits)
        if m.n_window:
            kw = np.stack([tk[i][t] for t in m.window_logical()], 1)
            vw = np.stack([tv[i][t] for t in m.window_logical()], 1)
        ref = oracle.decode_attn(wl.bf16_bits(q[i].cpu()), bits, kc, ks, vc, vs, kw, vw, 0.1)
        assert_close(out[i], ref, f"attention after fused steps, view {i}")


def test_fused_step_head_dim_256_gqa8(cuda_device):
    configs = [(4, 32, 700, 32, 7, 800), (2, 32, 64, 20, 0, 128), (8, 0, 300, 0, 0, 400)]
    run_steps(configs, 2, 16, 256, 6, cuda_device, seed=11, scale=1 / 16)


def test_fused_step_many_views(cuda_device):
    """More views than one append launch (128) and one attention launch (96) hold."""
    configs = [((2, 3, 4, 8)[i % 4], 4, 40 + i, 4, i % 4, 64 + i) for i in range(200)]
    run_steps(configs, 2, 4, 64, 3, cuda_device, seed=12)


def test_fused_step_capacity_error_leaves_state(cuda_device):
    H, D = 2, 64
    view = kvq.View(H, D, 4, 2, 0, device=cuda_device)
    kn = torch.zeros((1, H, D), dtype=torch.bfloat16, device=cuda_device)
    q = torch.zeros((1, 4, D), dtype=torch.bfloat16, device=cuda_device)
    kvq.append_decode_attn([view], kn, kn, q, 0.1)
    kvq.append_decode_attn([view], kn, kn, q, 0.1)
    assert view.n_packed == 2
    with pytest.raises(kvq.KvqError) as e:
        kvq.append_decode_attn([view], kn, kn, q, 0.1)
    assert e.value.status == kvq.KVQ_ERR_CAPACITY
    assert view.n_packed == 2
