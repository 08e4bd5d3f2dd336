"""kvq_append on the GPU against the oracle's window bookkeeping model and its
quantizer: after every append the packed rows are bit-exact oracle codes of
exactly the tokens the model says were flushed, the ring holds the last W
tokens in the slots the model names, and attention over the result matches
the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from helpers import assert_close

pytestmark = pytest.mark.gpu


def setup_views(configs, H, D, device):
    """configs: list of (bits, W, n_prefill, n_window0, head0, cap_packed)."""
    views, models, tokens_k, tokens_v = [], [], [], []
    for i, (bits, W, n0, nw0, head0, cap) in enumerate(configs):
        g = wl.generator(1000 + i)
        k, v = wl.kv_pair(g, H, n0 + nw0, D, None)
        view = kvq.View(H, D, bits, cap, W, device=device)
        if n0:
            view.fill_packed(k[:, :n0].to(device), v[:, :n0].to(device))
        if W:
            view.fill_window(k[:, n0:].to(device), v[:, n0:].to(device), head=head0)
        views.append(view)
        models.append(oracle.WindowModel(W, range(n0), range(n0, n0 + nw0), head=head0))
        tokens_k.append([wl.bf16_bits(k[:, t]) for t in range(n0 + nw0)])
        tokens_v.append([wl.bf16_bits(v[:, t]) for t in range(n0 + nw0)])
    return views, models, tokens_k, tokens_v


def check_state(view, model, tk, tv, what):
    H, D, bits = view.n_kv_heads, view.head_dim, view.bits
    assert view.n_packed == len(model.packed), what
    assert view.n_window == model.n_window and (view.cap_window == 0 or view.window_head == model.head), what
    if model.packed:
        kx = np.stack([tk[t] for t in model.packed], axis=1)   # [H, n, D]
        vx = np.stack([tv[t] for t in model.packed], axis=1)
        for x, codes, sm in ((kx, view.k_codes, view.k_scalemin), (vx, view.v_codes, view.v_scalemin)):
            want_c, want_s = oracle.quantize(x, bits)
            n = len(model.packed)
            assert np.array_equal(codes[:, :n].cpu().numpy(), want_c), what
            assert np.array_equal(sm[:, :n].cpu().numpy().view(np.uint32), want_s.view(np.uint32)), what
    for slot, tok in enumerate(model.slots):
        if tok is None or slot >= view.cap_window:
            continue
        if tok in model.window_logical():
            assert np.array_equal(wl.bf16_bits(view.k_window[:, slot]), tk[tok]), what
            assert np.array_equal(wl.bf16_bits(view.v_window[:, slot]), tv[tok]), what


def test_append_sequence_matches_model(cuda_device):
    H, D = 4, 128
    configs = [(4, 8, 20, 3, 0, 64), (2, 8, 0, 8, 5, 64), (3, 0, 7, 0, 0, 64), (8, 1, 1, 1, 0, 64),
               (4, 16, 33, 16, 15, 64)]
    views, models, tk, tv = setup_views(configs, H, D, cuda_device)
    g = wl.generator(4242)
    for step in range(25):
        kn = wl.normal_bf16(g, (len(views), H, D))
        vn = wl.normal_bf16(g, (len(views), H, D))
        kvq.append(views, kn.to(cuda_device), vn.to(cuda_device))
        torch.cuda.synchronize()
        for i, m in enumerate(models):
            tok = len(tk[i])
            tk[i].append(wl.bf16_bits(kn[i]))
            tv[i].append(wl.bf16_bits(vn[i]))
            m.append(tok)
        if step % 6 == 5 or step == 24:
            for i in range(len(views)):
                check_state(views[i], models[i], tk[i], tv[i], f"step {step} view {i}")
    # attention over the appended caches equals the oracle over the model's placement
    q = wl.normal_bf16(wl.generator(7), (len(views), 8, D))
    out = kvq.decode_attn(views, q.to(cuda_device), 0.1).cpu().numpy().astype(np.float64)
    for i, (view, m) in enumerate(zip(views, models)):
        bits = view.bits
        kc = ks = vc = vs = kw = vw = None
        if m.packed:
            kc, ks = oracle.quantize(np.stack([tk[i][t] for t in m.packed], 1), bits)
            vc, vs = oracle.quantize(np.stack([tv[i][t] for t in m.packed], 1), bits)
        if m.n_window:
            kw = np.stack([tk[i][t] for t in m.window_logical()], 1)
            vw = np.stack([tv[i][t] for t in m.window_logical()], 1)
        ref = oracle.decode_attn(wl.bf16_bits(q[i]), bits, kc, ks, vc, vs, kw, vw, 0.1)
        assert_close(out[i], ref, f"attention after appends, view {i}")


def test_append_capacity_error_leaves_state(cuda_device):
    H, D = 2, 64
    view = kvq.View(H, D, 4, 2, 0, device=cuda_device)
    kn = torch.zeros((1, H, D), dtype=torch.bfloat16, device=cuda_device)
    kvq.append([view], kn, kn)
    kvq.append([view], kn, kn)
    assert view.n_packed == 2
    with pytest.raises(kvq.KvqError) as e:
        kvq.append([view], kn, kn)
    assert e.value.status == kvq.KVQ_ERR_CAPACITY
    assert view.n_packed == 2
