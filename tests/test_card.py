"""CacheCard on the GPU: a card packed from live views holds, bit for bit,
the oracle's codes and scale/min of exactly the tokens the window model says
were flushed and the window tokens oldest first; restored into fresh views
(other capacities, ring from slot 0, or through a file) the caches attend
exactly as the originals did and keep taking decode steps identically."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from test_append import setup_views

pytestmark = pytest.mark.gpu

H, D, HQ = 4, 128, 8
VIEW_CASES = [(4, 8, 300, 8, 3, 400), (2, 8, 0, 5, 5, 64), (3, 0, 77, 0, 0, 96), (8, 16, 33, 16, 15, 64),
           (4, 1, 1, 1, 0, 40)]


def advance(views, models, tk, tv, steps, seed):
    g = wl.generator(seed)
    for _ in range(steps):
        kn = wl.normal_bf16(g, (len(views), H, D))
        vn = wl.normal_bf16(g, (len(views), H, D))
        kvq.append(views, kn.cuda(), vn.cuda())
        for i, m in enumerate(models):
            tok = len(tk[i])
            tk[i].append(wl.bf16_bits(kn[i]))
            tv[i].append(wl.bf16_bits(vn[i]))
            m.append(tok)
    torch.cuda.synchronize()


def section(card, rec, k, H, D):
    """Bytes of section k of a view's data, from the documented layout."""
    n_p, n_w, b = rec["n_packed"], rec["n_window"], rec["bits"]
    codes = H * n_p * D * b // 8
    sm = H * n_p * (D // 64) * 8
    win = H * n_w * D * 2
    sizes = (codes, codes, sm, sm, win, win)
    off = rec["data_offset"]
    for j in range(k):
        off = (off + sizes[j] + 15) // 16 * 16
    return card[off:off + sizes[k]]


def test_card_matches_oracle_and_restores_exactly(cuda_device, tmp_path):
    views, models, tk, tv = setup_views(VIEW_CASES, H, D, cuda_device)
    advance(views, models, tk, tv, 11, seed=515)
    positions = [3, 0, 1000, 7, -1]
    card = kvq.card_pack(views, model_id=0x5151, position_offsets=positions)
    host = card.cpu()
    info = kvq.card_info(host)
    assert info["n_views"] == len(views) and info["n_kv_heads"] == H and info["head_dim"] == D
    assert info["model_id"] == 0x5151
    raw = host.numpy()
    import struct
    for i, (view, m, r) in enumerate(zip(views, models, info["views"])):
        assert (r["bits"], r["n_packed"], r["n_window"], r["position_offset"]) == \
            (view.bits, len(m.packed), m.n_window, positions[i])
        r = dict(r, data_offset=struct.unpack_from("<Q", raw, 64 + 64 * i + 24)[0])
        if m.packed:
            kx = np.stack([tk[i][t] for t in m.packed], axis=1)
            vx = np.stack([tv[i][t] for t in m.packed], axis=1)
            for k, x in ((0, kx), (1, vx)):
                want_c, want_s = oracle.quantize(x, view.bits)
                assert np.array_equal(section(raw, r, k, H, D), want_c.reshape(-1)), f"view {i} codes {k}"
                assert np.array_equal(section(raw, r, 2 + k, H, D).view(np.uint32), want_s.view(np.uint32).reshape(-1))
        if m.n_window:
            for k, tok in ((4, tk[i]), (5, tv[i])):
                want = np.stack([tok[t] for t in m.window_logical()], axis=1)   # [H][n_w][D] bf16 bits
                assert np.array_equal(section(raw, r, k, H, D).view(np.uint16), want.reshape(-1)), f"view {i} win"

    q = wl.normal_bf16(wl.generator(9), (len(views), HQ, D)).cuda()
    ref = kvq.decode_attn(views, q, 0.1)

    # restore into views with other capacities (ring from slot 0)
    fresh = kvq.views_for_card(host, cap_window=32, extra_packed=20)
    kvq.card_unpack(host, fresh)
    got = kvq.decode_attn(fresh, q, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)

    # through a file
    path = str(tmp_path / "agents.kvqcard")
    kvq.save_card(path, card)
    loaded = kvq.load_card(path)
    assert torch.equal(loaded, host)
    again = kvq.views_for_card(loaded, extra_packed=20)
    kvq.card_unpack(loaded, again)
    assert torch.equal(kvq.decode_attn(again, q, 0.1), ref)

    # restored caches with the originals' window sizes (every window is full
    # here) keep taking decode steps like the originals
    assert [v.cap_window for v in again] == [v.cap_window for v in views]
    g = wl.generator(77)
    for _ in range(6):
        kn = wl.normal_bf16(g, (len(views), H, D)).cuda()
        vn = wl.normal_bf16(g, (len(views), H, D)).cuda()
        a = kvq.append_decode_attn(views, kn, vn, q, 0.1)
        b = kvq.append_decode_attn(again, kn, vn, q, 0.1)
        torch.cuda.synchronize()
        # the same plan (counts and widths agree; only capacities and ring
        # slots differ) on the same kernels: bitwise the originals' outputs
        assert torch.equal(a, b)


def test_card_unpack_rejects_mismatched_views(cuda_device):
    views, _, _, _ = setup_views(VIEW_CASES[:2], H, D, cuda_device)
    host = kvq.card_pack(views).cpu()
    wrong = [kvq.View(H, D, 3, 400, 8, device=cuda_device), kvq.View(H, D, 2, 64, 8, device=cuda_device)]
    with pytest.raises(kvq.KvqError) as e:
        kvq.card_unpack(host, wrong)
    assert e.value.status == kvq.KVQ_ERR_INVALID_ARG
    small = [kvq.View(H, D, 4, 100, 8, device=cuda_device), kvq.View(H, D, 2, 64, 8, device=cuda_device)]
    with pytest.raises(kvq.KvqError) as e:
        kvq.card_unpack(host, small)
    assert e.value.status == kvq.KVQ_ERR_CAPACITY
    assert small[0].n_packed == 0


def test_card_of_many_views_spans_launches(cuda_device):
    configs = [((2, 3, 4, 8)[i % 4], 4, 20 + i, 4, i % 4, 64 + i) for i in range(130)]
    views, _, _, _ = setup_views(configs, 2, 64, cuda_device)
    host = kvq.card_pack(views, model_id=1).cpu()
    fresh = kvq.views_for_card(host)
    kvq.card_unpack(host, fresh)
    q = wl.normal_bf16(wl.generator(3), (len(views), 4, 64)).cuda()
    assert torch.equal(kvq.decode_attn(fresh, q, 0.125), kvq.decode_attn(views, q, 0.125))
