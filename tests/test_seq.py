"""kvq_decode_attn_seq on the GPU against the fp64 oracle: sequences held by
several views (segments) of different widths, as after a change of a layer's
width (old blocks keep theirs) or with per-token widths {2, 4, 8, bf16}.
Tolerance as for kvq_decode_attn: 2e-3 max-abs and 1e-3 relative L2 per
(sequence, head)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from helpers import ViewSpec, assert_close, build_case

pytestmark = pytest.mark.gpu


def segment(case, i):
    """The oracle's segment for view i of a case: its packed tokens quantized
    by the oracle, its window tokens oldest first."""
    s, h = case.specs[i], case.host[i]
    seg = dict(bits=s.bits)
    if s.n_packed:
        seg["k_codes"], seg["k_sm"] = oracle.quantize(h["k"][:, :s.n_packed], s.bits)
        seg["v_codes"], seg["v_sm"] = oracle.quantize(h["v"][:, :s.n_packed], s.bits)
    if s.n_window:
        seg["k_win"], seg["v_win"] = h["k"][:, s.n_packed:], h["v"][:, s.n_packed:]
    return seg


def seq_queries(n_seqs, Hq, D, seed):
    q = wl.normal_bf16(wl.generator(seed), (n_seqs, Hq, D))
    return q.cuda(), wl.bf16_bits(q)


def run_seq(views, seq_begin, q, scale, workspace=None):
    out = kvq.decode_attn_seq(views, seq_begin, q, scale, workspace=workspace)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def check(case, seq_begin, scale, seed=5, what="seq"):
    Hq, D = case.n_q_heads, case.head_dim
    q, qb = seq_queries(len(seq_begin) - 1, Hq, D, seed)
    out = run_seq(case.views, seq_begin, q, scale)
    for s in range(len(seq_begin) - 1):
        segs = [segment(case, i) for i in range(seq_begin[s], seq_begin[s + 1])]
        ref = oracle.decode_attn_segments(qb[s], segs, scale)
        assert_close(out[s], ref, f"{what} sequence {s}")
    return out, q


def test_mixed_width_sequences_match_oracle(cuda_device):
    specs = [ViewSpec(300, 0, 0, 4, seed=1), ViewSpec(100, 16, 16, 2, head=5, seed=2),     # A
             ViewSpec(50, 0, 0, 8, seed=3), ViewSpec(70, 0, 0, 3, seed=4),                 # B
             ViewSpec(0, 20, 24, 4, head=3, seed=5),                                        # B: bf16 tokens only
             ViewSpec(1000, 64, 64, 4, head=10, seed=6),                                   # C
             ViewSpec(0, 0, 0, 2, seed=7), ViewSpec(33, 0, 0, 3, seed=8)]                  # D: an empty view
    case = build_case(8, 2, 128, specs)
    check(case, [0, 2, 5, 6, 8], 1 / np.sqrt(128))


@pytest.mark.parametrize("D,hq,hkv", [(64, 4, 2), (256, 16, 8)])
def test_sequences_other_shapes(cuda_device, D, hq, hkv):
    specs = [ViewSpec(129, 7, 8, 8, head=4, seed=10), ViewSpec(31, 0, 0, 2, seed=11),
             ViewSpec(64, 0, 0, 3, seed=12), ViewSpec(2, 1, 1, 4, seed=13)]
    case = build_case(hq, hkv, D, specs)
    check(case, [0, 2, 4], 1 / np.sqrt(D))


def test_one_view_per_sequence_is_decode_attn_bitwise(cuda_device):
    specs = [ViewSpec(400 + 9 * i, 8, 8, (2, 3, 4, 8)[i % 4], head=i % 8, seed=20 + i) for i in range(6)]
    case = build_case(8, 2, 128, specs)
    a = kvq.decode_attn_seq(case.views, list(range(7)), case.q, 0.1)
    b = kvq.decode_attn(case.views, case.q, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_sequences_spanning_launches_and_determinism(cuda_device):
    # 40 sequences of three widths: each width group is a launch of its own,
    # so every sequence's chunks come from three concurrent grids
    specs = []
    for s in range(40):
        for j, b in enumerate((2, 4, 8)):
            specs.append(ViewSpec(40 + 13 * ((s + j) % 7), 8 if b == 8 else 0, 8 if b == 8 else 0, b,
                                  head=s % 8, seed=100 + 3 * s + j))
    case = build_case(4, 2, 64, specs)
    sb = list(range(0, 121, 3))
    q, qb = seq_queries(40, 4, 64, 7)
    ws = kvq.new_seq_workspace(case.views, sb, 4, device=cuda_device)
    first = run_seq(case.views, sb, q, 0.125, ws)
    for s in (0, 1, 17, 39):
        segs = [segment(case, i) for i in range(3 * s, 3 * s + 3)]
        assert_close(first[s], oracle.decode_attn_segments(qb[s], segs, 0.125), f"sequence {s}")
    again = run_seq(case.views, sb, q, 0.125, ws)
    assert np.array_equal(first, again)
    assert int(ws[:4].view(torch.int32).item()) == 0


def test_long_sequence_chunk_cap(cuda_device, monkeypatch):
    # short chunks would give 3 x 125 = 375 chunks; the sequence's combine
    # takes at most 256, so the planner trims them: results stay in tolerance
    specs = [ViewSpec(4000, 0, 0, 4, seed=31), ViewSpec(4000, 0, 0, 2, seed=32), ViewSpec(3968, 32, 32, 8, seed=33)]
    case = build_case(8, 2, 64, specs)
    q, qb = seq_queries(1, 8, 64, 9)
    ref = oracle.decode_attn_segments(qb[0], [segment(case, i) for i in range(3)], 0.125)
    for chunk in ("32", "512"):
        monkeypatch.setenv("KVQ_CHUNK_TOKENS", chunk)
        out = run_seq(case.views, [0, 3], q, 0.125)
        assert_close(out[0], ref, f"chunk {chunk}")


def test_new_segment_continues_at_the_new_width(cuda_device):
    # a view at 4 bits with an 8-token window takes 20 decode tokens, then the
    # layer's width becomes 2: old blocks stay at 4 bits, the window moves to
    # the new segment, and 30 more tokens flush at 2 bits
    H, D, W = 2, 64, 8
    g = wl.generator(61)
    k0, v0 = wl.kv_pair(g, H, 40, D, None)
    view = kvq.View(H, D, 4, 64, W, device=cuda_device)
    view.fill_packed(k0.cuda(), v0.cuda())
    tk = [wl.bf16_bits(k0[:, t]) for t in range(40)]
    tv = [wl.bf16_bits(v0[:, t]) for t in range(40)]
    model = oracle.WindowModel(W, packed_tokens=range(40))
    width_of = {t: 4 for t in range(40)}
    cur, bits = view, 4

    def step(n, seed):
        gs = wl.generator(seed)
        for _ in range(n):
            kn = wl.normal_bf16(gs, (1, H, D))
            vn = wl.normal_bf16(gs, (1, H, D))
            kvq.append([cur], kn.cuda(), vn.cuda())
            tok = len(tk)
            tk.append(wl.bf16_bits(kn[0]))
            tv.append(wl.bf16_bits(vn[0]))
            flushed = model.append(tok)
            if flushed is not None:
                width_of[flushed] = bits

    step(20, 62)
    seg = view.new_segment(2, 64)
    assert view.cap_window == 0 and view.n_window == 0 and seg.n_window == W
    cur, bits = seg, 2
    step(30, 63)
    torch.cuda.synchronize()
    assert view.n_packed == 52 and seg.n_packed == 30 and seg.n_window == W

    def packed(b):
        toks = [t for t in model.packed if width_of[t] == b]
        kx = np.stack([tk[t] for t in toks], axis=1)
        vx = np.stack([tv[t] for t in toks], axis=1)
        kc, ks = oracle.quantize(kx, b)
        vc, vs = oracle.quantize(vx, b)
        return dict(bits=b, k_codes=kc, k_sm=ks, v_codes=vc, v_sm=vs)

    win = model.window_logical()
    segs = [packed(4), packed(2),
            dict(bits=2, k_win=np.stack([tk[t] for t in win], axis=1), v_win=np.stack([tv[t] for t in win], axis=1))]
    q, qb = seq_queries(1, 4, D, 64)
    out = run_seq([view, seg], [0, 2], q, 0.125)
    assert_close(out[0], oracle.decode_attn_segments(qb[0], segs, 0.125), "new segment")


def test_per_token_widths(cuda_device):
    # one sequence whose tokens carry widths {2, 4, 8, bf16} by importance:
    # one view per width holds its tokens (bf16 ones as a window-only view)
    H, D, T = 2, 128, 500
    g = wl.generator(71)
    k, v = wl.kv_pair(g, H, T, D, wl.outlier_mask(g, H, D, 0.02))
    widths = torch.tensor([2, 4, 8, 16])[torch.randint(0, 4, (T,), generator=g)]
    views, segs = [], []
    for b in (2, 4, 8, 16):
        idx = torch.nonzero(widths == b).flatten()
        kb, vb = k[:, idx], v[:, idx]
        if b == 16:
            view = kvq.View(H, D, 4, 2, len(idx), device=cuda_device)
            view.fill_window(kb.cuda(), vb.cuda())
            segs.append(dict(bits=4, k_win=wl.bf16_bits(kb), v_win=wl.bf16_bits(vb)))
        else:
            view = kvq.View(H, D, b, len(idx), 0, device=cuda_device)
            view.fill_packed(kb.cuda(), vb.cuda())
            kc, ks = oracle.quantize(wl.bf16_bits(kb), b)
            vc, vs = oracle.quantize(wl.bf16_bits(vb), b)
            segs.append(dict(bits=b, k_codes=kc, k_sm=ks, v_codes=vc, v_sm=vs))
        views.append(view)
    q, qb = seq_queries(1, 8, D, 72)
    out = run_seq(views, [0, 4], q, 1 / np.sqrt(D))
    assert_close(out[0], oracle.decode_attn_segments(qb[0], segs, 1 / np.sqrt(D)), "per-token widths")
