"""kvq_sparse_decode_attn on the GPU against the fp64 oracle (RECAS top-K
sparse decode over the packed cache; the bf16 window always active).

The selection is an integer decision taken on floating-point scores: the GPU
scores in fp32, the oracle in fp64.  Each case uses a top_k at which the
oracle's K-th and (K+1)-th scores of every (view, KV head) are at least 1e-4
apart, ten times the fp32 score error at these sizes, so the selected set is unique; the
test then requires the same indices and the outputs within 2e-3 max-abs /
1e-3 relative L2."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl
from helpers import ViewSpec, assert_close, build_case, oracle_view

pytestmark = pytest.mark.gpu

GAP = 1e-4


def oracle_parts(case, i):
    s, h = case.specs[i], case.host[i]
    kc = ks = vc = vs = kw = vw = None
    if s.n_packed:
        kc, ks = oracle.quantize(h["k"][:, :s.n_packed], s.bits)
        vc, vs = oracle.quantize(h["v"][:, :s.n_packed], s.bits)
    if s.n_window:
        kw, vw = h["k"][:, s.n_packed:], h["v"][:, s.n_packed:]
    return kc, ks, vc, vs, kw, vw


def oracle_scores(case, i, scale):
    """fp64 scores of view i's packed tokens per KV head (only to pick a top_k
    with a clear gap; the expected values come from oracle.sparse_decode_attn)."""
    s = case.specs[i]
    kc, ks, _, _, _, _ = oracle_parts(case, i)
    k = oracle.affine(kc, ks, case.head_dim, s.bits)
    q = (case.q_bits[i].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    G = case.n_q_heads // case.n_kv_heads
    return [np.max(np.stack([scale * (k[hk] @ q[h]) for h in range(hk * G, (hk + 1) * G)]), axis=0)
            for hk in range(case.n_kv_heads)]


def oracle_over_selection(case, i, scale, sel_i):
    """fp64 oracle attention of view i over a given selection: per KV head,
    the packed rows sel_i[hk] (entries >= 0) plus the whole window, the
    quantities of the oracle's own quantization.  Validates a selection that
    differs from the oracle's at a near tie."""
    s = case.specs[i]
    kc, ks, vc, vs, kw, vw = oracle_parts(case, i)
    G = case.n_q_heads // case.n_kv_heads
    out = np.zeros((case.n_q_heads, case.head_dim))
    for hk in range(case.n_kv_heads):
        rows = sel_i[hk][sel_i[hk] >= 0]
        pick = (lambda a: None if a is None or len(rows) == 0 else np.ascontiguousarray(a[hk:hk + 1][:, rows]))
        win = (lambda a: None if a is None else np.ascontiguousarray(a[hk:hk + 1]))
        out[hk * G:(hk + 1) * G] = oracle.decode_attn(case.q_bits[i][hk * G:(hk + 1) * G], s.bits, pick(kc),
                                                      pick(ks), pick(vc), pick(vs), win(kw), win(vw), scale)
    return out


def pick_top_k(case, scale, candidates):
    scores = [sc for i, s in enumerate(case.specs) if s.n_packed for sc in oracle_scores(case, i, scale)]
    for k in candidates:
        ok = True
        for sc in scores:
            if k < len(sc):
                srt = np.sort(sc)[::-1]
                ok &= srt[k - 1] - srt[k] >= GAP
        if ok:
            return k
    raise AssertionError("no top_k with a clear score gap among the candidates")


def run_sparse(case, scale, top_k, workspace=None):
    n, Hkv = len(case.specs), case.n_kv_heads
    sel = torch.full((n, Hkv, top_k), -7, dtype=torch.int32, device=case.q.device)
    out, _ = kvq.sparse_decode_attn(case.views, case.q, scale, top_k, selected=sel, workspace=workspace)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), sel.cpu().numpy()


def check(case, scale, top_k, what):
    out, sel = run_sparse(case, scale, top_k)
    for i, s in enumerate(case.specs):
        kc, ks, vc, vs, kw, vw = oracle_parts(case, i)
        ref, ref_sel = oracle.sparse_decode_attn(case.q_bits[i], s.bits, kc, ks, vc, vs, kw, vw, scale, top_k)
        for hk in range(case.n_kv_heads):
            want = np.full(top_k, -1)
            want[:len(ref_sel[hk])] = ref_sel[hk]
            assert np.array_equal(sel[i, hk], want), f"{what}: view {i} head {hk} selection"
        assert_close(out[i], ref, f"{what}: view {i} {s}")
    return out, sel


def test_sparse_llama_shape_small(cuda_device):
    specs = [ViewSpec(700 + 37 * i, 32, 32, 4, head=i, seed=200 + i) for i in range(4)]
    case = build_case(32, 8, 128, specs)
    scale = 1 / np.sqrt(128)
    k = pick_top_k(case, scale, range(64, 300))
    check(case, scale, k, "llama")


# groups of up to 8 query heads score on the attention grid's tensor-core QK
# path, wider ones (32 / 2) on the SIMT score kernel; the gathered rows are
# copied in 16-byte pieces, or 8-byte ones where a row is not a 16-byte
# multiple (3-bit codes at head_dim 64 and 192, scale/min rows of head_dim 64
# and 192)
@pytest.mark.parametrize("bits,D,hq,hkv", [(2, 64, 2, 2), (3, 128, 8, 2), (8, 256, 16, 8), (4, 64, 64, 8),
                                           (4, 128, 32, 2), (3, 64, 4, 2), (3, 192, 6, 2), (4, 192, 8, 4)])
def test_sparse_widths_shapes_groups(cuda_device, bits, D, hq, hkv):
    specs = [ViewSpec(300, 8, 8, bits, head=3, seed=300 + bits), ViewSpec(129, 0, 0, bits, seed=301 + bits),
             ViewSpec(0, 5, 8, bits, head=6, seed=302 + bits)]
    case = build_case(hq, hkv, D, specs)
    scale = 1 / np.sqrt(D)
    k = pick_top_k(case, scale, list(range(17, 128)) + [1, 2, 3])
    check(case, scale, k, f"b{bits} D{D} {hq}/{hkv}")


def test_sparse_k1_and_k_at_least_n(cuda_device):
    specs = [ViewSpec(200, 16, 16, 4, head=2, seed=410), ViewSpec(64, 0, 0, 8, seed=411)]
    case = build_case(8, 2, 128, specs)
    scale = 1 / np.sqrt(128)
    check(case, scale, pick_top_k(case, scale, [1, 2, 3, 4]), "small k")
    # every packed token selected: the dense result
    for k in (200, 256):
        out, sel = run_sparse(case, scale, k)
        for i in range(2):
            assert_close(out[i], oracle_view(case, i, scale), f"k {k} view {i}")
        assert np.array_equal(sel[1, 0], np.r_[np.arange(64), np.full(k - 64, -1)])


def test_sparse_error_bound_on_gpu_outputs(cuda_device):
    # RECAS, Metodologia B: ||o - o'|| <= 2 V_max delta, with delta the full
    # attention mass on the packed tokens left out (fp64 oracle quantities)
    specs = [ViewSpec(500, 16, 16, 4, head=1, seed=500), ViewSpec(333, 0, 0, 2, seed=501)]
    case = build_case(8, 2, 64, specs)
    scale = 0.2
    k = pick_top_k(case, scale, range(40, 200))
    sparse, sel = run_sparse(case, scale, k)
    dense = kvq.decode_attn(case.views, case.q, scale).cpu().numpy().astype(np.float64)
    for i, s in enumerate(specs):
        kc, ks, vc, vs, kw, vw = oracle_parts(case, i)
        _, probs = oracle.decode_attn(case.q_bits[i], s.bits, kc, ks, vc, vs, kw, vw, scale, want_probs=True)
        v = oracle.affine(vc, vs, 64, s.bits)
        if s.n_window:
            v = np.concatenate([v, (vw.astype(np.uint32) << 16).view(np.float32).astype(np.float64)], axis=1)
        for h in range(8):
            hk = h // 4
            left = np.setdiff1d(np.arange(s.n_packed), sel[i, hk][sel[i, hk] >= 0])
            delta = probs[h][left].sum()
            vmax = np.sqrt((v[hk] ** 2).sum(axis=1)).max()
            err = np.sqrt(((dense[i, h] - sparse[i, h]) ** 2).sum())
            assert err <= 2 * vmax * delta + 4e-3, (i, h, err, 2 * vmax * delta)


def test_sparse_many_views_and_workspace_reuse_while_growing(cuda_device):
    # more views than one launch holds; then decode steps append to every view
    # and the same workspace serves the next calls
    specs = [ViewSpec(150 + 11 * (i % 9), 4, 4, (2, 3, 4, 8)[i % 4], head=i % 4, seed=600 + i) for i in range(110)]
    case = build_case(4, 2, 64, specs, extra_packed=4)
    scale = 0.125
    top_k = 40
    ws = torch.zeros(kvq.sparse_workspace_size(case.views, 4, top_k) + (1 << 20), dtype=torch.uint8,
                     device=cuda_device)
    for step in range(3):
        out, sel = run_sparse(case, scale, top_k, workspace=ws)
        assert np.all(np.isfinite(out))
        for i in (0, 1, 95, 96, 109):
            s = case.specs[i]
            kc, ks, vc, vs, kw, vw = oracle_parts(case, i)
            ref, ref_sel = oracle.sparse_decode_attn(case.q_bits[i], s.bits, kc, ks, vc, vs, kw, vw, scale, top_k)
            # the selection can differ from the oracle's only at a near tie
            sc = oracle_scores(case, i, scale)
            for hk in range(2):
                srt = np.sort(sc[hk])[::-1]
                if srt[top_k - 1] - srt[top_k] >= GAP:
                    assert np.array_equal(sel[i, hk], ref_sel[hk]), (step, i, hk)
                    continue
                # near tie: K distinct packed tokens in ascending order, every
                # one scoring within GAP of the K-th best (a valid top-K set)
                picks = sel[i, hk]
                assert len(picks) == top_k and np.all(np.diff(picks) > 0), (step, i, hk)
                assert 0 <= picks[0] and picks[-1] < s.n_packed, (step, i, hk)
                assert np.all(sc[hk][picks] >= srt[top_k - 1] - GAP), (step, i, hk)
            if all(np.array_equal(sel[i, hk], ref_sel[hk]) for hk in range(2)):
                assert_close(out[i], ref, f"step {step} view {i}")
            else:
                # the output is the oracle's attention over the GPU's own selection
                assert_close(out[i], oracle_over_selection(case, i, scale, sel[i]),
                             f"step {step} view {i}, near-tie selection")
        # one decode token for every view: the window flushes into the packed part
        g = wl.generator(700 + step)
        kn = wl.normal_bf16(g, (110, 2, 64))
        vn = wl.normal_bf16(g, (110, 2, 64))
        kvq.append(case.views, kn.cuda(), vn.cuda())
        for i, s in enumerate(case.specs):
            h = case.host[i]
            h["k"] = np.concatenate([h["k"], wl.bf16_bits(kn[i])[:, None]], axis=1)
            h["v"] = np.concatenate([h["v"], wl.bf16_bits(vn[i])[:, None]], axis=1)
            s.n_packed += 1  # the window was full: its oldest token moved to the packed part
        torch.cuda.synchronize()


def test_sparse_long_views_both_select_paths(cuda_device):
    # 32768 packed tokens (one select CTA, 32 keys a lane), 65536 (a cluster
    # of 2, 32 keys a lane), 70001 (a cluster of 4, 18 keys a lane), 140000
    # (beyond the shared-memory select: the radix select reading the scores
    # from memory) and 5000, top_k in the thousands
    specs = [ViewSpec(32768, 16, 16, 4, head=2, seed=810), ViewSpec(140000, 16, 16, 4, head=0, seed=811),
             ViewSpec(5000, 0, 0, 2, seed=812), ViewSpec(70001, 8, 8, 3, head=5, seed=813),
             ViewSpec(65536, 4, 4, 8, head=1, seed=814)]
    case = build_case(8, 2, 128, specs, q_seed=21)
    scale = 1 / np.sqrt(128)
    k = pick_top_k(case, scale, range(1500, 2400, 7))
    check(case, scale, k, "long views")


@pytest.mark.parametrize("cluster", ["1", "2", "4"])
def test_sparse_select_cluster_sizes(cuda_device, monkeypatch, cluster):
    # the same selections whatever the number of CTAs a (view, KV head) is
    # split over (a view whose keys would exceed 32 a lane takes more);
    # ragged slices: views shorter than one CTA's share, and lengths that are
    # no multiple of 32
    monkeypatch.setenv("KVQ_SELECT_CLUSTER", cluster)
    specs = [ViewSpec(3001, 16, 16, 4, head=1, seed=840), ViewSpec(9000, 0, 0, 3, seed=841),
             ViewSpec(20011, 8, 8, 4, head=5, seed=842), ViewSpec(700, 4, 4, 8, head=0, seed=843)]
    case = build_case(8, 2, 64, specs, q_seed=23)
    scale = 0.125
    k = pick_top_k(case, scale, range(400, 690, 3))
    check(case, scale, k, f"cluster {cluster}")


def dup_case(n_packed, n_window, bits, D, hq, hkv, block, copies, seed, stride=None):
    """One view whose first `block` packed tokens repeat `copies` times, at
    multiples of `stride` (default `block`; equal K and V rows, so equal
    scores on both sides)."""
    stride = stride or block
    g = wl.generator(seed)
    mask = wl.outlier_mask(g, hkv, D, 0.0)
    k, v = wl.kv_pair(g, hkv, n_packed + n_window, D, mask)
    for m in range(1, copies):
        k[:, m * stride:m * stride + block] = k[:, :block]
        v[:, m * stride:m * stride + block] = v[:, :block]
    view = kvq.View(hkv, D, bits, n_packed + 2, n_window, device="cuda")
    view.fill_packed(k[:, :n_packed].cuda(), v[:, :n_packed].cuda())
    view.fill_window(k[:, n_packed:].cuda(), v[:, n_packed:].cuda(), head=0)
    gq = wl.generator(seed + 1)
    q = wl.normal_bf16(gq, (1, hq, D))
    from helpers import Case
    return Case(hq, hkv, D, [ViewSpec(n_packed, n_window, n_window, bits, seed=seed)], [view], q.cuda(),
                [dict(k=wl.bf16_bits(k), v=wl.bf16_bits(v))], wl.bf16_bits(q))


def test_sparse_exact_ties_take_lowest_indices(cuda_device):
    # 8 copies of a 32-token block: the K-th score falls inside a group of 8
    # equal scores for at least one KV head, where the tie rule (lowest index
    # first) decides; the other heads have a clear gap at K.  20000 tokens:
    # the copies 2500 tokens apart, in different CTAs of the cluster
    for n, seed, stride in ((4096, 830, 32), (20000, 831, 2500)):
        case = dup_case(n, 16, 4, 128, 8, 2, 32, 8, seed, stride)
        scale = 1 / np.sqrt(128)
        sc = oracle_scores(case, 0, scale)
        chosen = None
        for k in range(64, n - 64):
            inside, ok = False, True
            for s in sc:
                srt = np.sort(s)[::-1]
                if srt[k - 1] - srt[k] >= GAP:
                    continue
                if srt[k - 1] != srt[k]:
                    ok = False
                    break
                # an exact tie group [lo, hi) around rank k, clear of its neighbours
                lo = k - 1
                while lo > 0 and srt[lo - 1] == srt[k]:
                    lo -= 1
                hi = k
                while hi < len(srt) and srt[hi] == srt[k]:
                    hi += 1
                ok &= (lo == 0 or srt[lo - 1] - srt[k] >= GAP) and (hi == len(srt) or srt[k] - srt[hi] >= GAP)
                inside = True
            if ok and inside:
                chosen = k
                break
        assert chosen is not None, "no top_k inside a tie group"
        check(case, scale, chosen, f"ties n {n}")
