"""Pins of the CPU oracle against facts fixed outside the oracle itself.

The pages print no worked numeric example, so every pin here is a closed form,
an invariant, a brute-force search, or a special case that reduces to a library
routine (torch's float->bf16 rounding, numpy/scipy softmax, torch SDPA in fp64).
Each targets a plausible mistake: wrong bit order, wrong rounding mode, 2^b in
place of 2^b-1, a dropped min term, a wrong GQA head map, a transposed operand.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_dequantize_b200 import workloads as wl

BITS = (2, 3, 4, 8)


def bf16_of(values):
    """float values -> bf16 bit patterns (torch RNE); values must be exact in bf16."""
    t = torch.tensor(np.asarray(values, np.float64), dtype=torch.float64).to(torch.bfloat16)
    back = t.to(torch.float64).numpy()
    assert np.array_equal(back, np.asarray(values, np.float64)), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits_u16):
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()


def packed_closed_form(codes, bits):
    """Little-endian, LSB-first bit packing as one big integer per group."""
    codes = list(int(c) for c in codes)
    out = bytearray()
    for g in range(len(codes) // 64):
        val = 0
        for j, c in enumerate(codes[64 * g: 64 * g + 64]):
            val |= c << (j * bits)
        out += val.to_bytes(8 * bits, "little")
    return np.frombuffer(bytes(out), np.uint8)


# ------------------------------------------------------------- packing ----

@pytest.mark.parametrize("bits", BITS)
def test_packing_closed_form_every_position_and_value(bits):
    qmax = (1 << bits) - 1
    rows = []
    expect_codes = []
    for j in range(64):
        for c in range(qmax + 1):
            codes = np.zeros(64, np.int64)
            # endpoints fix mn = 0 and mx = qmax (s = 1) without touching slot j
            codes[(j + 1) % 64] = 0
            codes[(j + 2) % 64] = qmax
            codes[j] = c
            rows.append(codes.astype(np.float64))
            expect_codes.append(codes)
    x = bf16_of(np.stack(rows))
    packed, sm = oracle.quantize(x, bits)
    assert np.all(sm[..., 0] == 1.0) and np.all(sm[..., 1] == 0.0)
    for r, codes in enumerate(expect_codes):
        assert np.array_equal(packed[r], packed_closed_form(codes, bits)), (bits, r)
    assert np.array_equal(oracle.unpack(packed, 64, bits), np.stack(expect_codes).astype(np.uint8))


def test_packing_b4_nibbles_and_b8_identity():
    rng = np.random.default_rng(0)
    for bits in (4, 8):
        qmax = (1 << bits) - 1
        codes = rng.integers(0, qmax + 1, size=(16, 128))
        codes[:, 0] = 0
        codes[:, 64] = 0
        codes[:, 1] = qmax
        codes[:, 65] = qmax
        packed, _ = oracle.quantize(bf16_of(codes.astype(np.float64)), bits)
        if bits == 8:
            assert np.array_equal(packed, codes.astype(np.uint8))
        else:
            lo, hi = codes[:, 0::2], codes[:, 1::2]
            assert np.array_equal(packed, (lo | (hi << 4)).astype(np.uint8))


# ------------------------------------------------------------ quantize ----

@pytest.mark.parametrize("bits", BITS)
@pytest.mark.parametrize("k", [0, 3, 4, 7])
def test_on_grid_round_trip_is_exact(bits, k):
    """x = mn + c * 2^-k with 0 and 2^b-1 present: codes, s, mn reproduced and
    dequantize returns x bit for bit."""
    rng = np.random.default_rng(100 * bits + k)
    qmax = (1 << bits) - 1
    s = 2.0 ** -k
    rows, want = [], []
    for mn in (0.0, -8.0, -2.0 ** -3, 1.5, -96.0):
        for _ in range(8):
            c = rng.integers(0, qmax + 1, size=128)
            for g0 in (0, 64):
                i0, i1 = rng.choice(64, size=2, replace=False)
                c[g0 + i0] = 0
                c[g0 + i1] = qmax
            vals = mn + c * s
            # keep only rows exact in bf16 (8 significant bits)
            t = torch.tensor(vals).to(torch.bfloat16).to(torch.float64).numpy()
            if np.array_equal(t, vals):
                rows.append(vals)
                want.append((c, mn))
    assert len(rows) >= 8
    x = bf16_of(np.stack(rows))
    packed, sm = oracle.quantize(x, bits)
    got = oracle.unpack(packed, 128, bits)
    for r, (c, mn) in enumerate(want):
        assert np.array_equal(got[r], c), (bits, k, r)
        assert np.all(sm[r, :, 0] == np.float32(s))
        assert np.all(sm[r, :, 1] == np.float32(mn))
    y = oracle.dequantize(packed, sm, 128, bits)
    assert np.array_equal(y, x)
    assert np.array_equal(oracle.affine(packed, sm, 128, bits), np.stack(rows))


def test_round_half_to_even():
    # b=2: mn=0, mx=3 -> s=1; x=0.5,1.5,2.5 are exact ties -> 0, 2, 2
    vals = np.zeros(64)
    vals[0], vals[1] = 0.0, 3.0
    vals[2:5] = [0.5, 1.5, 2.5]
    packed, sm = oracle.quantize(bf16_of(vals[None]), 2)
    c = oracle.unpack(packed, 64, 2)[0]
    assert sm[0, 0, 0] == 1.0
    assert list(c[2:5]) == [0, 2, 2]
    # b=4: ties k+0.5 for k=0..14 -> even neighbour
    vals = np.zeros(64)
    vals[0], vals[1] = 0.0, 15.0
    vals[2:17] = np.arange(15) + 0.5
    packed, _ = oracle.quantize(bf16_of(vals[None]), 4)
    c = oracle.unpack(packed, 64, 4)[0][2:17]
    want = [k if k % 2 == 0 else k + 1 for k in range(15)]
    assert list(c) == want


def test_constant_groups():
    for bits in BITS:
        for v in (0.0, -0.0, 1.0, -3.5, 1e-30):
            vals = np.full((1, 64), v)
            x = torch.tensor(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            packed, sm = oracle.quantize(x, bits)
            assert np.all(packed == 0)
            assert sm[0, 0, 0] == 0.0
            mn_bits = np.float32(sm[0, 0, 1]).view(np.uint32)
            if v == 0.0:
                assert mn_bits == 0  # -0 stored as +0
            y = oracle.dequantize(packed, sm, 64, bits)
            yv = bf16_to_f64(y)
            assert np.all(yv == (0.0 if v == 0.0 else bf16_to_f64(x)[0, 0]))


def random_groups(seed, n_rows, head_dim=128, outliers=True):
    g = wl.generator(seed)
    mask = wl.outlier_mask(g, n_rows, head_dim, 0.0, first4=outliers)
    t = wl.normal_bf16(g, (n_rows, 1, head_dim), scale_mask=mask)[:, 0, :]
    return wl.bf16_bits(t)


@pytest.mark.parametrize("bits", BITS)
def test_error_bound_endpoints_and_brute_force(bits):
    qmax = (1 << bits) - 1
    x = random_groups(7 + bits, 48)
    packed, sm = oracle.quantize(x, bits)
    codes = oracle.unpack(packed, 128, bits).astype(np.int64)
    xv = bf16_to_f64(x)
    for r in range(x.shape[0]):
        for g in range(2):
            seg = xv[r, 64 * g: 64 * g + 64]
            cs = codes[r, 64 * g: 64 * g + 64]
            s, mn = float(sm[r, g, 0]), float(sm[r, g, 1])
            mx = seg.max()
            assert mn == seg.min()
            # scale: within one fp32 ulp of (mx - mn) / (2^b - 1)
            exact_s = (mx - mn) / qmax
            assert abs(s - exact_s) <= np.spacing(np.float32(s)) * 1.0
            # endpoints
            assert cs[np.argmin(seg)] == 0 and cs[np.argmax(seg)] == qmax
            # error bound |x - (mn + s c)| <= s (1/2 + 2^(b-23))
            err = np.abs(seg - (mn + s * cs))
            assert np.all(err <= s * (0.5 + 2.0 ** (bits - 23)))
            # brute force: nearest grid point over all codes, ties to even,
            # measured in exact rational arithmetic; near-ties accept either
            # neighbour, since the two fp32 roundings before the integer step
            # move the quotient by up to 2^(b-23) (relative 2^-23 of <= 2^b)
            S, MN = Fraction(s), Fraction(mn)
            for i in range(64):
                X = Fraction(seg[i])
                dist = [abs(X - (MN + S * c)) for c in range(qmax + 1)]
                best = min(dist)
                cands = [c for c in range(qmax + 1) if dist[c] == best]
                nearest = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
                qstar = (X - MN) / S
                frac = qstar - int(qstar)
                if abs(frac - Fraction(1, 2)) < Fraction(1, 1 << (21 - bits)):
                    assert cs[i] in (int(qstar), int(qstar) + 1)
                else:
                    assert cs[i] == nearest, (bits, r, g, i)


# ---------------------------------------------------------- dequantize ----

def bf16_nearest_exact(v: Fraction):
    """Nearest bf16 value to an exact rational (ties to even), as float."""
    if v == 0:
        return 0.0
    f = float(v)
    lo = torch.tensor([f], dtype=torch.float64).to(torch.bfloat16)
    cand = set()
    base = lo.view(torch.int16).item() & 0xFFFF
    for d in (-1, 0, 1):
        b = (base + d) & 0xFFFF
        val = torch.tensor([b], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).to(torch.float64).item()
        cand.add(val)
    best = min(cand, key=lambda c: (abs(Fraction(c) - v), 0))
    return best


@pytest.mark.parametrize("bits", BITS)
def test_dequantize_matches_library_rounding(bits):
    x = random_groups(40 + bits, 24)
    packed, sm = oracle.quantize(x, bits)
    y = oracle.dequantize(packed, sm, 128, bits)
    codes = oracle.unpack(packed, 128, bits).astype(np.float64)
    s = np.repeat(sm[..., 0].astype(np.float64), 64, axis=-1)
    mn = np.repeat(sm[..., 1].astype(np.float64), 64, axis=-1)
    # c*s + mn is exact in fp64 here (<= 32 significant bits, small exponent
    # spread), so rounding it to fp32 is the single rounding of fmaf
    f32 = (codes * s + mn).astype(np.float32)
    want = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(y, want)
    # and the result is a nearest bf16 of the exact affine value (a near-tie
    # may go either way through the fp32 step)
    yv = bf16_to_f64(y)
    exact = codes * s + mn
    ulp = np.spacing(np.abs(yv).astype(np.float32)).astype(np.float64) * 2 ** 16
    assert np.all(np.abs(yv - exact) <= 0.5 * ulp * (1 + 2 ** -10) + 1e-300)


def test_bf16_rounding_ties():
    # exact bf16 midpoints: 1 + 2^-8 (tie -> 1.0), 1 + 3*2^-8 (tie -> 1 + 2^-6)
    codes = np.zeros((1, 8), np.uint8)  # b=8, 64 codes; only first used
    for val, want in ((1.0 + 2 ** -8, 1.0), (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6),
                      (-(1.0 + 2 ** -8), -1.0)):
        codes = np.zeros((1, 64), np.uint8)
        sm = np.array([[[0.0, val]]], np.float32)
        y = oracle.dequantize(codes, sm, 64, 8)
        assert bf16_to_f64(y)[0, 0] == want


# ----------------------------------------------------------- attention ----

def make_view(seed, Hq=4, Hkv=2, D=64, n_p=40, n_w=7, bits=4):
    g = wl.generator(seed)
    mask = wl.outlier_mask(g, Hkv, D, 0.0, first4=True)
    k, v = wl.kv_pair(g, Hkv, n_p + n_w, D, mask)
    q = wl.normal_bf16(g, (Hq, D))
    kb, vb, qb = wl.bf16_bits(k), wl.bf16_bits(v), wl.bf16_bits(q)
    kc, ks = oracle.quantize(kb[:, :n_p], bits)
    vc, vs = oracle.quantize(vb[:, :n_p], bits)
    return dict(q=qb, bits=bits, k_codes=kc, k_sm=ks, v_codes=vc, v_sm=vs,
                k_win=kb[:, n_p:], v_win=vb[:, n_p:], D=D, Hq=Hq, Hkv=Hkv)


def dense_kv(view):
    D, bits = view["D"], view["bits"]
    kp = oracle.affine(view["k_codes"], view["k_sm"], D, bits)
    vp = oracle.affine(view["v_codes"], view["v_sm"], D, bits)
    k = np.concatenate([kp, bf16_to_f64(view["k_win"])], axis=1)
    v = np.concatenate([vp, bf16_to_f64(view["v_win"])], axis=1)
    return k, v


def run(view, scale, probs=False):
    return oracle.decode_attn(view["q"], view["bits"], view["k_codes"], view["k_sm"],
                              view["v_codes"], view["v_sm"], view["k_win"], view["v_win"],
                              scale, want_probs=probs)


def test_attention_matches_numpy_scipy_brute_force():
    from scipy.special import softmax
    view = make_view(11)
    scale = 1 / 8
    out = run(view, scale)
    k, v = dense_kv(view)
    q = bf16_to_f64(view["q"])
    G = view["Hq"] // view["Hkv"]
    for h in range(view["Hq"]):
        logits = scale * (k[h // G] @ q[h])
        p = softmax(logits)
        np.testing.assert_allclose(out[h], p @ v[h // G], rtol=1e-12, atol=1e-12)


def test_attention_matches_torch_sdpa_fp64():
    import torch.nn.functional as F
    view = make_view(12, Hq=8, Hkv=2, D=128, n_p=33, n_w=5)
    scale = 0.3
    out = run(view, scale)
    k, v = dense_kv(view)
    q = torch.from_numpy(bf16_to_f64(view["q"]))[None, :, None, :]
    kk = torch.from_numpy(k)[None]
    vv = torch.from_numpy(v)[None]
    ref = F.scaled_dot_product_attention(q, kk, vv, scale=scale, enable_gqa=True)[0, :, 0, :]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_window_only_view_is_textbook_bf16_attention():
    import torch.nn.functional as F
    g = wl.generator(13)
    Hq, Hkv, D, n = 6, 3, 64, 19
    k, v = wl.kv_pair(g, Hkv, n, D, None)
    q = wl.normal_bf16(g, (Hq, D))
    out = oracle.decode_attn(wl.bf16_bits(q), 4, None, None, None, None,
                             wl.bf16_bits(k), wl.bf16_bits(v), 1 / 8)
    ref = F.scaled_dot_product_attention(q.double()[None, :, None], k.double()[None], v.double()[None],
                                         scale=1 / 8, enable_gqa=True)[0, :, 0]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_softmax_rows_sum_to_one_and_match_probs():
    view = make_view(14)
    out, p = run(view, 1 / 8, probs=True)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p >= 0)
    _, v = dense_kv(view)
    G = view["Hq"] // view["Hkv"]
    for h in range(view["Hq"]):
        np.testing.assert_allclose(out[h], p[h] @ v[h // G], rtol=1e-12, atol=1e-12)


def test_identical_keys_give_mean_of_values():
    g = wl.generator(15)
    Hq, Hkv, D, n = 4, 2, 64, 23
    k1, v = wl.kv_pair(g, Hkv, n, D, None)
    k = k1[:, :1, :].expand(Hkv, n, D).contiguous()
    q = wl.normal_bf16(g, (Hq, D))
    out = oracle.decode_attn(wl.bf16_bits(q), 4, None, None, None, None,
                             wl.bf16_bits(k), wl.bf16_bits(v), 0.2)
    mean = v.double().mean(dim=1).numpy()
    for h in range(Hq):
        np.testing.assert_allclose(out[h], mean[h // 2], rtol=1e-12, atol=1e-12)


def test_dominant_logit_selects_its_value_row():
    g = wl.generator(16)
    Hq, Hkv, D, n = 2, 1, 64, 30
    k = torch.zeros(Hkv, n, D)
    k[0, 17, 0] = 40.0  # q = e_0 -> logit 40 for token 17, 0 elsewhere
    q = torch.zeros(Hq, D)
    q[:, 0] = 1.0
    _, v = wl.kv_pair(g, Hkv, n, D, None)
    out = oracle.decode_attn(wl.bf16_bits(q.bfloat16()), 4, None, None, None, None,
                             wl.bf16_bits(k.bfloat16()), wl.bf16_bits(v), 1.0)
    np.testing.assert_allclose(out[0], v[0, 17].double().numpy(), atol=1e-15 * 0 + 1e-15 + np.exp(-40) * 30 * 5)


def test_token_permutation_invariance():
    view = make_view(17, n_p=50, n_w=9)
    base = run(view, 1 / 8)
    rng = np.random.default_rng(0)
    pp = rng.permutation(50)
    pw = rng.permutation(9)
    perm = dict(view)
    for key in ("k_codes", "k_sm", "v_codes", "v_sm"):
        perm[key] = view[key][:, pp]
    for key in ("k_win", "v_win"):
        perm[key] = view[key][:, pw]
    np.testing.assert_allclose(run(perm, 1 / 8), base, rtol=1e-12, atol=1e-13)


def test_gqa_identical_queries_in_group_give_identical_outputs():
    view = make_view(18, Hq=8, Hkv=2)
    q = view["q"].copy()
    q[1:4] = q[0]
    q[5:8] = q[4]
    view["q"] = q
    out = run(view, 1 / 8)
    for h in range(1, 4):
        assert np.array_equal(out[h], out[0])
    for h in range(5, 8):
        assert np.array_equal(out[h], out[4])
    assert not np.allclose(out[0], out[4])


def test_key_and_value_roles_are_not_swapped():
    # keys all equal, values distinct: output is the mean of V, not of K
    view = make_view(19)
    view["k_codes"] = np.repeat(view["k_codes"][:, :1], 40, axis=1)
    view["k_sm"] = np.repeat(view["k_sm"][:, :1], 40, axis=1)
    view["k_win"] = np.repeat(view["k_win"][:, :1], 7, axis=1)
    # make the window key identical to the packed key's exact value as well
    kp = oracle.affine(view["k_codes"][:, :1], view["k_sm"][:, :1], 64, 4)
    out = run(view, 1 / 8)
    _, v = dense_kv(view)
    k, _ = dense_kv(view)
    q = bf16_to_f64(view["q"])
    from scipy.special import softmax
    for h in range(4):
        p = softmax((1 / 8) * (k[h // 2] @ q[h]))
        np.testing.assert_allclose(out[h], p @ v[h // 2], rtol=1e-12, atol=1e-12)
    assert kp.shape[1] == 1


# ------------------------------------------- sequences of several views ---

def seg_of(view, rows=None, window=True, bits=None):
    """A segment dict holding the packed rows `rows` (a slice) of a view and,
    optionally, its window."""
    rows = slice(0, view["k_codes"].shape[1]) if rows is None else rows
    seg = dict(bits=view["bits"] if bits is None else bits)
    for key in ("k_codes", "k_sm", "v_codes", "v_sm"):
        seg[key] = view[key][:, rows]
    if window:
        seg["k_win"], seg["v_win"] = view["k_win"], view["v_win"]
    return seg


def test_one_segment_is_the_view_attention():
    view = make_view(21, n_p=45, n_w=6)
    got = oracle.decode_attn_segments(view["q"], [seg_of(view)], 1 / 8)
    np.testing.assert_allclose(got, run(view, 1 / 8), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("cut", [1, 17, 44])
def test_view_split_into_segments_changes_nothing(cut):
    # the packed rows cut in two segments (the window with the second): the
    # union of tokens is the view's, so is the attention
    view = make_view(22, n_p=45, n_w=6)
    segs = [seg_of(view, slice(0, cut), window=False), seg_of(view, slice(cut, 45))]
    got = oracle.decode_attn_segments(view["q"], segs, 1 / 8)
    np.testing.assert_allclose(got, run(view, 1 / 8), rtol=1e-12, atol=1e-13)
    # and the window as a segment of its own, listed first
    only_win = dict(bits=4, k_win=view["k_win"], v_win=view["v_win"])
    segs = [only_win, seg_of(view, slice(0, cut), window=False), seg_of(view, slice(cut, 45), window=False)]
    np.testing.assert_allclose(oracle.decode_attn_segments(view["q"], segs, 1 / 8), run(view, 1 / 8),
                               rtol=1e-12, atol=1e-13)


def test_segments_of_different_widths_match_brute_force_and_order():
    # three widths and a bf16-only segment; textbook softmax over all rows
    from scipy.special import softmax
    views = [make_view(30 + b, n_p=20 + 3 * b, n_w=0 if b != 8 else 5, bits=b) for b in (2, 3, 8)]
    q = views[0]["q"]
    segs = [seg_of(v, window=v["k_win"].shape[1] > 0) for v in views]
    got = oracle.decode_attn_segments(q, segs, 0.15)
    ks, vs = zip(*[dense_kv(v) for v in views])
    k, v = np.concatenate(ks, axis=1), np.concatenate(vs, axis=1)
    qd = bf16_to_f64(q)
    for h in range(4):
        p = softmax(0.15 * (k[h // 2] @ qd[h]))
        np.testing.assert_allclose(got[h], p @ v[h // 2], rtol=1e-12, atol=1e-13)
    rev = oracle.decode_attn_segments(q, segs[::-1], 0.15)
    np.testing.assert_allclose(rev, got, rtol=1e-12, atol=1e-13)
    # a dropped segment changes the result
    assert not np.allclose(oracle.decode_attn_segments(q, segs[:2], 0.15), got, atol=1e-6)


def test_identical_keys_over_segments_give_mean_of_all_values():
    # every key zero (code 0, s = mn = 0) in every segment: all logits equal,
    # so the output is the plain mean of all segments' values
    views = [make_view(40 + b, n_p=11 + b, n_w=3, bits=b) for b in (2, 4)]
    segs = []
    for v in views:
        seg = seg_of(v)
        seg["k_codes"] = np.zeros_like(seg["k_codes"])
        seg["k_sm"] = np.zeros_like(seg["k_sm"])
        seg["k_win"] = np.zeros_like(seg["k_win"])
        segs.append(seg)
    got = oracle.decode_attn_segments(views[0]["q"], segs, 0.3)
    vals = np.concatenate([dense_kv(v)[1] for v in views], axis=1)
    for h in range(4):
        np.testing.assert_allclose(got[h], vals[h // 2].mean(axis=0), rtol=1e-12, atol=1e-13)


# ------------------------------------------------- top-K sparse decode ---

def run_sparse(view, scale, top_k):
    return oracle.sparse_decode_attn(view["q"], view["bits"], view["k_codes"], view["k_sm"], view["v_codes"],
                                     view["v_sm"], view["k_win"], view["v_win"], scale, top_k)


@pytest.mark.parametrize("top_k", [45, 46, 1000])
def test_sparse_with_every_token_selected_is_dense(top_k):
    view = make_view(50, n_p=45, n_w=6)
    out, sel = run_sparse(view, 1 / 8, top_k)
    np.testing.assert_allclose(out, run(view, 1 / 8), rtol=1e-12, atol=1e-13)
    assert all(np.array_equal(s, np.arange(45)) for s in sel)


@pytest.mark.parametrize("bits,top_k", [(2, 1), (4, 5), (4, 20), (8, 33), (3, 44)])
def test_sparse_error_within_discarded_mass_bound(bits, top_k):
    # RECAS (Metodologia B): with ||v|| <= V_max for every token and delta the
    # full attention's mass on the tokens left out, ||o - o'|| <= 2 V_max delta
    view = make_view(51 + bits, Hq=8, Hkv=2, n_p=45, n_w=6, bits=bits)
    dense, probs = run(view, 0.3, probs=True)
    sparse, sel = run_sparse(view, 0.3, top_k)
    _, v = dense_kv(view)
    G = 4
    for h in range(8):
        hk = h // G
        left_out = np.setdiff1d(np.arange(45), sel[hk])
        delta = probs[h][left_out].sum()
        vmax = np.sqrt((v[hk] ** 2).sum(axis=1)).max()
        err = np.sqrt(((dense[h] - sparse[h]) ** 2).sum())
        assert err <= 2 * vmax * delta * (1 + 1e-9) + 1e-12
        assert len(sel[hk]) == top_k


def test_sparse_selects_a_planted_key_and_attends_it_with_the_window():
    # one packed key far more aligned with q than all others: with K = 1 it is
    # the selection, and the output is attention over it and the window only
    view = make_view(60, Hq=2, Hkv=1, n_p=30, n_w=4, bits=8)
    q = np.zeros((2, 64), np.uint16)
    q[:, 0] = 0x3F80                                   # q = e_0 (bf16 1.0)
    view["q"] = q
    codes = view["k_codes"].copy()
    sm = view["k_sm"].copy()
    sm[0, 17, 0] = (1.0, 0.0)                          # token 17: k_0 = code (s = 1, mn = 0)
    codes[0, 17, 0] = 255
    view["k_codes"], view["k_sm"] = codes, sm
    out, sel = run_sparse(view, 1.0, 1)
    assert list(sel[0]) == [17]
    k, v = dense_kv(view)
    rows = [17] + list(range(30, 34))
    logits = k[0][rows] @ bf16_to_f64(q[0])
    p = np.exp(logits - logits.max())
    p /= p.sum()
    np.testing.assert_allclose(out[0], p @ v[0][rows], rtol=1e-12, atol=1e-13)


def test_sparse_score_takes_the_group_maximum_and_ties_go_low():
    # two query heads share the KV head; a token liked by either is selected;
    # among equal scores the lower index wins
    view = make_view(61, Hq=2, Hkv=1, n_p=10, n_w=0, bits=8)
    q = np.zeros((2, 64), np.uint16)
    q[0, 0] = 0x3F80
    q[1, 1] = 0x3F80
    view["q"] = q
    codes = np.zeros_like(view["k_codes"])
    sm = np.zeros_like(view["k_sm"])
    sm[0, :, 0, 0] = 1.0                               # s = 1, mn = 0: k = codes
    codes[0, 3, 0] = 200                               # head 0 likes token 3
    codes[0, 7, 1] = 150                               # head 1 likes token 7
    codes[0, 5, 1] = 100                               # and token 5 less
    codes[0, 8, 0] = 100                               # token 8 ties with token 5
    view["k_codes"], view["k_sm"] = codes, sm
    assert list(run_sparse(view, 1.0, 2)[1][0]) == [3, 7]
    assert list(run_sparse(view, 1.0, 3)[1][0]) == [3, 5, 7]
    assert list(run_sparse(view, 1.0, 4)[1][0]) == [3, 5, 7, 8]
    assert list(run_sparse(view, 1.0, 5)[1][0]) == [0, 3, 5, 7, 8]


# ------------------------------------------------ width allocation ---

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_sensitivity_bounds_the_error_of_quantizing_recent_tokens(bits):
    # quantize a view's recent K and V at `bits` (oracle quantizer) and attend
    # with the same q: the output moves by no more than the bound the
    # sensitivity is built from, V_max (e^(2 Delta/(2^b-1)) - 1) + E_v/(2^b-1)
    for seed in range(3):
        g = wl.generator(80 + seed)
        Hq, Hkv, D, n = 8, 2, 128, 48
        mask = wl.outlier_mask(g, Hkv, D, 0.02)
        k, v = wl.kv_pair(g, Hkv, n, D, mask)
        q = wl.bf16_bits(wl.normal_bf16(g, (Hq, D)))
        kb, vb = wl.bf16_bits(k), wl.bf16_bits(v)
        scale = 1 / np.sqrt(D)
        S, deltas, evs, vmaxs = oracle.width_sensitivity(q, kb, vb, scale)
        exact = oracle.decode_attn(q, bits, None, None, None, None, kb, vb, scale)
        kc, ks = oracle.quantize(kb, bits)
        vc, vs = oracle.quantize(vb, bits)
        quant = oracle.decode_attn(q, bits, kc, ks, vc, vs, None, None, scale)
        m = 2 ** bits - 1
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            err = np.sqrt(((exact[h] - quant[h]) ** 2).sum())
            bound = vmaxs[hk] * np.expm1(2 * deltas[hk] / m) + evs[hk] / m
            assert err <= bound * (1 + 1e-6) + 1e-9, (bits, seed, h, err, bound)
            assert err > 0
        assert S == max(2 * vm * d + e for vm, d, e in zip(vmaxs, deltas, evs))


def test_sensitivity_closed_form():
    # one KV head, one query head, head_dim 64, two recent tokens worked by
    # hand: K ranges 2 (token 1's last channel is 2, the rest 0), q all ones
    # (|q|_1 = 64), scale 1/8: Delta = 1/8 * 64 * 2/2 = 8.  V: token 1 is
    # 3 e_0, so R_v = 3, V_max = 3, E_v = sqrt(64 * 1.5^2) = 12.
    # S = 2 * 3 * 8 + 12 = 60.
    bf = lambda x: (np.asarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    k = np.zeros((1, 2, 64), np.float32)
    k[0, 1, 63] = 2.0
    v = np.zeros((1, 2, 64), np.float32)
    v[0, 1, 0] = 3.0
    q = np.ones((1, 64), np.float32)
    S, deltas, evs, vmaxs = oracle.width_sensitivity(bf(q), bf(k), bf(v), 0.125)
    assert (S, deltas[0], evs[0], vmaxs[0]) == (60.0, 8.0, 12.0, 3.0)
    # two query heads on the KV head: Delta takes the larger one; a second
    # group (head_dim 128) adds its own range terms
    k2 = np.zeros((1, 2, 128), np.float32)
    k2[0, 1, 63] = 2.0
    k2[0, 0, 100] = -1.0                      # group 1 range 1
    v2 = np.zeros((1, 2, 128), np.float32)
    v2[0, 1, 0] = 3.0
    v2[0, 0, 127] = 4.0                       # group 1 range 4; ||v_0|| = 4
    q2 = np.zeros((2, 128), np.float32)
    q2[0, :64] = 1.0                          # head 0: |q[0]|_1 = 64, |q[1]|_1 = 0
    q2[1, 64:] = 2.0                          # head 1: |q[1]|_1 = 128
    S, deltas, evs, vmaxs = oracle.width_sensitivity(bf(q2), bf(k2), bf(v2), 0.125)
    # Delta = 1/8 * max(64 * 2/2, 128 * 1/2) = 8; E_v = sqrt(64 * (1.5^2 + 2^2)) = 20
    assert (deltas[0], evs[0], vmaxs[0]) == (8.0, 20.0, 4.0)
    assert S == 2 * 4.0 * 8.0 + 20.0


def test_sensitivity_of_a_constant_window_is_zero():
    # every group constant: ranges 0, nothing to lose at any width
    k = np.full((2, 5, 64), 0x3F80, np.uint16)
    v = np.full((2, 5, 64), 0xC000, np.uint16)
    q = wl.bf16_bits(wl.normal_bf16(wl.generator(5), (4, 64)))
    assert oracle.width_sensitivity(q, k, v, 0.125)[0] == 0.0
    assert oracle.width_sensitivity(q, k[:, :0], v[:, :0], 0.125)[0] == 0.0


def brute_force_allocation(sens, cap, H, D, budget, units):
    import itertools
    unit = -(-budget // units)
    best = None
    for combo in itertools.product(oracle.WIDTHS, repeat=len(sens)):
        used = sum(-(-(c * 2 * H * (D * b // 8 + D // 64 * 8)) // unit) for c, b in zip(cap, combo))
        if used > budget // unit:
            continue
        err = sum(s / (2 ** b - 1) for s, b in zip(sens, combo))
        if best is None or err < best[1] - 1e-12:
            best = (list(combo), err)
    return best


@pytest.mark.parametrize("seed", range(6))
def test_allocation_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 6))
    sens = rng.exponential(1.0, n)
    cap = rng.integers(100, 5000, n)
    H, D = 2, 128
    lo = sum(c * 2 * H * (D * 2 // 8 + D // 64 * 8) for c in cap)
    hi = sum(c * 2 * H * (D * 8 // 8 + D // 64 * 8) for c in cap)
    for budget in (int(lo * 1.02), int((lo + hi) / 2), int(hi * 0.9), hi + 1000):
        got = oracle.allocate_widths(sens, cap, H, D, budget, units=256)
        want = brute_force_allocation(sens, cap, H, D, budget, 256)
        assert got is not None and want is not None
        assert abs(got[1] - want[1]) <= 1e-12 * max(1.0, want[1]), (seed, budget, got, want)


def test_allocation_extremes():
    sens, cap, H, D = [3.0, 1.0, 0.5], [1000, 2000, 500], 8, 128
    per = lambda b: 2 * H * (D * b // 8 + D // 64 * 8)
    everything = sum(c * per(8) for c in cap)
    assert oracle.allocate_widths(sens, cap, H, D, everything * 2)[0] == [8, 8, 8]
    floor = sum(c * per(2) for c in cap)
    assert oracle.allocate_widths(sens, cap, H, D, floor - 1) is None
    # more budget never gives a larger total error
    errs = [oracle.allocate_widths(sens, cap, H, D, int(floor * f))[1] for f in (1.05, 1.5, 2.0, 3.0, 4.0)]
    assert all(a >= b for a, b in zip(errs, errs[1:]))
    # the most sensitive view is never given fewer bits than a less sensitive
    # one of the same size
    bits, _ = oracle.allocate_widths([5.0, 1.0], [1000, 1000], H, D, int(1000 * (per(8) + per(2)) * 1.01))
    assert bits[0] >= bits[1]


# --------------------------------------------------------- window model ---

@pytest.mark.parametrize("W", [0, 1, 4, 7])
def test_window_model_invariant(W):
    rng = np.random.default_rng(W)
    m = oracle.WindowModel(W)
    n = 0
    for _ in range(40):
        m.append(n)
        n += 1
        split = max(0, n - W)
        assert m.packed == list(range(split))
        assert (m.window_logical() if W else []) == list(range(split, n))
    assert rng is not None
