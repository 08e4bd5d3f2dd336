"""CPU oracle for the quantized KV-cache codec and decode attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The product package
never imports this module, and this module never imports the product package;
the two share no code.

The arithmetic lives in ``kvq_oracle.c`` (plain C, built with gcc, no FMA
contraction, no fast-math).  This file only marshals numpy arrays and holds the
recent-window bookkeeping model used to check appends, which is pure list
logic with no arithmetic of the method.

Sources: "QKVShare: Quantized KV-Cache Handoff for Multi-Agent On-Device LLMs"
(Metodologia: quantized card, dequantize-then-inject); "Agent Memory Below the
Prompt: Persistent Q4 KV Cache ..." (Abstract: attention over several agents'
4-bit caches); "Coordinated Mixed-Precision KV Cache Quantization ..."
(Abstract: per-(agent, layer) widths, recent states kept native, only newly
quantized blocks get a width).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle_kvq.so")
GROUP = 64

_lib = None


def build(force: bool = False) -> str:
    """Compile kvq_oracle.c into oracle/_build/liboracle_kvq.so (gcc)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class use_library:
    """Context manager: route every oracle call through another build of
    kvq_oracle.c (the mutation tests plant mistakes in a copy)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        self.saved = _lib
        _lib = None
        _load(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved


def _load(path: str | None = None):
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(path or build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_quantize_rows.argtypes = [P, i64, i32, i32, P, P]
        lib.oracle_dequantize_rows.argtypes = [P, P, i64, i32, i32, P]
        lib.oracle_unpack_rows.argtypes = [P, i64, i32, i32, P]
        lib.oracle_affine_rows.argtypes = [P, P, i64, i32, i32, P]
        lib.oracle_decode_attn.argtypes = [i32, i32, i32, i32, i64, P, P, P, P,
                                           i64, P, P, P, f64, P, P]
        for f in (lib.oracle_quantize_rows, lib.oracle_dequantize_rows,
                  lib.oracle_unpack_rows, lib.oracle_affine_rows, lib.oracle_decode_attn):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def row_bytes(head_dim: int, bits: int) -> int:
    return head_dim // 8 * bits


def quantize(x_bf16_bits: np.ndarray, bits: int):
    """x: uint16 (bf16 bit patterns) [..., head_dim].

    Returns (codes uint8 [..., head_dim*bits/8], scalemin float32 [..., head_dim/64, 2]).
    """
    x = _c(x_bf16_bits, np.uint16)
    D = x.shape[-1]
    rows = int(np.prod(x.shape[:-1], dtype=np.int64))
    codes = np.zeros(x.shape[:-1] + (row_bytes(D, bits),), np.uint8)
    sm = np.zeros(x.shape[:-1] + (D // GROUP, 2), np.float32)
    rc = _load().oracle_quantize_rows(_ptr(x), rows, D, bits, _ptr(codes), _ptr(sm))
    if rc:
        raise ValueError(f"oracle_quantize_rows rejected the arguments (status {rc})")
    return codes, sm


def dequantize(codes: np.ndarray, scalemin: np.ndarray, head_dim: int, bits: int) -> np.ndarray:
    """Returns uint16 bf16 bit patterns [..., head_dim]."""
    codes = _c(codes, np.uint8)
    sm = _c(scalemin, np.float32)
    rows = int(np.prod(codes.shape[:-1], dtype=np.int64))
    y = np.zeros(codes.shape[:-1] + (head_dim,), np.uint16)
    rc = _load().oracle_dequantize_rows(_ptr(codes), _ptr(sm), rows, head_dim, bits, _ptr(y))
    if rc:
        raise ValueError(f"oracle_dequantize_rows rejected the arguments (status {rc})")
    return y


def unpack(codes: np.ndarray, head_dim: int, bits: int) -> np.ndarray:
    """Integer code values, uint8 [..., head_dim]."""
    codes = _c(codes, np.uint8)
    rows = int(np.prod(codes.shape[:-1], dtype=np.int64))
    out = np.zeros(codes.shape[:-1] + (head_dim,), np.uint8)
    rc = _load().oracle_unpack_rows(_ptr(codes), rows, head_dim, bits, _ptr(out))
    if rc:
        raise ValueError(f"oracle_unpack_rows rejected the arguments (status {rc})")
    return out


def affine(codes: np.ndarray, scalemin: np.ndarray, head_dim: int, bits: int) -> np.ndarray:
    """Exact fp64 values mn + s*c, [..., head_dim]."""
    codes = _c(codes, np.uint8)
    sm = _c(scalemin, np.float32)
    rows = int(np.prod(codes.shape[:-1], dtype=np.int64))
    out = np.zeros(codes.shape[:-1] + (head_dim,), np.float64)
    rc = _load().oracle_affine_rows(_ptr(codes), _ptr(sm), rows, head_dim, bits, _ptr(out))
    if rc:
        raise ValueError(f"oracle_affine_rows rejected the arguments (status {rc})")
    return out


def decode_attn(q: np.ndarray, bits: int,
                k_codes: np.ndarray | None, k_sm: np.ndarray | None,
                v_codes: np.ndarray | None, v_sm: np.ndarray | None,
                k_win: np.ndarray | None, v_win: np.ndarray | None,
                softmax_scale: float, want_probs: bool = False):
    """One view's decode attention in fp64.

    q: uint16 bf16 [H_q][D].  Packed: k_codes/v_codes uint8 [H_kv][n_p][rb],
    k_sm/v_sm float32 [H_kv][n_p][D/64][2] (or None when n_p == 0).  Window:
    k_win/v_win uint16 bf16 [H_kv][n_w][D] in logical (oldest-first) order
    (or None when n_w == 0).  Returns out float64 [H_q][D] (and probabilities
    [H_q][n_p + n_w] when want_probs).
    """
    q = _c(q, np.uint16)
    Hq, D = q.shape
    if k_codes is not None:
        k_codes = _c(k_codes, np.uint8); v_codes = _c(v_codes, np.uint8)
        k_sm = _c(k_sm, np.float32); v_sm = _c(v_sm, np.float32)
        Hkv, n_p = k_codes.shape[:2]
    else:
        n_p = 0
    if k_win is not None:
        k_win = _c(k_win, np.uint16); v_win = _c(v_win, np.uint16)
        Hkv, n_w = k_win.shape[:2]
    else:
        n_w = 0
    if n_p == 0 and n_w == 0:
        raise ValueError("empty view")
    out = np.zeros((Hq, D), np.float64)
    probs = np.zeros((Hq, n_p + n_w), np.float64) if want_probs else None
    null = ctypes.c_void_p(0)
    rc = _load().oracle_decode_attn(
        Hq, Hkv, D, bits, n_p,
        _ptr(k_codes) if n_p else null, _ptr(k_sm) if n_p else null,
        _ptr(v_codes) if n_p else null, _ptr(v_sm) if n_p else null,
        n_w, _ptr(k_win) if n_w else null, _ptr(v_win) if n_w else null,
        _ptr(q), float(softmax_scale), _ptr(out), _ptr(probs) if want_probs else null)
    if rc:
        raise ValueError(f"oracle_decode_attn rejected the arguments (status {rc})")
    return (out, probs) if want_probs else out


def _bf16_to_f64(bits_u16: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> their exact fp64 values (a bf16 is the top half of an fp32)."""
    return (_c(bits_u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_attn_segments(q: np.ndarray, segments, softmax_scale: float) -> np.ndarray:
    """Decode attention of one sequence whose tokens are held by several
    segments, each with its own width, in fp64.

    Sources: "Coordinated Mixed-Precision KV Cache Quantization ..." (Abstract:
    only newly quantized blocks take a new allocation, old ones keep theirs)
    and "QKVShare ..." (Metodologia: per-token widths {2, 4, 8, FP16}).
    Reading: the sequence's cache is the union of its segments' (key, value)
    pairs, the packed ones attended as their exact affine values mn + s*c and
    the window ones as bf16; softmax attention depends on that set only, not on
    where each pair sits.  So this is textbook softmax attention over the
    segments' rows concatenated: logits = scale * K q, p = softmax(logits),
    out = p V, with query head h reading KV head h // (Hq / Hkv).

    q: uint16 bf16 [H_q][D].  segments: list of dicts with "bits" and any of
    k_codes/v_codes (uint8 [H_kv][n_p][rb]), k_sm/v_sm (float32
    [H_kv][n_p][D/64][2]), k_win/v_win (uint16 bf16 [H_kv][n_w][D], oldest
    first); missing or zero-length parts hold no tokens.  Returns float64
    [H_q][D].
    """
    q = _c(q, np.uint16)
    Hq, D = q.shape
    ks, vs = [], []
    for seg in segments:
        kc = seg.get("k_codes")
        if kc is not None and kc.shape[1] > 0:
            ks.append(affine(kc, seg["k_sm"], D, seg["bits"]))
            vs.append(affine(seg["v_codes"], seg["v_sm"], D, seg["bits"]))
        kw = seg.get("k_win")
        if kw is not None and kw.shape[1] > 0:
            ks.append(_bf16_to_f64(kw))
            vs.append(_bf16_to_f64(seg["v_win"]))
    if not ks:
        raise ValueError("empty sequence")
    k = np.concatenate(ks, axis=1)
    v = np.concatenate(vs, axis=1)
    Hkv = k.shape[0]
    if Hq % Hkv:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    G = Hq // Hkv
    qd = _bf16_to_f64(q)
    out = np.zeros((Hq, D), np.float64)
    for h in range(Hq):
        logits = softmax_scale * (k[h // G] @ qd[h])
        w = np.exp(logits - logits.max())
        out[h] = (w / w.sum()) @ v[h // G]
    return out


def sparse_decode_attn(q: np.ndarray, bits: int, k_codes, k_sm, v_codes, v_sm, k_win, v_win,
                       softmax_scale: float, top_k: int):
    """Top-K sparse decode attention over one view, in fp64.

    Source: "Reasoning-Aware Error-Bounded KV-Cache Compression and Sparse
    Attention for Long-Context LLMs" (Metodologia C, dynamic sparse decode
    attention: the top-K entries by a query-aware score form the active set,
    the others stay in the cache unused for this step).  Readings: the score
    of a packed token for a KV head is its instantaneous query-key
    compatibility, the largest logit softmax_scale * q_h . k over the query
    heads h of that KV head's group (the page's utility terms need attention
    history and a reasoning-phase signal, which the decode step does not
    have); the K highest-scoring packed tokens are selected per KV head, equal
    scores going to the lower token index; the bf16 recent window is always
    active (recent states are kept native and never evicted).  Attention is
    then plain softmax attention over the active tokens.

    Arguments as decode_attn, plus top_k >= 1.  Returns (out float64 [H_q][D],
    selected: list over KV heads of ascending packed-token index arrays).
    """
    q = _c(q, np.uint16)
    Hq, D = q.shape
    n_p = 0 if k_codes is None else k_codes.shape[1]
    n_w = 0 if k_win is None else k_win.shape[1]
    if n_p + n_w == 0 or top_k < 1:
        raise ValueError("empty view or top_k < 1")
    Hkv = (k_codes if n_p else k_win).shape[0]
    G = Hq // Hkv
    qd = _bf16_to_f64(q)
    kp = affine(k_codes, k_sm, D, bits) if n_p else np.zeros((Hkv, 0, D))
    vp = affine(v_codes, v_sm, D, bits) if n_p else np.zeros((Hkv, 0, D))
    kw = _bf16_to_f64(k_win) if n_w else np.zeros((Hkv, 0, D))
    vw = _bf16_to_f64(v_win) if n_w else np.zeros((Hkv, 0, D))
    out = np.zeros((Hq, D), np.float64)
    selected = []
    for hk in range(Hkv):
        heads = range(hk * G, (hk + 1) * G)
        if n_p:
            score = np.max(np.stack([softmax_scale * (kp[hk] @ qd[h]) for h in heads]), axis=0)
            # descending score, ties to the lower index (stable sort of -score)
            order = np.argsort(-score, kind="stable")
            sel = np.sort(order[:min(top_k, n_p)])
        else:
            sel = np.zeros(0, np.int64)
        selected.append(sel)
        k = np.concatenate([kp[hk][sel], kw[hk]], axis=0)
        v = np.concatenate([vp[hk][sel], vw[hk]], axis=0)
        for h in heads:
            logits = softmax_scale * (k @ qd[h])
            w = np.exp(logits - logits.max())
            out[h] = (w / w.sum()) @ v
    return out, selected


def width_sensitivity(q: np.ndarray, k_win: np.ndarray, v_win: np.ndarray, softmax_scale: float) -> float:
    """Sensitivity S of one view to the width of its next quantized blocks, in
    fp64: quantizing at b bits is expected to move the attention output by at
    most about S / (2^b - 1).

    Source: "Coordinated Mixed-Precision KV Cache Quantization ..." (Abstract:
    sensitivity from a local attention-error bound on recent queries, keys and
    values, with no calibration data and no trial quantization).  The page
    prints no formula; this is the first-order bound that the format gives.
    A group of range R quantized at b bits moves each element by at most
    s/2 = R / (2 (2^b - 1)).  For KV head hk, over its recent (window) tokens:
      R_k[g], R_v[g] = the largest group range of K, V in group g;
      V_max = the largest ||v_t||_2;
      Delta = scale * max over the group's query heads h of
              sum_g ||q_h[g]||_1 * R_k[g] / 2          (logit shift * (2^b - 1));
      E_v = sqrt(sum_g 64 * (R_v[g] / 2)^2)            (value shift * (2^b - 1)).
    A logit shift of at most delta moves the softmax by at most e^(2 delta) - 1
    in L1, so the output moves by at most V_max (e^(2 Delta/(2^b-1)) - 1) +
    E_v / (2^b - 1); to first order that is S / (2^b - 1) with
    S = 2 V_max Delta + E_v.  The view's S is the largest over its KV heads;
    0 without recent tokens.

    q: uint16 bf16 [H_q][D]; k_win, v_win: uint16 bf16 [H_kv][n_w][D].
    Returns (S, Delta, E_v, V_max) with the last three per KV head.
    """
    q = _bf16_to_f64(q)
    k = _bf16_to_f64(k_win)
    v = _bf16_to_f64(v_win)
    Hq, D = q.shape
    Hkv, n_w = k.shape[:2]
    G, NG = Hq // Hkv, D // GROUP
    S, deltas, evs, vmaxs = 0.0, [], [], []
    for hk in range(Hkv):
        if n_w == 0:
            deltas.append(0.0); evs.append(0.0); vmaxs.append(0.0)
            continue
        kg = k[hk].reshape(n_w, NG, GROUP)
        vg = v[hk].reshape(n_w, NG, GROUP)
        rk = (kg.max(axis=2) - kg.min(axis=2)).max(axis=0)
        rv = (vg.max(axis=2) - vg.min(axis=2)).max(axis=0)
        vmax = np.sqrt((v[hk] ** 2).sum(axis=1)).max()
        l1 = np.abs(q[hk * G:(hk + 1) * G].reshape(G, NG, GROUP)).sum(axis=2)
        delta = softmax_scale * (l1 * rk / 2).sum(axis=1).max()
        ev = np.sqrt((64 * (rv / 2) ** 2).sum())
        deltas.append(delta); evs.append(ev); vmaxs.append(vmax)
        S = max(S, 2 * vmax * delta + ev)
    return S, deltas, evs, vmaxs


WIDTHS = (8, 4, 3, 2)


def allocate_widths(sens, capacity, n_kv_heads: int, head_dim: int, budget_bytes: int, units: int = 4096):
    """Joint width allocation under a shared byte budget.

    Source: "Coordinated Mixed-Precision KV Cache Quantization ..." (Abstract:
    a shared controller combines the sensitivity scores with the remaining
    quantizable capacity and byte-level storage costs to minimize total
    estimated error).  Reading: view v, given width b, stores its capacity_v
    tokens still to be quantized at 2 * n_kv_heads * (head_dim*b/8 +
    (head_dim/64)*8) bytes each and contributes sens_v / (2^b - 1) to the
    total estimated error.  The budget is cut into `units` equal units (a
    unit is ceil(budget / units) bytes) and each option's cost is rounded up
    to whole units, so a chosen allocation never exceeds the budget; among
    allocations within it the total error is minimal (dynamic programming
    over views and units).  Equal totals keep the earlier choice in the
    order 8, 4, 3, 2 bits of the earlier view.  Returns (bits per view,
    total error), or None when even all-2-bit does not fit.
    """
    n = len(sens)
    unit = -(-int(budget_bytes) // units) if budget_bytes > 0 else 1
    cap_units = int(budget_bytes) // unit
    INF = float("inf")
    best = np.full(cap_units + 1, INF)        # best[u]: least error of the views so far using exactly u units
    best[0] = 0.0
    choice = np.zeros((n, cap_units + 1), np.int8)
    for i in range(n):
        new = np.full(cap_units + 1, INF)
        pick = np.zeros(cap_units + 1, np.int8)
        for j, b in enumerate(WIDTHS):
            cost = -(-(int(capacity[i]) * 2 * n_kv_heads * (head_dim * b // 8 + head_dim // 64 * 8)) // unit)
            err = float(sens[i]) / (2 ** b - 1)
            for u in range(cost, cap_units + 1):
                cand = best[u - cost] + err
                if cand < new[u]:
                    new[u] = cand
                    pick[u] = j
        best = new
        choice[i] = pick
    # the least total error over every budget use; the smallest such use
    u = int(np.argmin(best))
    if best[u] == INF:
        return None
    total = float(best[u])
    bits = [0] * n
    for i in range(n - 1, -1, -1):
        j = int(choice[i][u])
        bits[i] = WIDTHS[j]
        cost = -(-(int(capacity[i]) * 2 * n_kv_heads * (head_dim * WIDTHS[j] // 8 + head_dim // 64 * 8)) // unit)
        u -= cost
    return bits, total


class WindowModel:
    """Bookkeeping model of one view's token placement under appends.

    From "Coordinated Mixed-Precision KV Cache Quantization ..." (Abstract):
    recent states keep native precision and only newly quantized blocks get a
    width.  Reading used here: the cache of a view that has seen tokens
    0..n-1 holds tokens [0, n - W) quantized, in order, and the last min(n, W)
    tokens in a bf16 ring of W slots; appending a token when the ring is full
    first quantizes the oldest ring token (at the view's width at that moment)
    and appends it to the packed part, then stores the new token in the freed
    slot.  With W == 0 every token is quantized on arrival.

    Pure list logic: it tracks which token sits where, never a value.
    """

    def __init__(self, capacity_window: int, packed_tokens=(), window_tokens=(), head: int = 0):
        self.W = capacity_window
        self.packed = list(packed_tokens)      # token ids, oldest first
        self.slots = [None] * capacity_window  # ring: slot -> token id
        self.head = head
        for i, tok in enumerate(window_tokens):
            self.slots[(head + i) % capacity_window] = tok
        self.n_window = len(window_tokens)

    def append(self, tok):
        """Returns the token id that was flushed into the packed part, or None."""
        if self.W == 0:
            self.packed.append(tok)
            return tok
        if self.n_window == self.W:
            old = self.slots[self.head]
            self.packed.append(old)
            self.slots[self.head] = tok
            self.head = (self.head + 1) % self.W
            return old
        self.slots[(self.head + self.n_window) % self.W] = tok
        self.n_window += 1
        return None

    def window_logical(self):
        return [self.slots[(self.head + i) % self.W] for i in range(self.n_window)]
