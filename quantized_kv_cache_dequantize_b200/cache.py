"""Pooled device memory for many (agent, layer) views, and the decode
workloads built from seeded inputs.

One allocation per tensor kind (codes, scale/min, window) holds every view's
slice, 256-byte aligned, so a workload of hundreds of views costs a handful of
cudaMallocs.  Filling a view quantizes its seeded bf16 prefill cache with the
library's own kvq_quantize; the oracle side regenerates the same bf16 bytes
from the same seeds and quantizes them itself.
"""
from __future__ import annotations

import torch

from . import View, row_bytes, GROUP
from . import workloads as wl


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class ViewPool:
    """Views over pooled tensors.  specs: list of dicts with keys
    n_kv_heads, head_dim, bits, cap_packed, cap_window."""

    def __init__(self, specs, device="cuda"):
        code_off, sm_off, win_off = [], [], []
        nc = ns = nw = 0
        for s in specs:
            cap = s["cap_packed"] + (s["cap_packed"] & 1)
            s["cap_packed"] = cap
            H, D, b, W = s["n_kv_heads"], s["head_dim"], s["bits"], s["cap_window"]
            cb = H * cap * row_bytes(D, b)
            sb = H * cap * (D // GROUP) * 2 * 4
            wb = H * W * D * 2
            code_off.append(nc); nc += 2 * _align(cb)
            sm_off.append(ns); ns += 2 * _align(sb)
            win_off.append(nw); nw += 2 * _align(wb)
        self.codes = torch.zeros(max(nc, 16), dtype=torch.uint8, device=device)
        self.sm = torch.zeros(max(ns, 16), dtype=torch.uint8, device=device)
        self.win = torch.zeros(max(nw, 16), dtype=torch.uint8, device=device)
        self.views = []
        for s, co, so, wo in zip(specs, code_off, sm_off, win_off):
            H, D, b, W, cap = s["n_kv_heads"], s["head_dim"], s["bits"], s["cap_window"], s["cap_packed"]
            cb = H * cap * row_bytes(D, b)
            sb = H * cap * (D // GROUP) * 2 * 4
            wb = H * W * D * 2
            t = dict(
                k_codes=self.codes[co:co + cb].view(H, cap, row_bytes(D, b)),
                v_codes=self.codes[co + _align(cb):co + _align(cb) + cb].view(H, cap, row_bytes(D, b)),
                k_scalemin=self.sm[so:so + sb].view(torch.float32).view(H, cap, D // GROUP, 2),
                v_scalemin=self.sm[so + _align(sb):so + _align(sb) + sb].view(torch.float32).view(H, cap, D // GROUP, 2),
                k_window=self.win[wo:wo + wb].view(torch.bfloat16).view(H, W, D),
                v_window=self.win[wo + _align(wb):wo + _align(wb) + wb].view(torch.bfloat16).view(H, W, D),
            )
            self.views.append(View(H, D, b, cap, W, device=device, tensors=t))

    def nbytes(self) -> int:
        return self.codes.numel() + self.sm.numel() + self.win.numel()


def view_inputs(w: wl.DecodeWorkload, agent: int, layer: int, device="cuda"):
    """Seeded bf16 K, V [H_kv, n_p + n_w, D] of one view (prefill then window
    tokens) and the ring slot of its oldest window token."""
    seed = wl.view_seed(w, agent, layer)
    gmask = wl.generator(seed ^ 0x5A5A5A5)
    mask = wl.outlier_mask(gmask, w.n_kv_heads, w.head_dim, w.outlier_frac, first4=w.outlier_first4)
    g = wl.generator(seed, device=device)
    n_p = w.view_len(agent)
    n_w = w.window
    k, v = wl.kv_pair(g, w.n_kv_heads, n_p + n_w, w.head_dim, mask, device)
    head = (agent * 7 + layer * 3) % w.window if w.window else 0
    return k, v, head


def decode_queries(w: wl.DecodeWorkload, step: int = 0, device="cuda") -> torch.Tensor:
    """bf16 q [n_views, H_q, D], view order (agent, layer) agent-major."""
    g = wl.generator(w.seed * 7919 + 17 + step, device=device)
    return wl.normal_bf16(g, (w.n_views, w.n_q_heads, w.head_dim), device)


def decode_new_tokens(w: wl.DecodeWorkload, step: int = 0, device="cuda"):
    g = wl.generator(w.seed * 104729 + 31 + step, device=device)
    k = wl.normal_bf16(g, (w.n_views, w.n_kv_heads, w.head_dim), device)
    v = wl.normal_bf16(g, (w.n_views, w.n_kv_heads, w.head_dim), device)
    return k, v


def build_decode(w: wl.DecodeWorkload, device="cuda", extra_packed: int = 0) -> ViewPool:
    """All views of a decode workload, filled: packed prefill tokens quantized
    with kvq_quantize, a full bf16 window placed in the ring.  extra_packed
    reserves packed rows for later appends."""
    specs = []
    for a in range(w.n_agents):
        for l in range(w.n_layers):
            specs.append(dict(n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, bits=w.view_bits(a, l),
                              cap_packed=w.view_len(a) + extra_packed, cap_window=w.window))
    pool = ViewPool(specs, device)
    i = 0
    for a in range(w.n_agents):
        for l in range(w.n_layers):
            k, v, head = view_inputs(w, a, l, device)
            n_p = w.view_len(a)
            view = pool.views[i]
            view.fill_packed(k[:, :n_p], v[:, :n_p])
            if w.window:
                view.fill_window(k[:, n_p:], v[:, n_p:], head=head)
            i += 1
            del k, v
    return pool
