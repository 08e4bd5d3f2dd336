"""Shared test plumbing: build views from seeded inputs, run both sides, compare.

Inputs come from the seeded generators in ``workloads``; the GPU side runs
through the C ABI (the package binding), the oracle side quantizes the same
bf16 bytes itself and attends in fp64.  Nothing computed by the CUDA path is
handed to the oracle.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
import quantized_kv_cache_dequantize_b200 as kvq
from quantized_kv_cache_dequantize_b200 import workloads as wl

ATOL = 2e-3      # max elementwise |o - o_ref|
RTOL_L2 = 1e-3   # max over (view, head) of ||o - o_ref|| / ||o_ref||


@dataclass
class ViewSpec:
    n_packed: int
    n_window: int
    cap_window: int
    bits: int = 4
    head: int = 0          # ring slot of the oldest window token
    seed: int = 0
    outlier_frac: float = 0.0
    first4: bool = False


@dataclass
class Case:
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    specs: list
    views: list = field(default_factory=list)
    q: torch.Tensor | None = None
    host: list = field(default_factory=list)   # per view: dict of numpy bf16 bits
    q_bits: np.ndarray | None = None


def build_case(n_q_heads, n_kv_heads, head_dim, specs, q_seed=99, device="cuda", extra_packed=0) -> Case:
    case = Case(n_q_heads, n_kv_heads, head_dim, list(specs))
    for s in specs:
        g = wl.generator(s.seed)
        mask = wl.outlier_mask(g, n_kv_heads, head_dim, s.outlier_frac, first4=s.first4)
        k, v = wl.kv_pair(g, n_kv_heads, s.n_packed + s.n_window, head_dim, mask)
        view = kvq.View(n_kv_heads, head_dim, s.bits, max(s.n_packed + extra_packed, 2), s.cap_window, device=device)
        if s.n_packed:
            view.fill_packed(k[:, :s.n_packed].to(device), v[:, :s.n_packed].to(device))
        if s.cap_window:
            view.fill_window(k[:, s.n_packed:].to(device), v[:, s.n_packed:].to(device), head=s.head)
        case.views.append(view)
        case.host.append(dict(k=wl.bf16_bits(k), v=wl.bf16_bits(v)))
    gq = wl.generator(q_seed)
    q = wl.normal_bf16(gq, (len(specs), n_q_heads, head_dim))
    case.q = q.to(device)
    case.q_bits = wl.bf16_bits(q)
    return case


def oracle_view(case: Case, i: int, scale: float) -> np.ndarray:
    s = case.specs[i]
    h = case.host[i]
    kw = vw = None
    kc = ks = vc = vs = None
    if s.n_packed:
        kc, ks = oracle.quantize(h["k"][:, :s.n_packed], s.bits)
        vc, vs = oracle.quantize(h["v"][:, :s.n_packed], s.bits)
    if s.n_window:
        kw, vw = h["k"][:, s.n_packed:], h["v"][:, s.n_packed:]
    return oracle.decode_attn(case.q_bits[i], s.bits, kc, ks, vc, vs, kw, vw, scale)


def run_gpu(case: Case, scale: float, workspace=None) -> np.ndarray:
    out = kvq.decode_attn(case.views, case.q, scale, workspace=workspace)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def compare(out: np.ndarray, ref: np.ndarray):
    """Returns (max_abs, max_rel_l2) over [..., H, D] arrays."""
    diff = np.abs(out - ref)
    num = np.sqrt(((out - ref) ** 2).sum(axis=-1))
    den = np.sqrt((ref ** 2).sum(axis=-1))
    rel = num / np.maximum(den, 1e-30)
    return float(diff.max()), float(rel.max())


def assert_close(out, ref, what=""):
    mx, rel = compare(out, ref)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    assert mx <= ATOL and rel <= RTOL_L2, f"{what}: max_abs {mx:.3e} (<= {ATOL}), rel_l2 {rel:.3e} (<= {RTOL_L2})"
    return mx, rel


def host_threads() -> int:
    import os
    return max(1, len(os.sched_getaffinity(0)))


class OracleRunner:
    """Runs oracle checks on host threads (the C oracle releases the GIL in
    ctypes calls) while the main thread prepares the next inputs.  submit()
    takes a function returning None (pass) or a failure message; at most
    `depth` checks are in flight, which bounds the host memory they hold."""

    def __init__(self, depth: int | None = None):
        from concurrent.futures import ThreadPoolExecutor
        self.n = host_threads()
        self.pool = ThreadPoolExecutor(self.n)
        self.depth = depth or 2 * self.n
        self.pending = []
        self.failures = []
        self.done = 0

    def _drain(self, keep: int):
        while len(self.pending) > keep:
            f = self.pending.pop(0)
            msg = f.result()
            self.done += 1
            if msg:
                self.failures.append(msg)

    def submit(self, fn, *args):
        self._drain(self.depth - 1)
        self.pending.append(self.pool.submit(fn, *args))

    def finish(self):
        self._drain(0)
        self.pool.shutdown()
        assert not self.failures, f"{len(self.failures)} of {self.done} checks failed; first: {self.failures[:3]}"
        return self.done


def close_msg(out, ref, what):
    """None if out is within the attention tolerance of ref, else a message."""
    if not np.all(np.isfinite(out)):
        return f"{what}: non-finite output"
    mx, rel = compare(out, ref)
    if mx <= ATOL and rel <= RTOL_L2:
        return None
    return f"{what}: max_abs {mx:.3e} (<= {ATOL}), rel_l2 {rel:.3e} (<= {RTOL_L2})"
