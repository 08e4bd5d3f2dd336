"""Seeded synthetic inputs for the five workloads (shared by tests and bench).

This module holds no arithmetic of the method: it only draws random numbers
and arranges them into the shapes of the workloads.  Both the CUDA path and
the oracle are fed from here.

Workloads (sizes follow the model shapes the pages evaluate):
  1 tiny       1 view, 4 q / 2 kv heads, head_dim 64, 256 packed tokens @4b,
               no window; K ~ N(0,1) with channels 0-3 of every kv head x10,
               V ~ N(0,1), q ~ N(0,1), softmax scale 1/8.
  2 handoff    quantize then dequantize one agent's prefill cache in
               Llama-3.1-8B shape: 32 layers x 8 kv heads x 32768 tokens x
               head_dim 128, K and V, 4-bit; K with 1% outlier channels x10.
  3 decode     10 agents x 32 layers, 32 q / 8 kv heads, head_dim 128,
               4096 packed tokens @4b + a 128-token bf16 window per view.
  4 varlen     6 agents x 48 layers, 16 q / 8 kv heads, head_dim 256,
               packed length per agent uniform from {4K, 8K, 16K, 32K},
               4-bit, 256-token window, K outlier channels x10.
  5 mixed      8 agents x 64 layers, 64 q / 8 kv heads, head_dim 128,
               packed length per agent uniform in [8192, 16384], widths per
               (agent, layer) with exact counts {8:32, 4:96, 3:128, 2:256}
               (mean 3.0 bits), 128-token window, K outlier channels x10.

Random numbers come from torch.Generator objects seeded per workload.  Small
draws use the CPU generator (bytes independent of the GPU); full-size draws
for the benchmark are made on the GPU with a seeded CUDA generator, and the
oracle is given copies of exactly those bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

GROUP = 64


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    n_agents: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    window: int                 # recent-window capacity W (tokens)
    lengths: tuple = ()         # packed length per agent (filled by make_*)
    bits: tuple = ()            # width per (agent, layer), agent-major
    outlier_frac: float = 0.0   # fraction of (kv head, channel) pairs of K scaled x10
    outlier_first4: bool = False
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def n_views(self) -> int:
        return self.n_agents * self.n_layers

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def view_bits(self, agent: int, layer: int) -> int:
        return self.bits[agent * self.n_layers + layer]

    def view_len(self, agent: int) -> int:
        return self.lengths[agent]


def tiny(seed: int = 1) -> DecodeWorkload:
    return DecodeWorkload("tiny single-agent", 1, 1, 4, 2, 64, 0, (256,), (4,),
                          outlier_first4=True, seed=seed)


def decode_llama8b(seed: int = 3, n_agents: int = 10, n_layers: int = 32,
                   length: int = 4096, window: int = 128) -> DecodeWorkload:
    return DecodeWorkload("batched multi-agent decode, Llama-3.1-8B shape", n_agents, n_layers,
                          32, 8, 128, window, (length,) * n_agents, (4,) * (n_agents * n_layers),
                          seed=seed)


def varlen_gemma12b(seed: int = 4, n_agents: int = 6, n_layers: int = 48,
                    choices=(4096, 8192, 16384, 32768), window: int = 256) -> DecodeWorkload:
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(0, len(choices), (n_agents,), generator=g).tolist()
    lengths = tuple(choices[i] for i in idx)
    return DecodeWorkload("variable-length decode, Gemma-3-12B shape", n_agents, n_layers,
                          16, 8, 256, window, lengths, (4,) * (n_agents * n_layers),
                          outlier_frac=0.01, seed=seed)


def mixed_qwen32b(seed: int = 5, n_agents: int = 8, n_layers: int = 64,
                  lo: int = 8192, hi: int = 16384, window: int = 128) -> DecodeWorkload:
    g = torch.Generator().manual_seed(seed)
    lengths = tuple(torch.randint(lo, hi + 1, (n_agents,), generator=g).tolist())
    n = n_agents * n_layers
    # exact counts for mean 3 bits over 512 views: 1/16 8-bit, 3/16 4-bit,
    # 1/4 3-bit, 1/2 2-bit; scaled proportionally for other view counts
    counts = {8: n // 16, 4: 3 * n // 16, 3: n // 4}
    counts[2] = n - sum(counts.values())
    pool = [b for b, c in counts.items() for _ in range(c)]
    perm = torch.randperm(n, generator=g).tolist()
    bits = tuple(pool[i] for i in perm)
    return DecodeWorkload("mixed-precision multi-agent decode, Qwen3-32B shape", n_agents, n_layers,
                          64, 8, 128, window, lengths, bits, outlier_frac=0.01, seed=seed)


@dataclass(frozen=True)
class HandoffWorkload:
    name: str
    n_layers: int
    n_kv_heads: int
    n_tokens: int
    head_dim: int
    bits: int
    outlier_frac: float
    seed: int


def handoff_llama8b(seed: int = 2, n_layers: int = 32, n_tokens: int = 32768) -> HandoffWorkload:
    return HandoffWorkload("bulk cache handoff, Llama-3.1-8B shape", n_layers, 8, n_tokens, 128, 4,
                           0.01, seed)


# ------------------------------------------------------------------ draws --

def generator(seed: int, device="cpu") -> torch.Generator:
    return torch.Generator(device=device).manual_seed(seed)


def outlier_mask(g: torch.Generator, n_kv_heads: int, head_dim: int, frac: float,
                 first4: bool = False) -> torch.Tensor:
    """Bool [n_kv_heads, head_dim]: the (head, channel) pairs of K scaled x10.

    first4: channels 0-3 of every head.  Otherwise ceil(frac * H * D) pairs
    drawn without replacement.
    """
    m = torch.zeros(n_kv_heads, head_dim, dtype=torch.bool)
    if first4:
        m[:, :4] = True
    elif frac > 0:
        k = math.ceil(frac * n_kv_heads * head_dim)
        idx = torch.randperm(n_kv_heads * head_dim, generator=g)[:k]
        m.view(-1)[idx] = True
    return m


def normal_bf16(g: torch.Generator, shape, device="cpu", scale_mask: torch.Tensor | None = None):
    """N(0,1) draws rounded to bf16; channels in scale_mask ([H, D], broadcast
    over tokens) multiplied by 10 before the rounding."""
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if scale_mask is not None:
        f = torch.ones(scale_mask.shape, dtype=torch.float32)
        f[scale_mask] = 10.0
        x = x * f.to(device).unsqueeze(-2)
    return x.to(torch.bfloat16)


def kv_pair(g: torch.Generator, n_kv_heads: int, n_tokens: int, head_dim: int,
            outliers: torch.Tensor | None, device="cpu"):
    """(K, V) bf16 [n_kv_heads, n_tokens, head_dim]; outliers on K only."""
    k = normal_bf16(g, (n_kv_heads, n_tokens, head_dim), device, outliers)
    v = normal_bf16(g, (n_kv_heads, n_tokens, head_dim), device, None)
    return k, v


def view_seed(wl, agent: int, layer: int, salt: int = 0) -> int:
    return (wl.seed * 1_000_003 + agent * 10_007 + layer * 101 + salt) & 0x7FFFFFFF


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
