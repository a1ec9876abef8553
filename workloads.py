"""Seeded synthetic workloads for causal self-attention.

This module is the only code shared by the CUDA path's tests/bench and the
fp64 oracle.  It draws random numbers and nothing else: it holds none of the
attention arithmetic (no scores, softmax, masking or gradients).

Workload shapes follow the nanoGPT model sizes the pages describe:

* "nanoGPT: a real GPT in two 300-line files", section 3 "Run it, tested"
  (baby GPT: 6 heads, n_embd 384, block 256, batch 64);
* "nanoGPT: Minimal, Readable, and Fast PyTorch Framework for Training Medium
  GPTs", feature list (GPT-2 124M and 1558M);
* the head size D = n_embd / n_head of "CausalSelfAttention" in section 2
  "How the code works" of the first page.

Recipe (same for every configuration): a CPU ``torch.Generator`` seeded with
``1000 + index``; q, k, v, dO drawn in that order as fp32 standard normals of
shape (B, H, T, D); q and k multiplied by ``qk_std``; then rounded to bf16
(round-to-nearest-even) for the GPU.  The oracle receives the *same*
bf16-rounded values upcast to fp64, so a comparison measures kernel error
only.  ``scale`` is 1/sqrt(D) everywhere.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    D: int
    qk_std: float = 1.0
    # the tiny check keeps its fp32 draws for the oracle's own self-tests
    fp32_inputs: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def BH(self) -> int:
        return self.B * self.H

    def describe(self) -> str:
        return f"B={self.B} H={self.H} T={self.T} D={self.D}"


# The five configurations, index 0..4.
WORKLOADS = [
    Workload("tiny_check_b1_h2_t64_d16", 1, 2, 64, 16, fp32_inputs=True),
    Workload("shakespeare_char_layer_b64_h6_t256_d64", 64, 6, 256, 64),
    Workload("gpt2_124m_layer_b16_h12_t1024_d64", 16, 12, 1024, 64),
    Workload("gpt2_1558m_layer_b8_h25_t1024_d64", 8, 25, 1024, 64),
    # q and k with std 2 each: scale*q.k has std 2*2 = 4 (peaked softmax)
    Workload("long_context_b2_h16_t8192_d128_logit_std4", 2, 16, 8192, 128,
             qk_std=2.0),
]

# The workload the benchmark headline is quoted on (GPT-2 124M layer).
HEADLINE = 2


def seed_for(index: int) -> int:
    return 1000 + index


def draw(B: int, H: int, T: int, D: int, seed: int, qk_std: float = 1.0):
    """Draw fp32 (q, k, v, dO) of shape (B, H, T, D) from one CPU generator.

    Order of draws is q, k, v, dO.  Returns CPU fp32 tensors (not rounded).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    shape = (B, H, T, D)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_std != 1.0:
        q.mul_(qk_std)
        k.mul_(qk_std)
    return q, k, v, do


def bf16_inputs(B, H, T, D, seed, qk_std=1.0):
    """(q, k, v, dO) rounded to bf16 (CPU tensors, contiguous (B,H,T,D))."""
    return tuple(t.to(torch.bfloat16).contiguous()
                 for t in draw(B, H, T, D, seed, qk_std))


def workload_inputs(index: int):
    """bf16 (q, k, v, dO) of workload ``index`` with its recipe seed."""
    w = WORKLOADS[index]
    return bf16_inputs(w.B, w.H, w.T, w.D, seed_for(index), w.qk_std)


def as_f64(t: torch.Tensor):
    """bf16/fp32 CPU tensor -> numpy float64 (exact upcast)."""
    return t.detach().to(torch.float64).cpu().numpy()


def draw_extra(shape, seed: int, std: float = 1.0, dtype=torch.bfloat16):
    """One extra standard-normal tensor (e.g. a synthetic O for the
    preprocess step, drawn independently of any kernel output)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype).contiguous()


def sample_heads(BH: int, n: int, seed: int):
    """A seeded sorted subsample of n flat (b*H + h) head indices."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    n = min(n, BH)
    return sorted(torch.randperm(BH, generator=g)[:n].tolist())
