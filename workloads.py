"""Seeded synthetic inputs for the Echo all-reduce simulation.

This module only draws random numbers and shapes them; it holds none of the
method's arithmetic, so both the CUDA path's tests/benchmark and the oracle
can use it. The workloads stand in for tensor-parallel activations of the
models the Echo pages evaluate (Llama-3-8B / Qwen3-8B hidden 4096, Qwen3-0.6B
depth 56); no dataset is involved.

Seeds: the stream of rank ``r`` at site ``t`` of workload ``c`` is seeded with
``c * 1_000_000 + t * 1_000 + r`` (workload ``tiny`` is c = 0, so rank 0 uses
seed 0). Values are drawn in float32 and rounded to bf16 by torch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    cid: int                 # seed namespace
    P: int
    tokens: int
    hidden: int
    bits: int = 4
    group: int = 128
    eta: float = 1.0
    alpha_long: float = 0.05
    alpha_short: float = 0.5
    w: float = 0.5
    dist: str = "normal"     # "normal" | "normal_outliers" | "student_t3"
    sites: int = 1           # > 1: a chain of calls with carried state
    int8_sites: int = 0      # chain: the first int8_sites sites use 8 bits
    decay: float = 0.9       # chain: site input = decay * previous output / P + noise
    notes: str = ""

    @property
    def n(self) -> int:
        return self.tokens * self.hidden

    def bits_at(self, site: int) -> int:
        return 8 if site < self.int8_sites else self.bits


# The five workloads: one tiny call, one 32 MB TP-shaped call with outlier
# channels, a 56-site chain, the 1 GB headline call, a mixed 8/4-bit chain.
TINY = Workload("tiny_p2_32x128", 0, P=2, tokens=32, hidden=128,
                notes="one call, N(0,1), zero EMAs")
TP8B = Workload("tp_p8_4096x4096_outliers", 1, P=8, tokens=4096, hidden=4096,
                dist="normal_outliers",
                notes="N(0,1), 0.1% of hidden channels (4) scaled x20 on every rank")
CHAIN56 = Workload("chain_p8_56x2048x1024", 2, P=8, tokens=2048, hidden=1024, sites=56,
                   notes="site input = 0.9 * previous output / P + N(0,1) noise")
HEADLINE = Workload("p8_1GB_student_t", 3, P=8, tokens=131072, hidden=4096,
                    dist="student_t3",
                    notes="1 GB bf16 message per rank, Student-t nu=3 scaled to unit variance")
CHAIN48_MIXED = Workload("chain_p4_48x1024x5120_int8x12", 4, P=4, tokens=1024, hidden=5120,
                         sites=48, int8_sites=12,
                         notes="first 12 sites 8-bit, the rest 4-bit, state carried over")

ALL = [TINY, TP8B, CHAIN56, HEADLINE, CHAIN48_MIXED]


def seed_of(cid: int, site: int, rank: int) -> int:
    return cid * 1_000_000 + site * 1_000 + rank


def _gen(device: torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_f32(n: int, seed: int, device="cpu") -> torch.Tensor:
    device = torch.device(device)
    return torch.randn(n, generator=_gen(device, seed), device=device, dtype=torch.float32)


def student_t3_unit_f32(n: int, seed: int, device="cpu") -> torch.Tensor:
    """Student-t with 3 degrees of freedom, divided by sqrt(3) (its std)."""
    device = torch.device(device)
    g = _gen(device, seed)
    z0 = torch.randn(n, generator=g, device=device, dtype=torch.float32)
    chi = torch.zeros(n, device=device, dtype=torch.float32)
    for _ in range(3):
        z = torch.randn(n, generator=g, device=device, dtype=torch.float32)
        chi.add_(z * z)
        del z
    t = z0 / torch.sqrt(chi / 3.0)
    del chi, z0
    return t / math.sqrt(3.0)


def outlier_channels(w: Workload, count: Optional[int] = None) -> torch.Tensor:
    count = max(1, round(0.001 * w.hidden)) if count is None else count
    g = _gen(torch.device("cpu"), seed_of(w.cid, 999, 999))
    return torch.randperm(w.hidden, generator=g)[:count]


def rank_input(w: Workload, rank: int, site: int = 0, device="cpu") -> torch.Tensor:
    """The bf16 partial sum of ``rank`` at ``site`` (flat, ``w.n`` elements)."""
    seed = seed_of(w.cid, site, rank)
    if w.dist == "student_t3":
        v = student_t3_unit_f32(w.n, seed, device)
    else:
        v = normal_f32(w.n, seed, device)
    if w.dist == "normal_outliers":
        ch = outlier_channels(w).to(v.device)
        v = v.view(w.tokens, w.hidden)
        v[:, ch] *= 20.0
        v = v.reshape(-1)
    return v.to(torch.bfloat16)


def inputs(w: Workload, site: int = 0, device="cpu") -> torch.Tensor:
    """All ranks' inputs as one ``[P, n]`` bf16 tensor."""
    out = torch.empty((w.P, w.n), dtype=torch.bfloat16, device=device)
    for r in range(w.P):
        out[r].copy_(rank_input(w, r, site, device))
    return out


def chain_noise(w: Workload, site: int, device="cpu") -> torch.Tensor:
    """``[P, n]`` float32 N(0,1) noise added at ``site`` of a chain."""
    out = torch.empty((w.P, w.n), dtype=torch.float32, device=device)
    for r in range(w.P):
        out[r].copy_(normal_f32(w.n, seed_of(w.cid, site, r), device))
    return out


def chain_next_input(y_bf16: torch.Tensor, noise_f32: torch.Tensor, P: int,
                     decay: float = 0.9) -> torch.Tensor:
    """Next site's inputs from this site's reduced output (the synthetic
    "network" between two all-reduce sites).

    ``x_next[r] = bf16_rn(decay * float(y[r]) / P + noise[r])`` in float32,
    one rounding per operation. Dividing by P keeps the summed signal a stable
    AR(1) process (a non-amplifying network); the literal ``decay * y`` per
    rank would multiply the sum by ``decay * P`` at every site.
    Always evaluated on the CPU so that every consumer gets identical bits.
    """
    y = y_bf16.detach().to("cpu").float()
    nz = noise_f32.detach().to("cpu")
    d = torch.tensor(decay, dtype=torch.float32)
    p = torch.tensor(float(P), dtype=torch.float32)
    t = torch.mul(y, d)
    t = torch.div(t, p)
    t = torch.add(t, nz)
    return t.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")


def from_bf16_bits(a) -> torch.Tensor:
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
