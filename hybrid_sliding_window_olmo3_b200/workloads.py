"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module holds workload shapes and random-number recipes only: none of the
attention arithmetic.  Both the GPU path and the oracle consume the exact
values it returns.

Recipe (the same for every consumer):

* seed = 20261202 + config index;
* q, k, v ~ N(0, 1) (float32 for the toy case, bfloat16 otherwise), drawn
  pre-norm, layer by layer, in the order q, k, v;
* QK-norm gains ~ U(0.5, 1.5), float32, sizes H*d and G*d;
* decode caches ~ N(0, 1) bfloat16 (read as already normed and rotated keys);
* ragged context lengths ~ U[1, 65536] (integers, inclusive).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SEED_BASE = 20261202


@dataclass(frozen=True)
class Shape:
    name: str
    n_layers: int
    H: int
    G: int
    d: int
    window: int = 4096
    eps: float = 1e-6
    theta: float = 500000.0


TOY = Shape("toy", 6, 2, 1, 64, window=4)
OLMO3_7B = Shape("olmo3-7b", 32, 32, 32, 128)
OLMO3_32B = Shape("olmo3-32b", 64, 40, 8, 128)


@dataclass(frozen=True)
class Workload:
    index: int               # position in the list of configurations (seeds the RNG)
    name: str
    shape: Shape
    B: int
    T: int = 0               # prefill tokens per sequence
    context: int = 0         # cached tokens per sequence before decoding
    steps: int = 0           # decode steps
    ragged: bool = False
    layers: tuple = field(default_factory=tuple)   # layer indices exercised (prefill)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index


WORKLOADS = {
    "toy": Workload(0, "toy", TOY, B=1, T=16, steps=8, layers=tuple(range(6))),
    "7b-prefill": Workload(1, "7b-prefill", OLMO3_7B, B=1, T=8192, layers=(0, 3)),
    "7b-decode": Workload(2, "7b-decode", OLMO3_7B, B=32, context=32768, steps=64),
    "32b-prefill": Workload(3, "32b-prefill", OLMO3_32B, B=2, T=8192, layers=(0, 3)),
    "32b-decode": Workload(3, "32b-decode", OLMO3_32B, B=8, context=65536, steps=64),
    "ragged-7b-decode": Workload(4, "ragged-7b-decode", OLMO3_7B, B=64, steps=32, ragged=True),
}


def toy_layer_inputs(seed: int = SEED_BASE, T_total: int = 24, shape: Shape = TOY):
    """Per-layer float32 numpy inputs of the toy case: list of dicts with
    q [1, T_total, H, d], k/v [1, T_total, G, d], gain_q [H*d], gain_k [G*d]."""
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(shape.n_layers):
        q = rng.standard_normal((1, T_total, shape.H, shape.d)).astype(np.float32)
        k = rng.standard_normal((1, T_total, shape.G, shape.d)).astype(np.float32)
        v = rng.standard_normal((1, T_total, shape.G, shape.d)).astype(np.float32)
        gq = rng.uniform(0.5, 1.5, shape.H * shape.d).astype(np.float32)
        gk = rng.uniform(0.5, 1.5, shape.G * shape.d).astype(np.float32)
        out.append(dict(q=q, k=k, v=v, gain_q=gq, gain_k=gk))
    return out


def qkv_bf16(B: int, T: int, H: int, G: int, d: int, seed: int, layer: int = 0):
    """CPU bfloat16 q [B,T,H,d], k/v [B,T,G,d] ~ N(0,1) and float32 gains ~ U(0.5,1.5)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000 + layer)
    q = torch.randn(B, T, H, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B, T, G, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, T, G, d, generator=g).to(torch.bfloat16)
    gq = torch.rand(H * d, generator=g) + 0.5
    gk = torch.rand(G * d, generator=g) + 0.5
    return q, k, v, gq.float(), gk.float()


def randn_bf16(shape, seed: int, device="cpu"):
    """bfloat16 N(0,1) tensor drawn on ``device`` from a seeded generator."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16) \
        if device == "cpu" else torch.randn(*shape, generator=g, device=device, dtype=torch.bfloat16)


def ragged_lengths(B: int, seed: int, lo: int = 1, hi: int = 65536) -> np.ndarray:
    """Context lengths ~ U[lo, hi] (inclusive), int64."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=B, dtype=np.int64)
