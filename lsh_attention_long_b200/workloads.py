"""Seeded synthetic inputs for shared-QK LSH attention.

This module only draws random tensors; it holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can consume its output
without sharing any of the method's code.

Every tensor is drawn in fp32 on the CPU from a ``torch.Generator`` seeded
per tensor, then rounded once to the workload's dtype.  Rotations are drawn the
same way and rounded to the input dtype too, so that the tensor-core hash
multiplies exactly representable values.

Workloads (B, H, L, d, n_buckets, n_rounds, chunk, causal, dtype):

* ``fwd_f32_L1024``      : 1, 1, 1024, 64, 32, 1, 64, non-causal, f32.  Q then V
  from seed 0 (one generator, Q first), rotations [1, 64, 16] from seed 1.
* ``fwd_bf16_L4096``     : 8, 8, 4096, 64, 64, 2, 64, causal, bf16.
* ``fwd_bf16_L16384_clustered`` : 2, 8, 16384, 64, 256, 4, 64, non-causal, bf16.
  Q is clustered: 512 unit-norm centres per (b, h) (seed 3), a uniformly drawn
  centre index per position (seed 4), plus N(0, 0.05^2) noise (seed 5).
* ``fwd_bf16_L65536``    : 1, 8, 65536, 64, 1024, 8, 64, causal, bf16.
* ``fwdbwd_bf16_L16384`` : 2, 8, 16384, 64, 256, 4, 64, causal, bf16, with an
  upstream gradient dO ~ N(0, 1) from seed 2.

Unless stated otherwise Q and V come from seed 0 (Q first), rotations from
seed 1.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int
    d: int
    n_buckets: int
    n_rounds: int
    chunk: int
    causal: bool
    dtype: str  # "f32" or "bf16"
    clustered: bool = False
    backward: bool = False

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def describe(self) -> dict:
        return dataclasses.asdict(self)


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("fwd_f32_L1024", 1, 1, 1024, 64, 32, 1, 64, False, "f32"),
        Workload("fwd_bf16_L4096", 8, 8, 4096, 64, 64, 2, 64, True, "bf16"),
        Workload("fwd_bf16_L16384_clustered", 2, 8, 16384, 64, 256, 4, 64, False, "bf16",
                 clustered=True),
        Workload("fwd_bf16_L65536", 1, 8, 65536, 64, 1024, 8, 64, True, "bf16"),
        Workload("fwdbwd_bf16_L16384", 2, 8, 16384, 64, 256, 4, 64, True, "bf16",
                 backward=True),
    ]
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def gaussian(shape, seed: int, dtype: torch.dtype, generator: Optional[torch.Generator] = None):
    """N(0, 1) drawn in fp32 from ``seed`` (or a supplied generator), rounded once to dtype."""
    g = generator if generator is not None else _gen(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)


def rotations(n_rounds: int, d: int, n_buckets: int, seed: int, dtype: torch.dtype):
    """Per-round Gaussian rotations [n_rounds, d, n_buckets // 2] (empty when n_buckets == 1)."""
    half = n_buckets // 2
    return gaussian((n_rounds, d, half), seed, dtype)


def clustered_queries(B: int, H: int, L: int, d: int, n_centres: int, sigma: float,
                      seed_centres: int, seed_assign: int, seed_noise: int,
                      dtype: torch.dtype):
    """Cluster-structured queries: unit-norm centres plus isotropic Gaussian noise."""
    centres = torch.randn(B, H, n_centres, d, generator=_gen(seed_centres), dtype=torch.float32)
    centres = centres / centres.norm(dim=-1, keepdim=True)
    assign = torch.randint(0, n_centres, (B, H, L), generator=_gen(seed_assign))
    noise = torch.randn(B, H, L, d, generator=_gen(seed_noise), dtype=torch.float32) * sigma
    q = torch.gather(centres, 2, assign.unsqueeze(-1).expand(B, H, L, d)) + noise
    return q.to(dtype)


def make_inputs(w: Workload) -> Dict[str, torch.Tensor]:
    """The seeded CPU tensors of a named workload: Q, V, rot (and dO when it has a backward)."""
    dt = w.torch_dtype
    shape = (w.B, w.H, w.L, w.d)
    g0 = _gen(0)
    q = gaussian(shape, 0, dt, generator=g0)
    v = gaussian(shape, 0, dt, generator=g0)
    if w.clustered:
        q = clustered_queries(w.B, w.H, w.L, w.d, 512, 0.05, 3, 4, 5, dt)
        v = gaussian(shape, 0, dt)
    out = {"Q": q, "V": v, "rot": rotations(w.n_rounds, w.d, w.n_buckets, 1, dt)}
    if w.backward:
        out["dO"] = gaussian(shape, 2, dt)
    return out


def make_random(B: int, H: int, L: int, d: int, n_buckets: int, n_rounds: int,
                dtype: torch.dtype, seed: int, backward: bool = False) -> Dict[str, torch.Tensor]:
    """Small seeded Gaussian inputs of arbitrary shape for parity and edge-case tests."""
    shape = (B, H, L, d)
    g = _gen(seed)
    out = {
        "Q": gaussian(shape, 0, dtype, generator=g),
        "V": gaussian(shape, 0, dtype, generator=g),
        "rot": gaussian((n_rounds, d, n_buckets // 2), 0, dtype, generator=g),
    }
    if backward:
        out["dO"] = gaussian(shape, 0, dtype, generator=g)
    return out


# ---------------------------------------------------------------------------
# chunked feed-forward (the companion op of LSH attention in a Reformer layer)
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class FfnWorkload:
    name: str
    tokens: int   # B * L positions
    d_model: int  # H * d: 8 heads of 64
    d_ff: int     # 4 * d_model
    chunk: int    # positions per chunk

    def describe(self) -> dict:
        return dataclasses.asdict(self)


# ``ffn_bf16_L65536``: the L=65536 sequence of one batch element through the
# feed-forward of width 512 (8 heads of 64) and hidden width 2048, 8192
# positions per chunk.
FFN_WORKLOADS: Dict[str, FfnWorkload] = {
    w.name: w for w in [FfnWorkload("ffn_bf16_L65536", 65536, 512, 2048, 8192)]
}


def ffn_inputs(tokens: int, d_model: int, d_ff: int, seed: int = 20,
               dtype: torch.dtype = torch.bfloat16, backward: bool = False):
    """Seeded feed-forward inputs: X ~ N(0, 1) [tokens, d_model] (seed),
    W1 ~ N(0, 1/d_model) [d_ff, d_model] (seed + 1), b1 ~ N(0, 0.1^2) (seed + 2),
    W2 ~ N(0, 1/d_ff) [d_model, d_ff] (seed + 3), b2 ~ N(0, 0.1^2) (seed + 4),
    drawn in fp32 and rounded once to dtype; with backward, dY ~ N(0, 1)
    (seed + 5).  The weight scales keep every pre-activation and output near
    unit variance."""
    def draw(shape, s, scale):
        return (torch.randn(*shape, generator=_gen(s), dtype=torch.float32) * scale).to(dtype)
    out = {"X": draw((tokens, d_model), seed, 1.0),
           "W1": draw((d_ff, d_model), seed + 1, d_model ** -0.5),
           "b1": draw((d_ff,), seed + 2, 0.1),
           "W2": draw((d_model, d_ff), seed + 3, d_ff ** -0.5),
           "b2": draw((d_model,), seed + 4, 0.1)}
    if backward:
        out["dY"] = draw((tokens, d_model), seed + 5, 1.0)
    return out
