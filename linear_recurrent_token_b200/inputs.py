"""Seeded synthetic inputs for the mLSTM / retention workloads.

This module only draws random numbers and rounds them to the storage type; it
holds none of the recurrence's arithmetic.  Both the GPU path (through the
binding) and the fp64 oracle are fed from the same arrays it returns, so the
oracle sees exactly the values the kernels see (bf16 -> fp64 is exact).

Workloads (shapes and distributions; per-head sizes follow xLSTM 7B's
8 heads with qk_dim 2048 / v_dim 4096, i.e. 256 / 512 per head):

  0 tiny_fp32      B1 NH2 S64 DHQK=DHV=16 chunk16, fp32
  1 small_blockdiag B4 NH4 S512 DHQK=DHV=64 chunk64 num_blocks=2, bf16
  2 retention      B8 NH8 S2048 D64 chunk64, bf16, retention flag
  3 large_head     B1 NH8 S8192 DHQK256 DHV512 chunk64, bf16
  4 decode         B128 NH8 DHQK256 DHV512, 1024 decode steps, bf16 q/k/v, fp32 state

q, v ~ N(0,1); k ~ N(0,1)/sqrt(DHQK) (1/16 for DHQK=256); input-gate
pre-activation ~ N(0,1); forget-gate pre-activation ~ N(3,1).  Seeds:
numpy default_rng(1000 + workload index), draws in the order q, k, v, igate,
fgate.  The decode workload draws its initial C ~ N(0, 0.1^2) and
n ~ N(0, 0.1^2) (m = 0) from default_rng(1004), and the inputs of step t from
default_rng(2000 + t) in the order q, k, v, igate, fgate.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    NH: int
    S: int
    DHQK: int
    DHV: int
    chunk: int
    num_blocks: int
    dtype: str  # "f32" or "bf16": storage type of q, k, v, o and h
    retention: bool
    k_scale: float
    steps: int = 0  # decode workloads: number of sequential steps

    @property
    def dk(self) -> int:
        return self.DHQK // self.num_blocks

    @property
    def dv(self) -> int:
        return self.DHV // self.num_blocks

    def describe(self) -> str:
        if self.steps:
            return (f"{self.name}: B{self.B} NH{self.NH} DHQK{self.DHQK} DHV{self.DHV} "
                    f"{self.steps} steps {self.dtype} q/k/v fp32 state")
        return (f"{self.name}: B{self.B} NH{self.NH} S{self.S} DHQK{self.DHQK} DHV{self.DHV} "
                f"chunk{self.chunk} nb{self.num_blocks} {self.dtype}"
                + (" retention" if self.retention else ""))


WORKLOADS = [
    Workload(0, "tiny_fp32", 1, 2, 64, 16, 16, 16, 1, "f32", False, 1.0 / 4.0),
    Workload(1, "small_blockdiag", 4, 4, 512, 64, 64, 64, 2, "bf16", False, 1.0 / 8.0),
    Workload(2, "retention", 8, 8, 2048, 64, 64, 64, 1, "bf16", True, 1.0 / 8.0),
    Workload(3, "large_head", 1, 8, 8192, 256, 512, 64, 1, "bf16", False, 1.0 / 16.0),
    Workload(4, "decode", 128, 8, 1, 256, 512, 64, 1, "bf16", False, 1.0 / 16.0, steps=1024),
]


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp64 draws to the storage type; returned as float32 holding exact values."""
    x32 = np.asarray(x, dtype=np.float32)
    if dtype == "f32":
        return x32
    if dtype == "bf16":
        import torch
        return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).to(torch.float32).numpy()
    raise ValueError(dtype)


def _draw(rng, shape, dtype, scale=1.0, mean=0.0):
    return round_to(rng.standard_normal(shape) * scale + mean, dtype)


def forward_inputs(w: Workload, seed: int | None = None, S: int | None = None, B: int | None = None):
    """Inputs of a chunkwise forward: dict of float32 numpy arrays (exact storage values).

    Keys: q, k [B,NH,S,DHQK]; v [B,NH,S,DHV]; igate, fgate [B,NH,S] (always fp32).
    ``S``/``B`` override the sequence length / batch (same distributions).
    """
    rng = np.random.default_rng(1000 + w.index if seed is None else seed)
    B = w.B if B is None else B
    S = w.S if S is None else S
    q = _draw(rng, (B, w.NH, S, w.DHQK), w.dtype)
    k = _draw(rng, (B, w.NH, S, w.DHQK), w.dtype, scale=w.k_scale)
    v = _draw(rng, (B, w.NH, S, w.DHV), w.dtype)
    ig = _draw(rng, (B, w.NH, S), "f32")
    fg = _draw(rng, (B, w.NH, S), "f32", mean=3.0)
    return dict(q=q, k=k, v=v, igate=ig, fgate=fg)


def decode_initial_state(w: Workload, seed: int | None = None, B: int | None = None):
    """Initial (C, n, m) of the decode workload: C, n ~ N(0, 0.1^2), m = 0 (fp32)."""
    rng = np.random.default_rng(1000 + w.index if seed is None else seed)
    B = w.B if B is None else B
    C = _draw(rng, (B, w.NH, w.num_blocks, w.dv, w.dk), "f32", scale=0.1)
    n = _draw(rng, (B, w.NH, w.num_blocks, w.dk), "f32", scale=0.1)
    m = np.zeros((B, w.NH), dtype=np.float32)
    return C, n, m


def decode_step_inputs(w: Workload, t: int, B: int | None = None):
    """Inputs of decode step t: q, k [B,NH,DHQK]; v [B,NH,DHV]; igate, fgate [B,NH]."""
    rng = np.random.default_rng(2000 + t)
    B = w.B if B is None else B
    q = _draw(rng, (B, w.NH, w.DHQK), w.dtype)
    k = _draw(rng, (B, w.NH, w.DHQK), w.dtype, scale=w.k_scale)
    v = _draw(rng, (B, w.NH, w.DHV), w.dtype)
    ig = _draw(rng, (B, w.NH), "f32")
    fg = _draw(rng, (B, w.NH), "f32", mean=3.0)
    return dict(q=q, k=k, v=v, igate=ig, fgate=fg)


def decode_sequence_inputs(w: Workload, steps: int, B: int | None = None):
    """Steps 0..steps-1 stacked along a sequence axis: q [B,NH,steps,DHQK] etc."""
    per = [decode_step_inputs(w, t, B) for t in range(steps)]
    return {key: np.stack([p[key] for p in per], axis=2) for key in per[0]}


# Gated DeltaNet-2 workloads (burn-gdn2 config.rs defaults: 16 heads of 128, value head 128,
# chunk 64): a prefill batch and a decode batch (one token per sequence, state in place).
@dataclasses.dataclass(frozen=True)
class Gdn2Workload:
    name: str
    B: int
    H: int
    T: int
    K: int
    V: int
    chunk: int
    dtype: str

    def describe(self) -> str:
        return f"{self.name}: B{self.B} H{self.H} T{self.T} K{self.K} V{self.V} chunk{self.chunk} {self.dtype}"


GDN2_WORKLOADS = [
    Gdn2Workload("gdn2_prefill", 8, 16, 2048, 128, 128, 64, "bf16"),
    Gdn2Workload("gdn2_decode", 256, 16, 1, 128, 128, 64, "bf16"),
]


def gdn2_inputs(B, H, T, K, V, dtype, seed, with_state=True):
    """Inputs of a GDN-2 call: q, v ~ N(0,1); k ~ N(0,1) scaled to unit length per token (the
    usual key normalisation, done by the caller); log decay g = -exp(N(-3, 1)) (alpha near
    0.95 on average, a few channels much lower); erase and write gates b, w ~ U(0,1); S0 ~
    N(0, 0.1^2).  Dict of float32 numpy arrays holding the exact stored values."""
    rng = np.random.default_rng(seed)
    q = _draw(rng, (B, H, T, K), dtype)
    kr = rng.standard_normal((B, H, T, K))
    k = round_to(kr / np.maximum(np.linalg.norm(kr, axis=-1, keepdims=True), 1e-12), dtype)
    v = _draw(rng, (B, H, T, V), dtype)
    g = round_to(-np.exp(rng.standard_normal((B, H, T, K)) - 3.0), "f32")
    b = round_to(rng.uniform(0, 1, (B, H, T, K)), "f32")
    w = round_to(rng.uniform(0, 1, (B, H, T, V)), "f32")
    S0 = _draw(rng, (B, H, K, V), "f32", scale=0.1) if with_state else None
    return dict(q=q, k=k, v=v, g=g, b=b, w=w, S0=S0)
