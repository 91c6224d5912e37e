"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws numbers: it holds none of the layer's arithmetic, so
both the CUDA path and the CPU oracle can take their inputs from it. It uses
numpy only (PCG64 streams, one per tensor, derived from the workload seed).

Weights are drawn as a pool of float32 128x128 blocks, N(0, 1/fan_in), plus
per-expert maps from block position to pool entry. A block of the pool is a
block of the weight matrix, so 128x128 block quantisation of the pool is the
quantisation of every expert. Small workloads use a pool with one entry per
block position (every block distinct); the V3-shape workloads use a pool of a
few thousand blocks so that 11 GB of weights can be built in seconds.
"""
from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    H: int            # hidden size
    N: int            # routed experts
    K: int            # routed experts per token
    I: int            # expert intermediate size (routed and shared)
    bias_range: float = 0.0      # bias ~ U(-r, r); 0 means bias = 0
    gamma: float = 1e-3          # bias update step
    steps: int = 1               # forward + update steps of the workload
    outlier_frac: float = 0.0    # fraction of channels scaled by outlier_scale
    outlier_scale: float = 1.0
    zipf_s: float = 0.0          # skewed gate rows: logit means alpha * r^-s
    zipf_alpha: float = 0.0
    pool13: int = 0              # 0: one pool entry per block position
    pool2: int = 0
    seed: int = 0

    @property
    def E(self) -> int:          # expert groups incl. the shared expert
        return self.N + 1

    def flops_per_token(self) -> float:
        """Algorithmic FLOPs of the expert FFNs for one token (K routed + 1
        shared expert, SwiGLU: up/gate 2*H*2I, down 2*I*H)."""
        return (self.K + 1) * (2.0 * self.H * 2 * self.I + 2.0 * self.I * self.H)


WORKLOADS = {
    "tiny": Workload("tiny", T=64, H=256, N=16, K=4, I=128, bias_range=0.1),
    "v3_prefill": Workload("v3_prefill", T=4096, H=7168, N=256, K=8, I=2048,
                           pool13=4096, pool2=2048),
    "skewed": Workload("skewed", T=8192, H=7168, N=256, K=8, I=2048, steps=50,
                       zipf_s=1.2, zipf_alpha=4.0, pool13=4096, pool2=2048),
    "large_prefill": Workload("large_prefill", T=32768, H=7168, N=256, K=8,
                              I=2048, bias_range=0.05, outlier_frac=0.01,
                              outlier_scale=20.0, pool13=4096, pool2=2048),
    "decode": Workload("decode", T=128, H=7168, N=256, K=8, I=2048,
                       bias_range=0.05, pool13=4096, pool2=2048),
    # profiler-sized case: V3 expert shape and ~128 tokens per expert as in
    # v3_prefill, but 32 routed experts, so 1.45 GB of weights (> L2, small
    # enough for multi-pass counter captures)
    "profile_small": Workload("profile_small", T=512, H=7168, N=32, K=8, I=2048,
                              pool13=4096, pool2=2048),
}


def _rng(w: Workload, stream: int) -> np.random.Generator:
    return np.random.default_rng([w.seed, stream])


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even.
    Inputs must be finite."""
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = bits + np.uint32(0x7FFF) + ((bits >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def skew_direction(w: Workload) -> np.ndarray:
    d = _rng(w, 7).standard_normal(w.H)
    return (d / np.linalg.norm(d)).astype(np.float32)


def outlier_channels(w: Workload) -> np.ndarray:
    n_out = int(round(w.outlier_frac * w.H))
    return np.sort(_rng(w, 8).choice(w.H, size=n_out, replace=False))


def make_x(w: Workload, step: int = 0, rows: int | None = None) -> np.ndarray:
    """Layer input x [T, H] as bf16 bit patterns (uint16).

    x ~ N(0,1); the skewed workload adds a unit direction d to every token;
    the outlier workload multiplies a fixed 1% of channels by 20 (before the
    bf16 rounding). `step` selects a fresh batch for multi-step workloads.
    """
    t = w.T if rows is None else rows
    x = _rng(w, 100 + step).standard_normal((t, w.H), dtype=np.float32)
    if w.zipf_s > 0:
        x += skew_direction(w)[None, :]
    if w.outlier_frac > 0:
        x[:, outlier_channels(w)] *= np.float32(w.outlier_scale)
    return f32_to_bf16_bits(x)


def make_gate_w(w: Workload) -> np.ndarray:
    """Expert centroids e_i [N, H] float32, N(0, 1/H).

    Skewed workload: e_i += alpha * r_i^-s * d, with r_i a seeded permutation
    of the ranks 1..N, so the mean logit of expert i is about alpha * r_i^-s.
    """
    g = _rng(w, 2).standard_normal((w.N, w.H), dtype=np.float32)
    g *= np.float32(1.0 / np.sqrt(w.H))
    if w.zipf_s > 0:
        ranks = _rng(w, 9).permutation(w.N) + 1
        amp = (w.zipf_alpha * ranks.astype(np.float64) ** (-w.zipf_s)).astype(np.float32)
        g += amp[:, None] * skew_direction(w)[None, :]
    return g.astype(np.float32)


def make_bias(w: Workload) -> np.ndarray:
    if w.bias_range == 0.0:
        return np.zeros(w.N, np.float32)
    return _rng(w, 3).uniform(-w.bias_range, w.bias_range, w.N).astype(np.float32)


@dataclasses.dataclass
class WeightPool:
    pool13: np.ndarray     # [P13, 128, 128] float32, N(0, 1/H)
    pool2: np.ndarray      # [P2, 128, 128] float32, N(0, 1/I)
    slot_gate: np.ndarray  # [E, I/128, H/128] int64 pool13 index
    slot_up: np.ndarray    # [E, I/128, H/128]
    slot_down: np.ndarray  # [E, H/128, I/128] pool2 index


def make_weight_pool(w: Workload) -> WeightPool:
    ib, hb = w.I // 128, w.H // 128
    n13 = w.E * 2 * ib * hb
    n2 = w.E * hb * ib
    r = _rng(w, 4)
    p13 = w.pool13 or n13
    p2 = w.pool2 or n2
    pool13 = r.standard_normal((p13, 128, 128), dtype=np.float32)
    pool13 *= np.float32(1.0 / np.sqrt(w.H))
    pool2 = r.standard_normal((p2, 128, 128), dtype=np.float32)
    pool2 *= np.float32(1.0 / np.sqrt(w.I))
    if w.pool13:
        s13 = r.integers(0, p13, size=n13)
    else:
        s13 = r.permutation(n13)
    if w.pool2:
        s2 = r.integers(0, p2, size=n2)
    else:
        s2 = r.permutation(n2)
    s13 = s13.reshape(w.E, 2, ib, hb)
    return WeightPool(pool13, pool2, s13[:, 0].copy(), s13[:, 1].copy(),
                      s2.reshape(w.E, hb, ib))
