"""Shared set-up for the GPU parity tests: one seeded workload, its oracle
inputs and its device tensors, plus the comparison rules.

Parity tiers (fixed by the benchmark spec of the method):
  * bit-exact: x codes and scales, counts, offsets, permutation, bias update;
  * routing ids may differ only for tokens whose oracle gap between the K-th
    and (K+1)-th biased score is below 1e-5 of the K-th score; for those
    tokens the GPU's choice is taken and everything downstream recomputed;
  * layer output: max_j |y_gpu - y_oracle| <= 2e-2 * RMS(y_oracle[t, :]) per row.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I

TIE_REL = 1e-5
Y_TOL = 2e-2


@dataclasses.dataclass
class Case:
    w: I.Workload
    x_bits: np.ndarray
    x: np.ndarray          # float32 values of the bf16 input
    gate_w: np.ndarray
    bias: np.ndarray
    pool: I.WeightPool
    ew: O.ExpertWeights


def make_case(w: I.Workload) -> Case:
    xb = I.make_x(w)
    pool = I.make_weight_pool(w)
    ew = O.ExpertWeights(pool.pool13, pool.pool2, pool.slot_gate, pool.slot_up, pool.slot_down)
    return Case(w, xb, I.bf16_bits_to_f32(xb), I.make_gate_w(w), I.make_bias(w), pool, ew)


def x_to_device(x_bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device).view(torch.bfloat16)


def near_tie_tokens(score: np.ndarray, k: int) -> np.ndarray:
    srt = -np.sort(-score, axis=1)
    if score.shape[1] <= k:
        return np.zeros(score.shape[0], bool)
    gap = srt[:, k - 1] - srt[:, k]
    return gap < TIE_REL * np.abs(srt[:, k - 1])


def reconcile_ids(gpu_ids: np.ndarray, oracle_ids: np.ndarray, score: np.ndarray, k: int):
    """Checks the GPU routing against the oracle's and returns the ids the
    oracle must use downstream (its own, except on near-tie tokens)."""
    near = near_tie_tokens(score, k)
    gs = np.sort(gpu_ids, axis=1)
    os_ = np.sort(oracle_ids, axis=1)
    differ = np.any(gs != os_, axis=1)
    bad = differ & ~near
    assert not bad.any(), f"routing differs on {bad.sum()} tokens without a near tie: {np.nonzero(bad)[0][:10]}"
    # on near-tie tokens the GPU choice must still be a valid top-K up to the tolerance
    for t in np.nonzero(differ)[0]:
        kth = -np.sort(-score[t])[k - 1]
        assert np.all(score[t, gpu_ids[t]] >= kth - TIE_REL * abs(kth))
        assert len(set(gpu_ids[t])) == k
    # order: biased score descending, unless two chosen scores are within the tolerance
    for t in np.nonzero(~differ)[0]:
        if not np.array_equal(gpu_ids[t], oracle_ids[t]):
            sc = score[t, oracle_ids[t]]
            assert np.min(np.abs(np.diff(sc))) < TIE_REL * np.abs(sc).max(), t
    # downstream the GPU's ids are used: their set equals the oracle's except
    # on near-tie tokens, and their order differs only between near-equal scores
    return gpu_ids.astype(np.int32), int(differ.sum()), int(near.sum())


def check_rows(y_gpu: np.ndarray, y_ref: np.ndarray, tol: float = Y_TOL) -> float:
    rms = np.sqrt(np.mean(y_ref ** 2, axis=1))
    err = np.max(np.abs(y_gpu - y_ref), axis=1)
    worst = float(np.max(err / rms))
    assert np.all(err <= tol * rms), f"worst row error {worst:.4g} x RMS"
    return worst


def bf16_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()
