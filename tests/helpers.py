"""Shared set-up for the GPU parity tests: one seeded workload, its oracle
inputs and its device tensors, plus the comparison rules.

Parity tiers (fixed by the benchmark spec of the method):
  * bit-exact: x codes and scales, counts, offsets, permutation, bias update;
  * routing ids may differ only for tokens whose oracle gap between the K-th
    and (K+1)-th biased score is below 1e-5 of the K-th score; for those
    tokens the GPU's choice is taken and everything downstream recomputed;
  * layer output: max_j |y_gpu - y_oracle| <= 2e-2 * RMS(y_oracle[t, :]) per row;
  * stage by stage (expert_path_parity): the h codes, the bf16 expert
    outputs and y are the oracle's roundings of its float64 values, except
    on near ties (a value within the fp32 error of a rounding midpoint),
    where the GPU's choice must be one of the two correct ones and the
    oracle continues with it, as for the ids.
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


# ---------------------------------------------------------------- expert path
#
# The expert outputs Y are bf16 ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load
# Balancing...", section V, Figure 6), each the rounding of an fp32 sum on the
# GPU and of a float64 sum in the oracle. Where a float64 sum lies within the
# fp32 accumulation error of a midpoint between two bf16 neighbours, either
# neighbour is a correct rounding: the near-tie rule of the ids, applied to
# the bf16 decision. The accumulation error is the one pinned for the down
# GEMM on identical operands: 1e-5 of the row's RMS.
ACC_REL = 1e-5


def bf16_choices(y64: np.ndarray, tol) -> tuple[np.ndarray, np.ndarray]:
    """The range of bf16 values a correct kernel may give for float64 sums
    y64 known to within tol (per row): rounding is monotonic, so any sum in
    [y64 - tol, y64 + tol] rounds into [round(y64 - tol), round(y64 + tol)].
    The two ends are equal unless a midpoint lies within tol."""
    return O.round_bf16(y64 - tol), O.round_bf16(y64 + tol)


def check_bf16(got: np.ndarray, y64: np.ndarray, what: str, rel: float = ACC_REL) -> int:
    """got (bf16 values) must be the bf16 rounding of a sum within rel x the
    row's RMS of y64: the oracle's own rounding, or on a near midpoint the
    other neighbour. Returns how many differ from the oracle's own rounding."""
    tol = rel * np.sqrt(np.mean(y64 ** 2, axis=1, keepdims=True))
    lo, hi = bf16_choices(y64, tol)
    ok = (got >= lo) & (got <= hi)
    bad = np.argwhere(~ok)
    assert ok.all(), (f"{what}: {len(bad)} values are not a rounding of the float64 sum, "
                      f"first {bad[:5].tolist()}")
    return int(np.sum(got != O.round_bf16(y64)))


# h codes: the GPU's G and U are fp32 sums (promoted per 128), h uses the
# hardware exp and reciprocal; against float64 they differ by far less than
# 1e-5 of the tile's amax (the value that scales to 448)
ACC_H = 1e-5


def check_h_codes(hq_g, hs_g, h64) -> tuple[int, int]:
    """The GPU's 1x128 codes of h against the oracle's float64 h: each tile's
    scale is the oracle's up to the fp32 error of the tile's amax (a near
    tie of the amax), and each code, with that scale, is the E4M3 rounding of
    a value within ACC_H x 448 of h * scale: the oracle's own code, or on a
    near midpoint its neighbour. Returns (codes equal to the oracle's own
    rounding with the GPU's scale, codes)."""
    hq_o, hs_o = O.quantize_1x128(h64.astype(np.float32))
    assert np.allclose(hs_g, hs_o, rtol=2e-5, atol=0)
    v = h64 * np.repeat(hs_g.astype(np.float64), 128, axis=1)
    tol = ACC_H * 448.0
    lo = O.e4m3_decode(O.e4m3_encode(v - tol))
    hi = O.e4m3_decode(O.e4m3_encode(v + tol))
    got = O.e4m3_decode(hq_g)
    ok = (got >= lo) & (got <= hi)
    assert ok.all(), f"{int((~ok).sum())} h codes are not a rounding of h * scale"
    own = O.e4m3_encode((h64.astype(np.float32) * np.repeat(hs_g, 128, axis=1)).astype(np.float32))
    return int(np.sum(hq_g == own)), int(hq_g.size)


def expert_path_parity(w, case, layer, y_gpu, use_ids, tokens) -> dict:
    """Parity of the expert path for the rows of `tokens` against the oracle,
    with the GPU's routing (use_ids, already reconciled). Every decision that
    floating point makes into an integer is the oracle's own unless it is a
    near tie, where the GPU's choice is checked to be one of the correct ones
    and the oracle continues with it (as the ids' near-tie rule does):

      up stage    the GPU's h codes and scales of every (token, expert) row
                  against the oracle's float64 h on the same x codes
                  (check_h_codes; the x codes are compared bit for bit
                  elsewhere);
      down stage  the GPU's bf16 Y rows against the oracle's float64 down
                  stage on those h codes, rounded to bf16 (check_bf16);
      combine     the GPU's y against the rounding of the oracle's float64
                  combine of those Y rows (check_bf16), and within 2e-2 of
                  each row's RMS (the layer output's tier).
    Returns counts of the near-tie choices taken and the worst row error (in
    RMS units) against the oracle's y."""
    tokens = np.asarray(tokens)
    L = layer.layout
    token_row = layer.view("token_row", torch.int32, (w.T, w.K)).cpu().numpy()
    h_q = layer.view("h_q", torch.uint8, (L.rows_total, w.I))
    h_s = layer.view("h_s", torch.float32, (L.rows_total, w.I // 128))
    y_rows = layer.view("y_rows", torch.bfloat16, (L.rows_total, w.H))
    xq, xs = O.quantize_1x128(case.x[tokens])
    s = O.sigmoid(O.gate_logits(case.x[tokens], case.gate_w))
    sub_ids = use_ids[tokens]
    sel = np.take_along_axis(s, sub_ids.astype(np.int64), axis=1)
    gates = sel / np.sum(sel, axis=1, keepdims=True)
    n_tok = len(tokens)
    yr = np.zeros((n_tok, w.K, w.H))
    stats = {"y_flips": 0, "h_equal": 0, "h_codes": 0}
    experts = [int(e) for e in np.unique(sub_ids)] + [w.N]
    for e in experts:
        if e == w.N:
            rr, kk = np.arange(n_tok), None
            rows = L.routed_cap + tokens
        else:
            rr, kk = np.nonzero(sub_ids == e)
            rows = token_row[tokens[rr], kk]
        idx = torch.from_numpy(rows.astype(np.int64)).cuda()
        hq_g = h_q[idx].cpu().numpy()
        hs_g = h_s[idx].cpu().numpy()
        yg = y_rows[idx].float().cpu().numpy().astype(np.float64)
        wg, wu, wd = case.ew.dequantised(e)
        h64, _, _ = O.expert_up_q(xq[rr], xs[rr], wg, wu)
        eq, n = check_h_codes(hq_g, hs_g, h64)
        stats["h_equal"] += eq
        stats["h_codes"] += n
        stats["y_flips"] += check_bf16(yg, O.expert_down_q(hq_g, hs_g, wd), f"Y of expert {e}")
        if kk is None:
            ysh = yg
        else:
            yr[rr, kk] = yg
    y_ref = O.combine(ysh, yr, sub_ids, gates)
    stats["y_combine_flips"] = check_bf16(y_gpu, y_ref, "combine")
    stats["worst_row"] = check_rows(y_gpu, y_ref)
    stats["y_ref"] = y_ref
    return stats
