"""CPU oracle for the DeepSeekMoE layer forward with FP8 fine-grained scaling.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously-correct
definition that the CUDA path is checked against. Only the tests, the smoke
check and the CPU-baseline leg of the benchmark may import it; the library
never does, and the oracle imports nothing from the library.

Arithmetic is float64 except where the method itself fixes a narrower type:
the E4M3 codes, the float32 tile scales and the float32 routing bias.

Sources (web pages on the DeepSeek-V3 technical report), cited by tag:
  [Explained]  "DeepSeek-V3, explained" (vibeengines.com), the numbered recipe
               and the symbol notes under it.
  [Dissection] "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
               Multi-Token Prediction, and FP8 Training at 671B Scale"
               (trishampatil.com); section III (routing equations, bias
               controller) and section V (FP8 details).
  [Deepforge]  "DeepSeek-V3 Technical Report" (deepforge.srivtx.xyz);
               "Per-tile FP8 scaling", "Balancing without a balance loss"
               and "Build it yourself".

Readings taken where the pages are silent (each is listed in the design
notes with its reason):
  * E4M3 is the OCP E4M3FN format, round-to-nearest-even, saturating to
    +-448; zero keeps its sign.
  * Tile scale = fp32(448 / amax) with an IEEE divide; codes are
    e4m3(fp32(x * scale)); an all-zero tile gets scale 1.
  * Top-K ties go to the lower expert id; output order is biased score
    descending.
  * Load target is the mean T*K/N, compared in integers as T*K - N*c_i.
  * Expert FFN outputs Y are BF16 (the FP8 GEMMs give BF16 outputs), each
    rounded once from its float64 sum; the combine sums them in float64,
    shared expert first, then routed experts by ascending id, and the layer
    output y is that float64 sum (the kernels round it once more, to bf16).
  * No residual add; no routed scaling factor.
  * Node-limited routing ranks groups by the sum of their K/M highest
    *biased* scores (the selection side, as [Deepforge] ranks experts by
    s_i + b_i; [Explained] says "affinities"); group ties go to the lower id.
  * Sequence balance statistics: f_i is the load normalised so a perfectly
    even split gives 1; P_i averages s_i / sum_j s_j over the sequence.

parity pins: every function here is pinned by a test under tests/ against a
closed form, a worked example, an invariant, a library routine or brute
force; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
TILE = 128


# ---------------------------------------------------------------------------
# E4M3 codec  ([Deepforge] "FP8 training, from first principles" and
# "Per-tile FP8 scaling": 4 exponent bits, 3 mantissa bits, largest 448)
# ---------------------------------------------------------------------------

def _build_decode_table() -> np.ndarray:
    """Value of each of the 256 byte codes, from the bit layout.

    Layout s eeee mmm, exponent bias 7. Exponent field 0 is subnormal
    (m/8 * 2^-6); field 15 with mantissa 7 is NaN (E4M3FN has no infinity).
    """
    table = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if (code >> 7) & 1 else 1.0
        exp_field = (code >> 3) & 0xF
        man_field = code & 0x7
        if exp_field == 0xF and man_field == 0x7:
            table[code] = np.nan
        elif exp_field == 0:
            table[code] = sign * (man_field / 8.0) * 2.0 ** (1 - 7)
        else:
            table[code] = sign * (1.0 + man_field / 8.0) * 2.0 ** (exp_field - 7)
    return table


E4M3_DECODE = _build_decode_table()
# positive finite values, codes 0x00 .. 0x7E, ascending
_E4M3_POS = E4M3_DECODE[:0x7F].copy()


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> float64 values."""
    return E4M3_DECODE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """float values -> uint8 E4M3 codes: nearest value, ties to even, saturate.

    The nearest representable magnitude is found by bracketing |v| between two
    adjacent positive codes; on an exact midpoint the code with the even
    mantissa (low bit 0) wins. Magnitudes above 448 (and +-inf) become 448.
    NaN becomes 0x7F. The sign bit is copied, so -0.0 encodes to 0x80.
    """
    v = np.asarray(v, dtype=np.float64)
    nan = np.isnan(v)
    neg = np.signbit(v)
    a = np.minimum(np.abs(np.where(nan, 0.0, v)), E4M3_MAX)
    hi = np.searchsorted(_E4M3_POS, a, side="left")  # first code with value >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(take_hi, hi, lo).astype(np.uint8)
    codes = np.where(neg, mag | 0x80, mag).astype(np.uint8)
    codes = np.where(nan, np.uint8(0x7F), codes).astype(np.uint8)
    return codes


# ---------------------------------------------------------------------------
# Fine-grained quantisation ([Explained] recipe step 7; [Dissection] section V
# "Four details", item 1; [Deepforge] "Per-tile FP8 scaling" formula:
# scale = max_fp8 / amax, X_fp8 = round(X * scale), X_hat = X_fp8 / scale)
# ---------------------------------------------------------------------------

def _tile_scale(amax_f32: np.ndarray) -> np.ndarray:
    """fp32(448 / amax) with IEEE float32 division; 1.0 for an all-zero tile."""
    amax_f32 = np.asarray(amax_f32, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = np.float32(E4M3_MAX) / amax_f32
    return np.where(amax_f32 > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_1x128(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Online activation quantisation, one scale per row per 128 columns.

    x: float array [rows, cols] (cols a multiple of 128), taken as float32.
    Returns codes uint8 [rows, cols] and scales float32 [rows, cols/128]
    (the multiplier 448/amax, as the per-tile formula stores it).
    """
    x = np.asarray(x, dtype=np.float32)
    rows, cols = x.shape
    assert cols % TILE == 0
    xt = x.reshape(rows, cols // TILE, TILE)
    amax = np.max(np.abs(xt), axis=2)
    scale = _tile_scale(amax)
    with np.errstate(invalid="ignore", over="ignore"):
        prod = (xt * scale[:, :, None]).astype(np.float32)  # one float32 multiply
    codes = e4m3_encode(prod).reshape(rows, cols)
    return codes, scale


def quantize_128x128(w: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Weight quantisation, one scale per 128x128 block.

    w: float array [rows, cols], both multiples of 128, taken as float32.
    Returns codes uint8 [rows, cols] and scales float32 [rows/128, cols/128].
    """
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    assert rows % TILE == 0 and cols % TILE == 0
    wb = w.reshape(rows // TILE, TILE, cols // TILE, TILE)
    amax = np.max(np.abs(wb), axis=(1, 3))
    scale = _tile_scale(amax)
    with np.errstate(invalid="ignore", over="ignore"):
        prod = (wb * scale[:, None, :, None]).astype(np.float32)
    codes = e4m3_encode(prod).reshape(rows, cols)
    return codes, scale


def dequantize_1x128(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """X_hat = X_fp8 / scale, in float64."""
    rows, cols = codes.shape
    v = e4m3_decode(codes).reshape(rows, cols // TILE, TILE)
    return (v / np.asarray(scales, np.float64)[:, :, None]).reshape(rows, cols)


def dequantize_128x128(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    rows, cols = codes.shape
    v = e4m3_decode(codes).reshape(rows // TILE, TILE, cols // TILE, TILE)
    return (v / np.asarray(scales, np.float64)[:, None, :, None]).reshape(rows, cols)


# ---------------------------------------------------------------------------
# Routing ([Dissection] section III "The mechanism": s = Sigmoid(u^T e_i),
# g' = s if s + b in TopK(s + b, K) else 0, g = g' / sum g';
# [Explained] recipe step 4 and the notes on b_i and K_r)
# ---------------------------------------------------------------------------

def gate_logits(x: np.ndarray, gate_w: np.ndarray) -> np.ndarray:
    """z[t, i] = u_t . e_i in float64 (gating stays in high precision,
    [Explained] recipe step 7; [Dissection] section V item 4)."""
    return np.asarray(x, np.float64) @ np.asarray(gate_w, np.float64).T


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))


def route(x: np.ndarray, gate_w: np.ndarray, bias: np.ndarray, k: int):
    """Sigmoid affinity, biased top-K selection, unbiased normalised gates.

    Returns (ids int32 [T,K], gates float64 [T,K], s float64 [T,N],
    score float64 [T,N]) with ids ordered by biased score descending and
    ties broken toward the lower expert id.
    """
    s = sigmoid(gate_logits(x, gate_w))
    score = s + np.asarray(bias, np.float32).astype(np.float64)
    # stable sort of -score: equal scores keep ascending expert id
    order = np.argsort(-score, axis=1, kind="stable")
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(s, ids, axis=1)
    gates = sel / np.sum(sel, axis=1, keepdims=True)
    return ids, gates, s, score


def route_grouped(x: np.ndarray, gate_w: np.ndarray, bias: np.ndarray, k: int,
                  n_groups: int, topk_groups: int):
    """Node-limited routing ([Explained] recipe step 5; [Deepforge]
    "Balancing without a balance loss"): the N routed experts are split into
    n_groups contiguous groups (the nodes that hold them); a group's score is
    the sum of its k / topk_groups highest biased scores s_i + b_i; only the
    topk_groups best groups are eligible (ties to the lower group id), and
    the K experts are the biased top-K among the eligible ones, as in route().

    Returns (ids, gates, s, score, group_score [T, n_groups]).
    """
    s = sigmoid(gate_logits(x, gate_w))
    score = s + np.asarray(bias, np.float32).astype(np.float64)
    t_count, n = score.shape
    size, per_group = n // n_groups, k // topk_groups
    assert size * n_groups == n and per_group * topk_groups == k and per_group <= size
    grouped = score.reshape(t_count, n_groups, size)
    best = -np.sort(-grouped, axis=2)[:, :, :per_group]
    group_score = best.sum(axis=2)
    chosen = np.argsort(-group_score, axis=1, kind="stable")[:, :topk_groups]
    eligible = np.zeros((t_count, n_groups), dtype=bool)
    np.put_along_axis(eligible, chosen, True, axis=1)
    masked = np.where(np.repeat(eligible, size, axis=1), score, -np.inf)
    order = np.argsort(-masked, axis=1, kind="stable")
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(s, ids, axis=1)
    gates = sel / np.sum(sel, axis=1, keepdims=True)
    return ids, gates, s, score, group_score


def balance_stats(s: np.ndarray, ids: np.ndarray, k: int, seq_len: int, alpha: float):
    """Complementary sequence-wise balance statistics ([Dissection] section
    III, "a complementary sequence-wise balance loss", and [Explained] recipe
    step 4): over the tokens of each sequence (consecutive runs of seq_len
    tokens; the last may be shorter),
      f_i = N / (K * T_seq) * #{(t, k): ids[t, k] = i}   (normalised load)
      P_i = (1 / T_seq) * sum_t s[t, i] / sum_j s[t, j]  (mean gate mass)
      L   = alpha * sum_i f_i * P_i.
    s are the unbiased affinities of all N routed experts.

    Returns f [S, N], P [S, N], loss [S] in float64.
    """
    s = np.asarray(s, np.float64)
    ids = np.asarray(ids)
    t_count, n = s.shape
    n_seq = -(-t_count // seq_len)
    f = np.zeros((n_seq, n))
    p = np.zeros((n_seq, n))
    loss = np.zeros(n_seq)
    for q in range(n_seq):
        lo, hi = q * seq_len, min(t_count, (q + 1) * seq_len)
        t_seq = hi - lo
        counts = np.bincount(ids[lo:hi].ravel(), minlength=n)
        f[q] = n * counts / (k * t_seq)
        p[q] = np.sum(s[lo:hi] / np.sum(s[lo:hi], axis=1, keepdims=True), axis=0) / t_seq
        loss[q] = alpha * np.sum(f[q] * p[q])
    return f, p, loss


def expert_counts(ids: np.ndarray, n_experts: int) -> np.ndarray:
    """c_i = number of tokens of this batch that selected expert i
    ([Dissection] section III "Measure per-expert load this step")."""
    return np.bincount(np.asarray(ids).ravel(), minlength=n_experts).astype(np.int32)


def permutation(ids: np.ndarray, n_experts: int):
    """Expert-major order of the (token, slot) pairs: expert ascending, then
    token ascending. Every pair is kept (no token dropping, [Explained]
    recipe step 5).

    Returns offsets int32 [N+1] (exclusive scan of the counts), tokens int32
    [T*K] (token of each position), rank int32 [T,K] (position of pair
    (t, k) inside its expert's segment).
    """
    ids = np.asarray(ids)
    t_count, k = ids.shape
    counts = expert_counts(ids, n_experts)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    tokens = np.empty(t_count * k, dtype=np.int32)
    rank = np.empty((t_count, k), dtype=np.int32)
    fill = np.zeros(n_experts, dtype=np.int64)
    for t in range(t_count):
        for j in range(k):
            e = ids[t, j]
            tokens[offsets[e] + fill[e]] = t
            rank[t, j] = fill[e]
            fill[e] += 1
    return offsets.astype(np.int32), tokens, rank


# ---------------------------------------------------------------------------
# Bias controller ([Dissection] section III "How the bias is set";
# [Explained] recipe step 4: overloaded b_i -= gamma, underloaded b_i += gamma)
# ---------------------------------------------------------------------------

def update_bias(bias: np.ndarray, counts: np.ndarray, t_count: int, k: int,
                gamma: float) -> np.ndarray:
    """b_i <- fp32(b_i + gamma * sign(mean load - c_i)).

    The mean load T*K/N is compared without division: sign(T*K - N*c_i).
    Exactly at the mean the bias does not move. float32 arithmetic, as the
    bias is stored.
    """
    bias = np.asarray(bias, np.float32)
    n = bias.shape[0]
    delta = np.sign(np.int64(t_count) * np.int64(k)
                    - np.int64(n) * np.asarray(counts, np.int64))
    step = (delta.astype(np.float32) * np.float32(gamma)).astype(np.float32)
    return (bias + step).astype(np.float32)


# ---------------------------------------------------------------------------
# Expert FFN (SwiGLU) and the combine ([Explained] recipe step 3 and the
# note on K_r and the shared expert; [Dissection] section II, DeepSeekMoE)
# ---------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (8 significant bits), half to even,
    in one step from the exact value. Values are assumed inside the bf16
    normal range (no overflow, no subnormals), as every expert output is."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                      # a = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def expert_up_q(xq: np.ndarray, xs: np.ndarray, wg_deq: np.ndarray, wu_deq: np.ndarray):
    """Up/gate stage of the quantised expert FFN for a set of rows.

    xq/xs: 1x128 codes and scales of the rows' input; wg_deq/wu_deq: float64
    dequantised gate and up weights [I, H]. G = x_hat W_gate^T and
    U = x_hat W_up^T in float64, h = silu(G) * U, then h is re-quantised 1x128
    from its float32 rounding (the down GEMM takes E4M3 inputs,
    [Dissection] section V, Figure 6).
    Returns (h float64 [rows, I], hq uint8 [rows, I], hs float32 [rows, I/128]).
    """
    x_hat = dequantize_1x128(xq, xs)
    g = x_hat @ wg_deq.T
    u = x_hat @ wu_deq.T
    h = silu(g) * u
    hq, hs = quantize_1x128(h.astype(np.float32))
    return h, hq, hs


def expert_down_q(hq: np.ndarray, hs: np.ndarray, wd_deq: np.ndarray) -> np.ndarray:
    """Down stage: Y = h_hat W_down^T summed in float64, not yet rounded.
    hq/hs: 1x128 codes and scales of h; wd_deq: float64 [H, I]."""
    return dequantize_1x128(hq, hs) @ wd_deq.T


def expert_ffn_q(xq: np.ndarray, xs: np.ndarray, wg_deq: np.ndarray,
                 wu_deq: np.ndarray, wd_deq: np.ndarray):
    """Quantisation-faithful expert FFN for a set of rows: expert_up_q, then
    expert_down_q, then the float64 sum rounded to bf16 (the FP8 GEMMs take
    E4M3 inputs, accumulate in FP32 and give BF16 outputs, [Dissection]
    section V, Figure 6).
    Returns (Y float64 [rows, H] holding bf16 values, hq uint8 [rows, I],
    hs float32 [rows, I/128]).
    """
    _, hq, hs = expert_up_q(xq, xs, wg_deq, wu_deq)
    return round_bf16(expert_down_q(hq, hs, wd_deq)), hq, hs


def expert_ffn_r(x: np.ndarray, wg: np.ndarray, wu: np.ndarray, wd: np.ndarray):
    """Unquantised float64 expert FFN (used only to measure FP8 error)."""
    x = np.asarray(x, np.float64)
    h = silu(x @ np.asarray(wg, np.float64).T) * (x @ np.asarray(wu, np.float64).T)
    return h @ np.asarray(wd, np.float64).T


def combine(y_shared: np.ndarray, y_routed: np.ndarray, ids: np.ndarray,
            gates: np.ndarray) -> np.ndarray:
    """y_t = FFN_shared(u_t) + sum_k g_{t,k} FFN_{id_k}(u_t).

    y_routed[t, k] is expert ids[t, k]'s output for token t. Summed in
    float64, shared first, then slots by ascending expert id.
    """
    out = np.array(y_shared, dtype=np.float64, copy=True)
    order = np.argsort(ids, axis=1, kind="stable")
    for t in range(out.shape[0]):
        for j in order[t]:
            out[t] += gates[t, j] * y_routed[t, j]
    return out


class ExpertWeights:
    """Per-expert weights assembled from a pool of 128x128 blocks.

    pool13/pool2: float32 blocks [P, 128, 128]; slot_gate/slot_up: [E, I/128,
    H/128] pool indices; slot_down: [E, H/128, I/128]. Expert E-1 is the
    shared expert. The oracle quantises the pool itself (128x128 blocks, so a
    block of the pool is a block of the weight matrix).
    """

    def __init__(self, pool13, pool2, slot_gate, slot_up, slot_down):
        self.pool13 = np.asarray(pool13, np.float32)
        self.pool2 = np.asarray(pool2, np.float32)
        self.slot_gate = np.asarray(slot_gate)
        self.slot_up = np.asarray(slot_up)
        self.slot_down = np.asarray(slot_down)
        self._q13 = None
        self._q2 = None

    def _quantised_pools(self):
        if self._q13 is None:
            p = self.pool13.shape[0]
            c13, s13 = quantize_128x128(self.pool13.reshape(p * TILE, TILE))
            self._q13 = (c13.reshape(p, TILE, TILE), s13.reshape(p))
            p = self.pool2.shape[0]
            c2, s2 = quantize_128x128(self.pool2.reshape(p * TILE, TILE))
            self._q2 = (c2.reshape(p, TILE, TILE), s2.reshape(p))
        return self._q13, self._q2

    def quantised_pools(self):
        """((codes13 [P,128,128], scales13 [P]), (codes2, scales2))."""
        return self._quantised_pools()

    @staticmethod
    def _assemble(blocks: np.ndarray, slots: np.ndarray) -> np.ndarray:
        nb, kb = slots.shape
        m = blocks[slots]  # [nb, kb, 128, 128]
        return m.transpose(0, 2, 1, 3).reshape(nb * TILE, kb * TILE)

    def dequantised(self, e: int):
        """(gate [I,H], up [I,H], down [H,I]) float64, dequantised."""
        if getattr(self, "_deq", None) is None:
            # dequantised pool blocks, kept: every expert is assembled from them
            (c13, s13), (c2, s2) = self._quantised_pools()
            self._deq = (e4m3_decode(c13) / s13.astype(np.float64)[:, None, None],
                         e4m3_decode(c2) / s2.astype(np.float64)[:, None, None])
        d13, d2 = self._deq
        return (self._assemble(d13, self.slot_gate[e]),
                self._assemble(d13, self.slot_up[e]),
                self._assemble(d2, self.slot_down[e]))

    def master(self, e: int):
        """(gate, up, down) float32 master weights, unquantised."""
        return (self._assemble(self.pool13, self.slot_gate[e]),
                self._assemble(self.pool13, self.slot_up[e]),
                self._assemble(self.pool2, self.slot_down[e]))


def moe_forward(x: np.ndarray, gate_w: np.ndarray, bias: np.ndarray, k: int,
                weights: ExpertWeights, mode: str = "Q", tokens=None,
                ids=None):
    """The MoE layer output for the rows `tokens` (all rows if None).

    mode "Q": quantisation-faithful (1x128 x, 128x128 weights, 1x128 h).
    mode "R": unquantised float64 reference (bf16 x and fp32 weights taken
    exactly), used only to measure the FP8 error.
    Routing always covers every token (the counts need them); `ids`, when
    given, replaces the routing decision (used for near-tie tokens) and the
    gates are recomputed from the unbiased affinities of those ids.
    Returns dict with y [len(tokens), H] float64, ids, gates, counts.
    """
    x = np.asarray(x, np.float32)
    t_count, h = x.shape
    n = gate_w.shape[0]
    r_ids, r_gates, s, _ = route(x, gate_w, bias, k)
    if ids is None:
        ids = r_ids
        gates = r_gates
    else:
        ids = np.asarray(ids, np.int32)
        sel = np.take_along_axis(s, ids, axis=1)
        gates = sel / np.sum(sel, axis=1, keepdims=True)
    counts = expert_counts(ids, n)
    if tokens is None:
        tokens = np.arange(t_count)
    tokens = np.asarray(tokens)
    xs_rows = x[tokens]
    if mode == "Q":
        xq, xsc = quantize_1x128(xs_rows)
    y_routed = np.zeros((len(tokens), k, h), dtype=np.float64)
    sub_ids = ids[tokens]
    for e in np.unique(sub_ids):
        rr, kk = np.nonzero(sub_ids == e)
        if mode == "Q":
            wg, wu, wd = weights.dequantised(int(e))
            y_e, _, _ = expert_ffn_q(xq[rr], xsc[rr], wg, wu, wd)
        else:
            wg, wu, wd = weights.master(int(e))
            y_e = expert_ffn_r(xs_rows[rr], wg, wu, wd)
        y_routed[rr, kk] = y_e
    shared = n  # expert index of the shared expert
    if mode == "Q":
        wg, wu, wd = weights.dequantised(shared)
        y_shared, _, _ = expert_ffn_q(xq, xsc, wg, wu, wd)
    else:
        wg, wu, wd = weights.master(shared)
        y_shared = expert_ffn_r(xs_rows, wg, wu, wd)
    y = combine(y_shared, y_routed, sub_ids, gates[tokens])
    return {"y": y, "ids": ids, "gates": gates, "counts": counts, "s": s}


# ---------------------------------------------------------------------------
# Backward of the expert path in FP8 ([Dissection] section V, Figure 6: the
# Fprop, Dgrad and Wgrad GEMMs of every linear layer run in FP8 with E4M3
# everywhere, fine-grained scales and fp32 accumulation; [Explained] step 7;
# gating stays in high precision, so the router's own backward is not here:
# the gate gradients are returned for it)
# ---------------------------------------------------------------------------

def quantize_128x1(a: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Tiles of 128 consecutive rows x 1 column: the 1x128 rule applied to
    the transposed matrix, for operands whose GEMM reduction runs over rows
    (the token dimension of a weight gradient). Rows are zero-padded to a
    multiple of 128 (padding does not change a tile's amax).

    Returns codes [C, R_pad] and scales [C, R_pad/128] of a.T (padded).
    """
    a = np.asarray(a, np.float32)
    r, c = a.shape
    r_pad = -(-r // TILE) * TILE
    pad = np.zeros((max(r_pad, TILE), c), np.float32)
    pad[:r] = a
    return quantize_1x128(np.ascontiguousarray(pad.T))


def dequantize_128x1(codes: np.ndarray, scales: np.ndarray, rows: int) -> np.ndarray:
    """Inverse of quantize_128x1, back to [rows, C] float64."""
    return dequantize_1x128(codes, scales).T[:rows]


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d silu(g) / dg = sigmoid(g) (1 + g (1 - sigmoid(g)))."""
    sg = 1.0 / (1.0 + np.exp(-g))
    return sg * (1.0 + g * (1.0 - sg))


def expert_ffn_backward_q(xq: np.ndarray, xs: np.ndarray, x: np.ndarray, dy: np.ndarray,
                          wg: np.ndarray, wu: np.ndarray, wd: np.ndarray):
    """FP8 backward of one expert over its rows (in the permutation's order).

    xq/xs: the forward's 1x128 codes/scales of the rows' input; x: the rows'
    input values (the bf16 x) for the weight gradient; dy: float32 [rows, H]
    upstream gradient of the expert's output rows (already times the gate);
    wg, wu [I, H] and wd [H, I]: dequantised weights.
      G, U, h recomputed from the dequantised x (float64)
      Dgrad down:  dh = Q1x128(dy) . Wd               (reduction over H)
      SwiGLU:      dG = dh U silu'(G),  dU = dh silu(G)
      Dgrad up:    dx = Q1x128(dG) . Wg + Q1x128(dU) . Wu   (reduction over I)
      Wgrad down:  dWd = Q128x1(dy)^T . Q128x1(h)     (reduction over rows)
      Wgrad up:    dWg = Q128x1(dG)^T . Q128x1(x),  dWu likewise with dU
    Every quantised operand is the float32 rounding of its float64 value; the
    forward's h quantisation is passed straight through (dh is the gradient
    of the quantised h). Returns dict of float64 arrays.
    """
    rows = dy.shape[0]
    x_hat = dequantize_1x128(xq, xs)
    g = x_hat @ wg.T
    u = x_hat @ wu.T
    h = silu(g) * u
    dyq, dys = quantize_1x128(np.asarray(dy, np.float32))
    dh = dequantize_1x128(dyq, dys) @ wd
    d_g = dh * u * silu_grad(g)
    d_u = dh * silu(g)
    dgq, dgs = quantize_1x128(d_g.astype(np.float32))
    duq, dus = quantize_1x128(d_u.astype(np.float32))
    dx = dequantize_1x128(dgq, dgs) @ wg + dequantize_1x128(duq, dus) @ wu
    q = lambda a: dequantize_128x1(*quantize_128x1(a), rows)
    x32 = np.asarray(x, np.float32)
    dwd = q(np.asarray(dy, np.float32)).T @ q(h.astype(np.float32))
    dwg = q(d_g.astype(np.float32)).T @ q(x32)
    dwu = q(d_u.astype(np.float32)).T @ q(x32)
    return {"dx": dx, "dwg": dwg, "dwu": dwu, "dwd": dwd, "dh": dh, "d_g": d_g, "d_u": d_u}


def expert_ffn_backward_r(x: np.ndarray, dy: np.ndarray, wg: np.ndarray, wu: np.ndarray,
                          wd: np.ndarray):
    """Unquantised float64 backward of expert_ffn_r (chain rule, no FP8)."""
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    wg, wu, wd = (np.asarray(w, np.float64) for w in (wg, wu, wd))
    g = x @ wg.T
    u = x @ wu.T
    h = silu(g) * u
    dh = dy @ wd
    d_g = dh * u * silu_grad(g)
    d_u = dh * silu(g)
    return {"dx": d_g @ wg + d_u @ wu, "dwg": d_g.T @ x, "dwu": d_u.T @ x, "dwd": dy.T @ h}


def moe_backward(x: np.ndarray, gate_w: np.ndarray, bias: np.ndarray, k: int,
                 weights: ExpertWeights, dy: np.ndarray, mode: str = "Q", ids=None,
                 tokens=None):
    """Backward of moe_forward's expert path for the upstream gradient dy
    [T, H] of y, with the routing held fixed (the router's backward stays in
    high precision and takes the gate gradients returned here):
      dY rows: g[t,k] * dy[t] for routed slots, dy[t] for the shared expert
      dx[t]  = sum over the token's K + 1 rows of the experts' input gradients
      dgates[t,k] = dy[t] . Y_k[t]  (the expert's forward output row)
      dW*: per expert (index N: the shared expert)
    Rows of each expert in ascending token order, as the permutation lays
    them out. With `tokens` (a subset), only those tokens' rows are run: dx
    and dgates of a token depend on its own rows alone (every Dgrad
    quantisation tile lies in one row), so they equal the full run's up to
    float64 rounding order; the weight gradients, which need every row, are
    then not returned.
    Returns dict: dx [T,H], dgates [T,K], dw {expert: (dwg [I,H], dwu [I,H],
    dwd [H,I])}.
    """
    x = np.asarray(x, np.float32)
    dy = np.asarray(dy, np.float32)
    t_count, h_dim = x.shape
    n = gate_w.shape[0]
    r_ids, r_gates, s, _ = route(x, gate_w, bias, k)
    if ids is None:
        ids, gates = r_ids, r_gates
    else:
        ids = np.asarray(ids, np.int32)
        sel = np.take_along_axis(s, ids, axis=1)
        gates = sel / np.sum(sel, axis=1, keepdims=True)
    if mode == "Q":
        xq, xsc = quantize_1x128(x)
    dx = np.zeros((t_count, h_dim))
    dgates = np.zeros((t_count, k))
    out_w = {}
    keep = np.zeros(t_count, bool)
    keep[np.arange(t_count) if tokens is None else np.asarray(tokens)] = True
    for e in list(np.unique(ids[keep])) + [n]:
        e = int(e)
        if e == n:
            rr = np.nonzero(keep)[0]
            kk = None
            dy_rows = dy[rr].astype(np.float64)
        else:
            rr, kk = np.nonzero((ids == e) & keep[:, None])   # ascending token order
            dy_rows = gates[rr, kk][:, None] * dy[rr].astype(np.float64)
        if mode == "Q":
            wg, wu, wd = weights.dequantised(e)
            res = expert_ffn_backward_q(xq[rr], xsc[rr], x[rr], dy_rows.astype(np.float32),
                                        wg, wu, wd)
            y_e, _, _ = expert_ffn_q(xq[rr], xsc[rr], wg, wu, wd)
        else:
            wg, wu, wd = weights.master(e)
            res = expert_ffn_backward_r(x[rr], dy_rows, wg, wu, wd)
            y_e = expert_ffn_r(x[rr], wg, wu, wd)
        np.add.at(dx, rr, res["dx"])
        if kk is not None:
            dgates[rr, kk] = np.sum(dy[rr].astype(np.float64) * y_e, axis=1)
        if tokens is None:
            out_w[e] = (res["dwg"], res["dwu"], res["dwd"])
    return {"dx": dx, "dgates": dgates, "dw": out_w, "ids": ids, "gates": gates}
