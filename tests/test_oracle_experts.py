"""Pins for the oracle's expert FFNs and combine.

"DeepSeek-V3, explained", recipe step 3 and the K_r note: a token uses the
shared expert at full weight plus K routed experts weighted by normalised
gates. "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...", section III:
g'_i = s_i when s_i + b_i is in the top K, else 0; g = g' / sum g'.
The sparse layer must equal the dense "run every expert, then mask" layer:
the masked terms are exact zeros, so the two differ only by the summation
order inside the float64 library matmuls (a few ulps).
"""
import math

import numpy as np
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I
from tests.test_oracle_codec import _page_rounding_rule


def _tiny_all():
    w = I.WORKLOADS["tiny"]
    x = I.bf16_bits_to_f32(I.make_x(w))
    pool = I.make_weight_pool(w)
    ew = O.ExpertWeights(pool.pool13, pool.pool2, pool.slot_gate, pool.slot_up, pool.slot_down)
    return w, x, I.make_gate_w(w), I.make_bias(w), pool, ew


def test_assembly_places_pool_blocks():
    w, _, _, _, pool, ew = _tiny_all()
    g, u, d = ew.master(3)
    assert g.shape == (w.I, w.H) and d.shape == (w.H, w.I)
    for nb in range(w.I // 128):
        for kb in range(w.H // 128):
            blk = g[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert np.array_equal(blk, pool.pool13[pool.slot_gate[3, nb, kb]])
            blk = u[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert np.array_equal(blk, pool.pool13[pool.slot_up[3, nb, kb]])
    for nb in range(w.H // 128):
        for kb in range(w.I // 128):
            blk = d[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert np.array_equal(blk, pool.pool2[pool.slot_down[3, nb, kb]])
    # the tiny pool has one entry per block: all blocks distinct
    assert len(np.unique(np.concatenate([pool.slot_gate.ravel(), pool.slot_up.ravel()]))) == pool.pool13.shape[0]


def test_swiglu_brute_force_loops():
    rng = np.random.default_rng(21)
    h_dim, i_dim = 256, 128
    x = rng.standard_normal((2, h_dim)).astype(np.float32)
    wg = (rng.standard_normal((i_dim, h_dim)) / 16).astype(np.float32)
    wu = (rng.standard_normal((i_dim, h_dim)) / 16).astype(np.float32)
    wd = (rng.standard_normal((h_dim, i_dim)) / 11).astype(np.float32)
    y = O.expert_ffn_r(x, wg, wu, wd)
    for t in range(2):
        hvec = []
        for j in range(i_dim):
            gj = sum(float(x[t, c]) * float(wg[j, c]) for c in range(h_dim))
            uj = sum(float(x[t, c]) * float(wu[j, c]) for c in range(h_dim))
            hvec.append(gj / (1.0 + np.exp(-gj)) * uj)
        for o in range(0, h_dim, 37):
            yo = sum(hvec[j] * float(wd[o, j]) for j in range(i_dim))
            assert abs(y[t, o] - yo) <= 1e-12 * (1 + abs(yo))


def test_quantised_ffn_uses_dequantised_operands():
    rng = np.random.default_rng(22)
    x = rng.standard_normal((3, 256)).astype(np.float32)
    wg = (rng.standard_normal((128, 256)) / 16).astype(np.float32)
    wu = (rng.standard_normal((128, 256)) / 16).astype(np.float32)
    wd = (rng.standard_normal((256, 128)) / 11).astype(np.float32)
    xq, xs = O.quantize_1x128(x)
    dg = O.dequantize_128x128(*O.quantize_128x128(wg))
    du = O.dequantize_128x128(*O.quantize_128x128(wu))
    dd = O.dequantize_128x128(*O.quantize_128x128(wd))
    y, hq, hs = O.expert_ffn_q(xq, xs, dg, du, dd)
    # h before re-quantisation, from the unquantised float64 FFN on the dequantised operands
    xh = O.dequantize_1x128(xq, xs)
    h = O.silu(xh @ dg.T) * (xh @ du.T)
    hq2, hs2 = O.quantize_1x128(h.astype(np.float32))
    assert np.array_equal(hq, hq2) and np.array_equal(hs, hs2)
    # bf16 outputs ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing...",
    # section V, Figure 6): 8 significant bits, within half a step of the
    # float64 sum, and torch's own bf16 cast of that sum (values exactly
    # representable in float32 are compared, so torch rounds once)
    y64 = O.dequantize_1x128(hq, hs) @ dd.T
    assert np.all(np.abs(y - y64) <= 2.0 ** -8 * np.abs(y64))
    y32 = y64.astype(np.float32)
    exact = y32.astype(np.float64) == y64
    ref = torch.from_numpy(y32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(y[exact], ref[exact])
    assert np.mean(y != y64) > 0.9


def _brute_h(x_hat, wg, wu):
    """h = silu(x_hat . wg) * (x_hat . wu) with plain Python sums."""
    rows, h_dim = x_hat.shape
    out = np.empty((rows, wg.shape[0]))
    for t in range(rows):
        for j in range(wg.shape[0]):
            gj = sum(float(x_hat[t, c]) * float(wg[j, c]) for c in range(h_dim))
            uj = sum(float(x_hat[t, c]) * float(wu[j, c]) for c in range(h_dim))
            out[t, j] = gj / (1.0 + math.exp(-gj)) * uj
    return out


def _page_tile_1x128(h):
    """The per-tile rule of "DeepSeek-V3 Technical Report" (deepforge),
    "Per-tile FP8 scaling", applied to rows of h in tiles of 128 channels:
    scale = 448 / amax (float32), X_fp8 = round(X * scale) with the page's
    E4M3 rounding, X_hat = X_fp8 / scale."""
    h32 = np.asarray(h, np.float32)
    out = np.empty(h32.shape)
    for t in range(h32.shape[0]):
        for c in range(0, h32.shape[1], 128):
            tile = h32[t, c:c + 128]
            scale = np.float32(448.0) / np.max(np.abs(tile))
            prod = (tile * scale).astype(np.float32).astype(np.float64)
            out[t, c:c + 128] = _page_rounding_rule(prod) / np.float64(scale)
    return out


def test_h_requantisation_seen_through_identity_down_weights():
    """With W_down = 2^-3 times the identity (H = I = 128: one 128x128 block,
    quantised losslessly: amax 2^-3, every diagonal code 448), Y = 2^-3 h_hat
    before its bf16 rounding, so the oracle's down stage exposes the 1x128
    re-quantised h element by element. It must equal the page's per-tile rule
    applied to h computed by plain loops; an oracle that skipped the
    re-quantisation of h, or tiled it another way, fails here."""
    rng = np.random.default_rng(23)
    x = rng.standard_normal((2, 128)).astype(np.float32)
    wg = (rng.standard_normal((128, 128)) / 11).astype(np.float32)
    wu = (rng.standard_normal((128, 128)) / 11).astype(np.float32)
    wd = (np.eye(128) * 2.0 ** -3).astype(np.float32)
    xq, xs = O.quantize_1x128(x)
    dg = O.dequantize_128x128(*O.quantize_128x128(wg))
    du = O.dequantize_128x128(*O.quantize_128x128(wu))
    dd = O.dequantize_128x128(*O.quantize_128x128(wd))
    assert np.array_equal(dd, wd.astype(np.float64))          # lossless block
    h = _brute_h(O.dequantize_1x128(xq, xs), dg, du)
    h_hat = _page_tile_1x128(h)
    assert np.max(np.abs(h_hat - h)) > 1e-3 * np.max(np.abs(h))  # quantisation is visible
    _, hq, hs = O.expert_up_q(xq, xs, dg, du)
    y64 = O.expert_down_q(hq, hs, dd)
    assert np.array_equal(y64, 2.0 ** -3 * h_hat)
    y, _, _ = O.expert_ffn_q(xq, xs, dg, du, dd)
    assert np.array_equal(y, O.round_bf16(2.0 ** -3 * h_hat))


def test_sparse_equals_dense_then_mask():
    w, x, g, b, pool, ew = _tiny_all()
    out = O.moe_forward(x, g, b, w.K, ew, mode="Q")
    # dense: every expert on every token, then the gate equation with zeros
    xq, xs = O.quantize_1x128(x)
    dense = []
    for e in range(w.N + 1):
        dg, du, dd = ew.dequantised(e)
        dense.append(O.expert_ffn_q(xq, xs, dg, du, dd)[0])
    s = 1.0 / (1.0 + np.exp(-(x.astype(np.float64) @ g.astype(np.float64).T)))
    score = s + b.astype(np.float64)
    y = np.array(dense[w.N], copy=True)
    for t in range(w.T):
        kth = np.sort(score[t])[::-1][w.K - 1]
        gp = np.where(score[t] >= kth, s[t], 0.0)   # g'_i (no exact ties here)
        assert np.count_nonzero(gp) == w.K
        gn = gp / gp.sum()
        for i in range(w.N):
            y[t] += gn[i] * dense[i][t]
    err = np.abs(out["y"] - y).max() / np.abs(y).max()
    assert err < 1e-13, err


def test_shared_expert_only_when_gates_are_zero():
    w, x, g, b, pool, ew = _tiny_all()
    xq, xs = O.quantize_1x128(x)
    ys, _, _ = O.expert_ffn_q(xq, xs, *ew.dequantised(w.N))
    yr = np.random.default_rng(0).standard_normal((w.T, w.K, w.H))
    ids = np.tile(np.arange(w.K), (w.T, 1))
    assert np.array_equal(O.combine(ys, yr, ids, np.zeros((w.T, w.K))), ys)


def test_token_subset_matches_full_forward():
    w, x, g, b, pool, ew = _tiny_all()
    full = O.moe_forward(x, g, b, w.K, ew, mode="Q")
    sub = np.array([0, 7, 33, 63])
    part = O.moe_forward(x, g, b, w.K, ew, mode="Q", tokens=sub)
    assert np.allclose(part["y"], full["y"][sub], rtol=1e-13, atol=1e-15)


def test_fp8_error_band_against_unquantised():
    """Mode Q against mode R: every E4M3 rounding adds about 2.6% RMS relative
    error per element on Gaussian data (uniform error within half a step of
    1/8 of a binade). The up/gate dot products inherit x and W errors (~3.7%),
    SwiGLU multiplies two such terms (~5.2%), re-quantising h and the down
    weights add two more roundings (~6.4%). The measured RMS-relative output
    error must sit in the band around that estimate."""
    w, x, g, b, pool, ew = _tiny_all()
    yq = O.moe_forward(x, g, b, w.K, ew, mode="Q")["y"]
    yr = O.moe_forward(x, g, b, w.K, ew, mode="R")["y"]
    rel = np.sqrt(np.mean((yq - yr) ** 2)) / np.sqrt(np.mean(yr ** 2))
    assert 0.04 < rel < 0.09, rel


def test_forced_routing_keeps_the_unbiased_gates():
    """The near-tie rule re-runs the layer with another routing decision
    (the GPU's ids). The gates then follow the pages' definition for those
    ids ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...", section
    III: g = s_i / sum of the chosen s, the bias only choosing): from the
    unbiased affinities, whatever the bias. Handing the layer its own routing
    back reproduces the unforced run exactly; a forced routing of the least
    likely experts under a large bias gets gates from sigma(u . e_i), computed
    here with plain loops, and the forward and backward agree on them."""
    w, x, g, b, pool, ew = _tiny_all()
    b = (np.sign(I.make_bias(w)) * 0.5).astype(np.float32)      # large bias
    base = O.moe_forward(x, g, b, w.K, ew, mode="Q")
    again = O.moe_forward(x, g, b, w.K, ew, mode="Q", ids=base["ids"])
    assert np.array_equal(again["y"], base["y"]) and np.array_equal(again["gates"], base["gates"])
    _, _, _, score = O.route(x, g, b, w.K)
    forced = np.argsort(score, axis=1, kind="stable")[:, :w.K].astype(np.int32)
    expect = np.empty(forced.shape)
    for t in range(w.T):
        s = [1.0 / (1.0 + math.exp(-sum(float(x[t, c]) * float(g[e, c]) for c in range(w.H))))
             for e in forced[t]]
        expect[t] = np.array(s) / sum(s)
    fw = O.moe_forward(x, g, b, w.K, ew, mode="Q", ids=forced)
    assert np.array_equal(fw["ids"], forced)
    assert np.max(np.abs(fw["gates"] - expect)) < 1e-12
    dy = np.random.default_rng(3).standard_normal((w.T, w.H)).astype(np.float32)
    bw = O.moe_backward(x, g, b, w.K, ew, dy, mode="Q", ids=forced, tokens=[0, 5])
    assert np.array_equal(bw["gates"], fw["gates"])
