"""Pins for the oracle's FP8 expert backward.

Against the chain rule, checked independently of the backward formulas by
central finite differences of the unquantised forward (routing and gates
held fixed, as the expert path's backward defines them); the gate gradient
dy . Y_k by differences in the gates; and, for the FP8 path ("DeepSeek-V3:
Auxiliary-Loss-Free MoE Load Balancing...", section V, Figure 6: Dgrad and
Wgrad in E4M3 with 1x128 activation tiles, 128x128 weight blocks, fp32
accumulation), exact scale invariance (doubling dy doubles every gradient
bit for bit, since the tile scale halves exactly), zero in -> zero out, and
the FP8-versus-float64 error band.
"""
import numpy as np

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I


def _small(t=6, n=16, k=2, seed=41):
    w = I.Workload("bw", T=t, H=256, N=n, K=k, I=128, bias_range=0.1, seed=seed)
    pool = I.make_weight_pool(w)
    ew = O.ExpertWeights(pool.pool13, pool.pool2, pool.slot_gate, pool.slot_up, pool.slot_down)
    x = I.bf16_bits_to_f32(I.make_x(w))
    dy = np.random.default_rng(seed).standard_normal((t, w.H)).astype(np.float32)
    return w, ew, x, I.make_gate_w(w), I.make_bias(w), dy


def _loss_r(x, ids, gates, ew, dy, n):
    """sum(dy * y) of the unquantised layer with the routing held fixed."""
    y_sh = O.expert_ffn_r(x, *ew.master(n))
    y_ro = np.zeros((x.shape[0], ids.shape[1], x.shape[1]))
    for t in range(x.shape[0]):
        for j in range(ids.shape[1]):
            y_ro[t, j] = O.expert_ffn_r(x[t:t + 1], *ew.master(int(ids[t, j])))[0]
    y = O.combine(y_sh, y_ro, ids, gates)
    return float(np.sum(dy.astype(np.float64) * y))


def test_dx_matches_finite_differences():
    w, ew, x, gw, b, dy = _small()
    res = O.moe_backward(x, gw, b, w.K, ew, dy, mode="R")
    ids, gates = res["ids"], res["gates"]
    x64 = x.astype(np.float64)
    rng = np.random.default_rng(0)
    for _ in range(6):
        t, j = rng.integers(w.T), rng.integers(w.H)
        eps = 1e-4
        xp, xm = x64.copy(), x64.copy()
        xp[t, j] += eps
        xm[t, j] -= eps
        fd = (_loss_r(xp, ids, gates, ew, dy, w.N) - _loss_r(xm, ids, gates, ew, dy, w.N)) / (2 * eps)
        assert abs(fd - res["dx"][t, j]) <= 1e-6 * (1 + abs(fd)), (t, j, fd, res["dx"][t, j])


def test_weight_gradients_match_finite_differences():
    w, ew, x, gw, b, dy = _small()
    res = O.moe_backward(x, gw, b, w.K, ew, dy, mode="R")
    ids, gates = res["ids"], res["gates"]
    e = int(ids[0, 0])
    rr, kk = np.nonzero(ids == e)
    dy_rows = gates[rr, kk][:, None] * dy[rr].astype(np.float64)
    wg, wu, wd = (m.astype(np.float64) for m in ew.master(e))
    dwg, dwu, dwd = res["dw"][e]
    rng = np.random.default_rng(1)
    eps = 1e-4
    for name, mat, grad in [("gate", wg, dwg), ("up", wu, dwu), ("down", wd, dwd)]:
        for _ in range(3):
            i, j = rng.integers(mat.shape[0]), rng.integers(mat.shape[1])
            vals = []
            for sgn in (1, -1):
                m2 = mat.copy()
                m2[i, j] += sgn * eps
                args = {"gate": (m2, wu, wd), "up": (wg, m2, wd), "down": (wg, wu, m2)}[name]
                vals.append(np.sum(dy_rows * O.expert_ffn_r(x[rr], *args)))
            fd = (vals[0] - vals[1]) / (2 * eps)
            assert abs(fd - grad[i, j]) <= 1e-6 * (1 + abs(fd)), (name, i, j, fd, grad[i, j])


def test_gate_gradients_are_dy_dot_expert_output():
    w, ew, x, gw, b, dy = _small()
    res = O.moe_backward(x, gw, b, w.K, ew, dy, mode="R")
    ids, gates = res["ids"], res["gates"]
    eps = 1e-6
    for t, j in [(0, 0), (3, 1), (5, 0)]:
        gp, gm = gates.copy(), gates.copy()
        gp[t, j] += eps
        gm[t, j] -= eps
        lp = _loss_r(x.astype(np.float64), ids, gp, ew, dy, w.N)
        lm = _loss_r(x.astype(np.float64), ids, gm, ew, dy, w.N)
        assert abs((lp - lm) / (2 * eps) - res["dgates"][t, j]) < 1e-6 * (1 + abs(res["dgates"][t, j]))


def test_fp8_backward_scale_invariance_is_exact():
    w, ew, x, gw, b, dy = _small(t=40, n=16, k=4, seed=42)
    r1 = O.moe_backward(x, gw, b, w.K, ew, dy, mode="Q")
    r2 = O.moe_backward(x, gw, b, w.K, ew, 2 * dy, mode="Q")
    assert np.array_equal(r2["dx"], 2 * r1["dx"])
    assert np.array_equal(r2["dgates"], 2 * r1["dgates"])
    for e in r1["dw"]:
        for a, c in zip(r1["dw"][e], r2["dw"][e]):
            assert np.array_equal(c, 2 * a)


def test_fp8_backward_zero_in_zero_out():
    w, ew, x, gw, b, dy = _small(seed=43)
    res = O.moe_backward(x, gw, b, w.K, ew, np.zeros_like(dy), mode="Q")
    assert not np.any(res["dx"]) and not np.any(res["dgates"])
    assert all(not np.any(m) for e in res["dw"] for m in res["dw"][e])


def test_fp8_backward_error_band():
    """E4M3 quantisation of dy, of dG/dU and (in the forward) of x, the
    weights and h moves the gradients by a few percent RMS against the
    unquantised float64 backward; the float32 accumulation does not."""
    w, ew, x, gw, b, dy = _small(t=64, n=16, k=4, seed=44)
    rq = O.moe_backward(x, gw, b, w.K, ew, dy, mode="Q")
    rr = O.moe_backward(x, gw, b, w.K, ew, dy, mode="R", ids=rq["ids"])
    rel = lambda a, c: np.sqrt(np.mean((a - c) ** 2) / np.mean(c ** 2))
    e_dx = rel(rq["dx"], rr["dx"])
    assert 0.01 < e_dx < 0.15, e_dx
    e_w = rel(rq["dw"][w.N][2], rr["dw"][w.N][2])
    assert 0.01 < e_w < 0.15, e_w


def test_quantize_128x1_tiles_run_down_the_rows():
    rng = np.random.default_rng(7)
    a = (rng.standard_normal((200, 256)) * rng.uniform(0.1, 5, (200, 1))).astype(np.float32)
    codes, scales = O.quantize_128x1(a)
    assert codes.shape == (256, 256) and scales.shape == (256, 2)
    for c in [0, 17, 255]:
        for blk, (lo, hi) in enumerate([(0, 128), (128, 200)]):
            amax = np.float32(np.max(np.abs(a[lo:hi, c])))
            assert scales[c, blk] == np.float32(448.0) / amax
    assert not np.any(codes[:, 200:])            # zero padding
    back = O.dequantize_128x1(codes, scales, 200)
    assert np.all(np.abs(back - a) <= np.abs(a) * 2.0 ** -4 + 2.0 ** -10 / np.repeat(scales, 128, 1).T[:200])


def test_token_subset_matches_full_run():
    w, ew, x, gw, b, dy = _small(t=40, n=16, k=4, seed=45)
    full = O.moe_backward(x, gw, b, w.K, ew, dy, mode="Q")
    toks = [3, 17, 29]
    sub = O.moe_backward(x, gw, b, w.K, ew, dy, mode="Q", tokens=toks)
    np.testing.assert_allclose(sub["dx"][toks], full["dx"][toks], rtol=0,
                               atol=1e-12 * np.abs(full["dx"]).max())
    np.testing.assert_allclose(sub["dgates"][toks], full["dgates"][toks], rtol=0,
                               atol=1e-12 * np.abs(full["dgates"]).max())
    assert sub["dw"] == {}


# --------------------------------------------------------------------------
# Lossless cases: every quantised operand sits on the E4M3 grid of its own
# tile (tile amax 448 * 2^m, so the tile scale is a power of two, or every
# element equal), so each FP8 GEMM must reproduce the float64 chain rule of
# expert_ffn_backward_r (itself pinned by finite differences above) up to
# float64 summation order; the same operands tiled along the other axis are
# lossy, so an oracle that tiled an operand the wrong way fails.
#
# Structure (H = I = 128, one block per weight): W_gate = 1/4 in channel c0
# of every row, so G = 64 everywhere for x = 256 (silu(64) = 64 and
# silu'(64) = 1 exactly in float64); W_up = 2^-3 P_sigma and
# W_down = 2^-2 P_pi (scaled permutations); so U = 32, h = 2048,
# dh = 2^-2 dy permuted, dG = 32 dh and dU = 64 dh.
# --------------------------------------------------------------------------

def _lossless_weights(seed):
    rng = np.random.default_rng(seed)
    wg = np.zeros((128, 128), np.float32)
    wg[:, 5] = 0.25
    wu = np.zeros((128, 128), np.float32)
    wu[np.arange(128), rng.permutation(128)] = 2.0 ** -3
    wd = np.zeros((128, 128), np.float32)
    wd[rng.permutation(128), np.arange(128)] = 2.0 ** -2
    deq = []
    for m in (wg, wu, wd):
        d = O.dequantize_128x128(*O.quantize_128x128(m))
        assert np.array_equal(d, m.astype(np.float64))      # lossless blocks
        deq.append(d)
    return deq


def _grid_values(rng, shape):
    """Random finite E4M3 values (both signs, subnormals included)."""
    codes = rng.integers(0, 0x7F, shape).astype(np.uint8)
    codes |= (rng.integers(0, 2, shape) << 7).astype(np.uint8)
    return O.e4m3_decode(codes)


def _on_grid(rows, cols, exps, axis, rng):
    """Values whose tiles along `axis` (1: along a row, 0: down a column)
    are lossless: grid values times 2^(m - 8), the tile's largest = 448 * 2^(m - 8)."""
    v = _grid_values(rng, (rows, cols))
    if axis == 1:
        v[np.arange(rows), rng.integers(0, cols, rows)] = 448.0
        v *= 2.0 ** (np.asarray(exps, np.float64)[:, None] - 8)
    else:
        v[rng.integers(0, rows, cols), np.arange(cols)] = 448.0
        v *= 2.0 ** (np.asarray(exps, np.float64)[None, :] - 8)
    return v.astype(np.float32)


def _fp8_vs_chain_rule(x, dy, wg, wu, wd):
    xq, xs = O.quantize_1x128(x)
    q = O.expert_ffn_backward_q(xq, xs, x, dy, wg, wu, wd)
    r = O.expert_ffn_backward_r(x, dy.astype(np.float64), wg, wu, wd)
    return q, r


def _close(a, b):
    return np.max(np.abs(a - b)) <= 1e-12 * np.max(np.abs(b))


def test_dgrad_lossless_rows_equal_the_chain_rule():
    """Dgrad quantises dy and dG/dU in 1x128 tiles along each row. Rows with
    magnitudes 2^40 apart make 128x1 tiles lossy, 1x128 tiles exact."""
    rng = np.random.default_rng(51)
    wg, wu, wd = _lossless_weights(51)
    x = np.full((8, 128), 256.0, np.float32)
    dy = _on_grid(8, 128, [-20, -14, -8, -2, 4, 10, 16, 20], axis=1, rng=rng)
    q, r = _fp8_vs_chain_rule(x, dy, wg, wu, wd)
    assert np.array_equal(q["dh"], dy.astype(np.float64) @ wd)
    assert _close(q["dx"], r["dx"])
    # the same dy in 128x1 tiles loses the small rows
    wrong = O.dequantize_128x1(*O.quantize_128x1(dy), 8)
    assert not _close(wrong, dy.astype(np.float64))


def test_wgrad_lossless_columns_equal_the_chain_rule():
    """Wgrad quantises dy and h in 128x1 tiles down each column for
    dW_down = Q(dy)^T . Q(h). Columns of dy with magnitudes up to 2^40 apart
    are exact in 128x1 tiles and lossy in 1x128 tiles. (dW_gate and dW_up
    take dG/dU from the Dgrad's row-quantised dy, which these columns make
    lossy; they are pinned by the next tests.)"""
    rng = np.random.default_rng(52)
    wg, wu, wd = _lossless_weights(52)
    x = np.full((128, 128), 256.0, np.float32)
    dy = _on_grid(128, 128, rng.integers(-20, 21, 128), axis=0, rng=rng)
    q, r = _fp8_vs_chain_rule(x, dy, wg, wu, wd)
    assert _close(q["dwd"], r["dwd"])
    wrong = O.dequantize_1x128(*O.quantize_1x128(dy))
    assert not _close(wrong, dy.astype(np.float64))


def test_wgrad_down_uses_h_quantised_down_its_columns():
    """dW_down = Q(dy)^T . Q(h) with h in 128x1 tiles. A dy that selects one
    row per output channel (a power of two, lossless) makes dW_down expose
    the quantised h row by row; it must equal the page's per-tile rule
    ("DeepSeek-V3 Technical Report" (deepforge), "Per-tile FP8 scaling")
    applied to each column of h, computed here from float64 products.
    Skipping h's quantisation, or tiling it along the rows, fails."""
    from tests.test_oracle_codec import _page_rounding_rule
    rng = np.random.default_rng(53)
    rows, h_dim, i_dim = 128, 256, 128
    x = I.bf16_bits_to_f32(I.f32_to_bf16_bits(rng.standard_normal((rows, h_dim)).astype(np.float32)))
    x *= np.float32(2.0) ** rng.integers(-3, 4, (rows, 1)).astype(np.float32)
    wg = O.dequantize_128x128(*O.quantize_128x128(
        (rng.standard_normal((i_dim, h_dim)) / 16).astype(np.float32)))
    wu = O.dequantize_128x128(*O.quantize_128x128(
        (rng.standard_normal((i_dim, h_dim)) / 16).astype(np.float32)))
    wd = O.dequantize_128x128(*O.quantize_128x128(
        (rng.standard_normal((h_dim, i_dim)) / 11).astype(np.float32)))
    pick = rng.integers(0, rows, h_dim)
    dy = np.zeros((rows, h_dim), np.float32)
    dy[pick, np.arange(h_dim)] = 2.0 ** -5
    xq, xs = O.quantize_1x128(x)
    q = O.expert_ffn_backward_q(xq, xs, x, dy, wg, wu, wd)
    # h from the forward's dequantised x, then the page's rule down each column
    x_hat = O.dequantize_1x128(xq, xs)
    h = (O.silu(x_hat @ wg.T) * (x_hat @ wu.T)).astype(np.float32)
    h_hat = np.empty(h.shape)
    for c in range(i_dim):
        scale = np.float32(448.0) / np.max(np.abs(h[:, c]))
        prod = (h[:, c] * scale).astype(np.float32).astype(np.float64)
        h_hat[:, c] = _page_rounding_rule(prod) / np.float64(scale)
    assert np.max(np.abs(h_hat - h)) > 1e-3 * np.max(np.abs(h))
    assert np.array_equal(q["dwd"], 2.0 ** -5 * h_hat[pick])


def test_wgrad_up_uses_x_quantised_down_its_columns():
    """dW_up = Q(dU)^T . Q(x) and dW_gate = Q(dG)^T . Q(x), with x and dG/dU
    in 128x1 tiles. With the lossless weights and x = 256 in channel c0
    (the largest of every row, so G = 64 exactly) but Gaussian elsewhere, a
    dy that selects one row per channel (a power of two) makes dU = 64 dh a
    power-of-two selector (lossless), so dW_up exposes the column-quantised
    x row by row: it must equal the page's per-tile rule applied to each
    column of x. dG = dh U holds one Gaussian value per column (lossless up
    to the float32 tile scale), so dW_gate = dG^T x_hat to 1e-6; tiling
    dG or x along the rows instead fails."""
    from tests.test_oracle_codec import _page_rounding_rule
    rng = np.random.default_rng(54)
    wg, wu, wd = _lossless_weights(54)
    rows = 128
    x = I.bf16_bits_to_f32(I.f32_to_bf16_bits(
        (rng.standard_normal((rows, 128)) * 10.0 ** rng.uniform(-1, 1, (1, 128))).astype(np.float32)))
    x[:, 5] = 256.0
    assert np.all(np.abs(np.delete(x, 5, axis=1)) < 256.0)
    pick = rng.integers(0, rows, 128)
    dy = np.zeros((rows, 128), np.float32)
    dy[pick, np.arange(128)] = 2.0 ** -3
    xq, xs = O.quantize_1x128(x)
    q = O.expert_ffn_backward_q(xq, xs, x, dy, wg, wu, wd)
    x_col = np.empty(x.shape)
    for c in range(128):
        scale = np.float32(448.0) / np.max(np.abs(x[:, c]))
        prod = (x[:, c] * scale).astype(np.float32).astype(np.float64)
        x_col[:, c] = _page_rounding_rule(prod) / np.float64(scale)
    assert np.max(np.abs(x_col - x)) > 1e-3 * np.max(np.abs(x))
    # dU[r, i] = 64 * dh[r, i] = 64 * 2^-2 * dy[r, perm(i)]: one entry per column
    du = q["d_u"]
    row_of = np.argmax(np.abs(du), axis=0)
    assert np.count_nonzero(du) == 128
    assert np.array_equal(q["dwu"], du[row_of, np.arange(128)][:, None] * x_col[row_of])
    dg = q["d_g"]
    assert np.count_nonzero(dg) == 128
    ref = dg[row_of, np.arange(128)][:, None] * x_col[row_of]
    assert np.max(np.abs(q["dwg"] - ref)) <= 1e-6 * np.max(np.abs(ref))
    wrong = O.dequantize_1x128(*O.quantize_1x128(x))
    assert np.max(np.abs(wrong - x_col)) > 1e-3 * np.max(np.abs(x))


def test_dgrad_quantises_dy_and_dg_du_in_row_tiles():
    """Where the Dgrad quantises, seen through scaled identity weights
    (H = I = 128, one lossless 128x128 block each: W_gate = 2^-3 I,
    W_up = 2^-4 I, W_down = 2^-2 I). Then dh = Q(dy) W_down = 2^-2 dy_hat,
    and dx = Q(dG) W_gate + Q(dU) W_up = 2^-3 dG_hat + 2^-4 dU_hat, element
    by element, with every hat the page's per-tile rule ("DeepSeek-V3
    Technical Report" (deepforge), "Per-tile FP8 scaling") applied along the
    rows. dG = dh U silu'(G) and dU = dh silu(G) use the forward's G and U
    from the dequantised x (silu and silu' are pinned above: brute-force
    loops and finite differences). Gaussian dy, x and activations are lossy
    under the rule, so an oracle that fed the unquantised dy, dG or dU to a
    Dgrad GEMM fails here."""
    from tests.test_oracle_experts import _page_tile_1x128
    rng = np.random.default_rng(55)
    rows = 6
    x = I.bf16_bits_to_f32(I.f32_to_bf16_bits(
        (rng.standard_normal((rows, 128)) * 2.0).astype(np.float32)))
    dy = (rng.standard_normal((rows, 128)) * 10.0 ** rng.uniform(-2, 2, (rows, 1))).astype(np.float32)
    cg, cu, cd = 2.0 ** -3, 2.0 ** -4, 2.0 ** -2
    wg, wu, wd = (O.dequantize_128x128(*O.quantize_128x128((np.eye(128) * c).astype(np.float32)))
                  for c in (cg, cu, cd))
    for m, c in ((wg, cg), (wu, cu), (wd, cd)):
        assert np.array_equal(m, np.eye(128) * c)             # lossless blocks
    xq, xs = O.quantize_1x128(x)
    q = O.expert_ffn_backward_q(xq, xs, x, dy, wg, wu, wd)
    dy_hat = _page_tile_1x128(dy)
    assert np.max(np.abs(dy_hat - dy)) > 1e-3 * np.max(np.abs(dy))   # dy's quantisation shows
    assert np.array_equal(q["dh"], cd * dy_hat)
    x_hat = _page_tile_1x128(x)
    g, u = cg * x_hat, cu * x_hat
    dh = cd * dy_hat
    d_g = dh * u * O.silu_grad(g)
    d_u = dh * O.silu(g)
    dg_hat, du_hat = _page_tile_1x128(d_g), _page_tile_1x128(d_u)
    for a, b in ((d_g, dg_hat), (d_u, du_hat)):
        assert np.max(np.abs(a - b)) > 1e-3 * np.max(np.abs(a))      # and dG's and dU's
    expect = cg * dg_hat + cu * du_hat
    assert np.max(np.abs(q["dx"] - expect)) <= 1e-12 * np.max(np.abs(expect))
