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
