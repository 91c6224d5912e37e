"""Pins for the oracle's routing, permutation and bias controller.

Against what the pages fix ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load
Balancing, Multi-Token Prediction, and FP8 Training at 671B Scale", section
III; "DeepSeek-V3, explained", recipe steps 4-5 and the symbol notes):
sigmoid affinities scored independently; the bias only decides selection;
gates are the unbiased affinities normalised over the K chosen; every token
gets exactly K experts; overloaded experts lose gamma, underloaded gain it;
gamma = 0 freezes the biases.
"""
import math
from fractions import Fraction

import numpy as np

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I


def _tiny():
    w = I.WORKLOADS["tiny"]
    x = I.bf16_bits_to_f32(I.make_x(w))
    return w, x, I.make_gate_w(w), I.make_bias(w)


def test_logits_exact_on_small_case():
    rng = np.random.default_rng(1)
    x = I.bf16_bits_to_f32(I.f32_to_bf16_bits(rng.standard_normal((3, 20)).astype(np.float32)))
    g = rng.standard_normal((5, 20)).astype(np.float32)
    z = O.gate_logits(x, g)
    assert z.shape == (3, 5)
    for t in range(3):
        for i in range(5):
            exact = sum(Fraction(float(x[t, h])) * Fraction(float(g[i, h])) for h in range(20))
            assert abs(z[t, i] - float(exact)) <= 1e-14 * (1 + abs(float(exact)))


def test_sigmoid_closed_forms():
    assert O.sigmoid(np.array(0.0)) == 0.5
    z = np.linspace(-30, 30, 101)
    assert np.allclose(O.sigmoid(z) + O.sigmoid(-z), 1.0, rtol=0, atol=1e-15)
    assert abs(O.sigmoid(np.array(math.log(3.0))) - 0.75) < 1e-15


def test_hand_built_routing():
    # centroids along one axis: z_i = c_i for x = e_0
    c = np.array([0.1, 2.0, -1.0, 3.0, 0.5, 2.0], np.float32)
    g = np.zeros((6, 4), np.float32)
    g[:, 0] = c
    x = np.zeros((1, 4), np.float32)
    x[0, 0] = 1.0
    s = [1.0 / (1.0 + math.exp(-float(ci))) for ci in c]
    # no bias: top-2 by affinity is experts 3, then the tie 1 vs 5 -> lower id 1
    ids, gates, _, _ = O.route(x, g, np.zeros(6, np.float32), 2)
    assert list(ids[0]) == [3, 1]
    assert np.allclose(gates[0], [s[3] / (s[3] + s[1]), s[1] / (s[3] + s[1])], rtol=1e-15)
    # a bias on expert 2 lifts it into the top-2, yet its gate is its unbiased affinity
    b = np.zeros(6, np.float32)
    b[2] = 0.9
    ids, gates, _, _ = O.route(x, g, b, 2)
    assert list(ids[0]) == [2, 3] if s[2] + 0.9 > s[3] else list(ids[0]) == [3, 2]
    assert set(ids[0]) == {2, 3}
    gsum = s[2] + s[3]
    got = dict(zip(ids[0], gates[0]))
    assert abs(got[2] - s[2] / gsum) < 1e-15 and abs(got[3] - s[3] / gsum) < 1e-15


def test_route_invariants_tiny():
    w, x, g, b = _tiny()
    ids, gates, s, score = O.route(x, g, b, w.K)
    assert ids.shape == (w.T, w.K)
    for t in range(w.T):
        assert len(set(ids[t])) == w.K
        chosen = set(ids[t])
        rest = [i for i in range(w.N) if i not in chosen]
        # every chosen biased score beats every other one (brute force)
        assert min(score[t, list(chosen)]) >= max(score[t, rest])
        # output order: biased score descending
        assert np.all(np.diff(score[t, ids[t]]) <= 0)
    assert np.allclose(gates.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(gates > 0)
    assert O.expert_counts(ids, w.N).sum() == w.T * w.K


def test_zero_bias_is_pure_affinity_topk():
    w, x, g, _ = _tiny()
    ids, _, s, _ = O.route(x, g, np.zeros(w.N, np.float32), w.K)
    for t in range(w.T):
        ranked = sorted(range(w.N), key=lambda i: (-s[t, i], i))
        assert list(ids[t]) == ranked[:w.K]


def test_bias_decides_which_not_how_much():
    w, x, g, b = _tiny()
    ids, gates, _, _ = O.route(x, g, b, w.K)
    # a uniform shift of every bias keeps every selection: gates bit-identical
    ids2, gates2, _, _ = O.route(x, g, (b + np.float32(0.25)).astype(np.float32), w.K)
    assert np.array_equal(ids, ids2) and np.array_equal(gates, gates2)
    # a bias that changes the selection changes the gates only through the set
    b3 = b.copy()
    b3[ids[0, 0]] = -10.0
    ids3, gates3, s3, _ = O.route(x, g, b3, w.K)
    assert ids[0, 0] not in ids3[0]
    sel = s3[0, ids3[0]]
    assert np.array_equal(gates3[0], sel / sel.sum())


def test_ties_break_to_lower_id():
    rng = np.random.default_rng(3)
    g = rng.standard_normal((8, 16)).astype(np.float32)
    g[6] = g[2]                     # experts 2 and 6 identical
    x = rng.standard_normal((50, 16)).astype(np.float32)
    ids, _, s, _ = O.route(x, g, np.zeros(8, np.float32), 3)
    for t in range(50):
        r = list(ids[t])
        if 6 in r:
            assert 2 in r and r.index(2) < r.index(6)


def test_permutation_definition():
    w, x, g, b = _tiny()
    ids, _, _, _ = O.route(x, g, b, w.K)
    offsets, tokens, rank = O.permutation(ids, w.N)
    counts = O.expert_counts(ids, w.N)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    for e in range(w.N):
        seg = tokens[offsets[e]:offsets[e + 1]]
        expect = [t for t in range(w.T) if e in ids[t]]
        assert list(seg) == expect
    for t in range(w.T):
        for k in range(w.K):
            assert tokens[offsets[ids[t, k]] + rank[t, k]] == t


def test_bias_update_hand_built_loads():
    gamma = 1e-3
    # N=4, T=8, K=2: mean load 4
    b = np.array([0.0, 0.0, 0.5, -0.25], np.float32)
    nb = O.update_bias(b, np.array([6, 2, 4, 4]), 8, 2, gamma)
    g32 = np.float32(gamma)
    assert nb[0] == -g32 and nb[1] == g32
    assert nb[2] == b[2] and nb[3] == b[3]
    # a mean that is not an integer (T*K/N = 1.5)
    nb = O.update_bias(np.zeros(2, np.float32), np.array([2, 1]), 3, 1, gamma)
    assert nb[0] == -g32 and nb[1] == g32


def test_bias_update_float32_rounding():
    b = np.array([1.0, 1.0], np.float32)
    nb = O.update_bias(b, np.array([3, 1]), 2, 2, 1e-3)
    g = float(np.float32(1e-3))
    # exact double result of a float32 add, then one rounding to float32
    assert nb[0] == np.float32(1.0 - g) and nb[1] == np.float32(1.0 + g)
    assert nb.dtype == np.float32
    # biases where adding the float32 gamma and adding the float64 1e-3 round
    # to different float32 values: the update is the float32 add (gamma = 1e-3f)
    b = np.array([-4.167452425463125e-05, 0.004282602109014988], np.float32)
    nb = O.update_bias(b, np.array([1, 3]), 2, 2, 1e-3)
    assert nb[0] == np.float32(float(b[0]) + g) and nb[1] == np.float32(float(b[1]) - g)
    assert nb[0] != np.float32(float(b[0]) + 1e-3) and nb[1] != np.float32(float(b[1]) - 1e-3)


def test_gamma_zero_freezes_bias():
    w, x, g, b = _tiny()
    ids, _, _, _ = O.route(x, g, b, w.K)
    c = O.expert_counts(ids, w.N)
    assert np.array_equal(O.update_bias(b, c, w.T, w.K, 0.0), b)


def test_bias_update_moves_load_toward_mean():
    """Repeated updates on a skewed toy router shrink the max/mean load."""
    rng = np.random.default_rng(5)
    n, k, t = 16, 2, 512
    g = rng.standard_normal((n, 32)).astype(np.float32)
    g[0] += 3.0   # expert 0 is hot for most tokens
    x = (rng.standard_normal((t, 32)) + 0.3).astype(np.float32)
    b = np.zeros(n, np.float32)
    first = None
    for _ in range(200):
        ids, _, _, _ = O.route(x, g, b, k)
        c = O.expert_counts(ids, n)
        if first is None:
            first = c.max() / c.mean()
        b = O.update_bias(b, c, t, k, 5e-3)
    last = c.max() / c.mean()
    assert first > 2.0 and last < 0.6 * first
