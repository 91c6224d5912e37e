"""Pins for the oracle's node-limited routing and sequence-wise balance
statistics.

Node-limited routing ("DeepSeek-V3, explained", recipe step 5; "DeepSeek-V3
Technical Report" (deepforge.srivtx.xyz), "Balancing without a balance
loss"): hand-worked cases in tests/golden/node_limited_routing.txt; with
every group eligible it is plain top-K; every token's experts lie in at most
M groups.

Balance statistics ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
Multi-Token Prediction, and FP8 Training at 671B Scale", section III, the
complementary sequence-wise loss): sum_i f_i = N and sum_i P_i = 1 per
sequence; an even split gives f_i = 1 and L = alpha; a hand-worked case in
exact binary fractions.
"""
import os

import numpy as np
import pytest

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "node_limited_routing.txt")


def _golden_cases():
    cases = []
    for ln in open(GOLDEN):
        if not ln.startswith("case "):
            continue
        fields = {}
        for part in ln.split("|"):
            key, *vals = part.split()
            fields[key] = vals
        cases.append(fields)
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["case"][0])
def test_node_limited_hand_cases(case):
    z = np.array([float(v) for v in case["z"]], np.float32)
    bias = np.array([float(v) for v in case["bias"]], np.float32)
    x = np.ones((1, 1), np.float32)
    gate_w = z.reshape(16, 1)
    ids, gates, s, score, gscore = O.route_grouped(x, gate_w, bias, 4, 4, 2)
    assert ids[0].tolist() == [int(v) for v in case["ids"]]
    np.testing.assert_allclose(gates[0], [float(v) for v in case["gates"]], atol=5e-9)
    plain, *_ = O.route(x, gate_w, bias, 4)
    assert plain[0].tolist() == [int(v) for v in case["plain"]]
    if case["case"][0] == "a":
        # sigmoid(4) + sigmoid(-4) = 1: the closed form of group 0's score
        assert abs(gscore[0, 0] - 1.0) < 1e-15


def test_all_groups_eligible_is_plain_topk():
    w = I.Workload("g", T=64, H=256, N=64, K=8, I=128, bias_range=0.1, seed=3)
    x = I.bf16_bits_to_f32(I.make_x(w))
    gw, b = I.make_gate_w(w), I.make_bias(w)
    ids_p, gates_p, _, _ = O.route(x, gw, b, w.K)
    for groups, top in [(8, 8), (4, 4), (1, 1)]:
        ids, gates, *_ = O.route_grouped(x, gw, b, w.K, groups, top)
        assert np.array_equal(ids, ids_p)
        assert np.array_equal(gates, gates_p)


def test_node_limited_invariants():
    w = I.Workload("g", T=200, H=256, N=64, K=8, I=128, bias_range=0.1, seed=4)
    x = I.bf16_bits_to_f32(I.make_x(w))
    gw, b = I.make_gate_w(w), I.make_bias(w)
    groups, top = 8, 4
    ids, gates, s, score, gscore = O.route_grouped(x, gw, b, w.K, groups, top)
    size = w.N // groups
    for t in range(w.T):
        used = set(int(e) // size for e in ids[t])
        assert len(used) <= top
        # the used groups are among the M best group scores
        best = np.sort(gscore[t])[::-1][top - 1]
        assert all(gscore[t, g] >= best for g in used)
        # inside the eligible groups, the K chosen have the K highest scores
        elig = [g for g in np.argsort(-gscore[t], kind="stable")[:top]]
        pool = np.concatenate([np.arange(g * size, (g + 1) * size) for g in elig])
        kth = np.sort(score[t, pool])[::-1][w.K - 1]
        assert np.all(score[t, ids[t]] >= kth)
        assert len(set(ids[t].tolist())) == w.K
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, rtol=1e-14)


def test_balance_stats_closed_forms():
    rng = np.random.default_rng(5)
    t_count, n, k = 37, 32, 4
    s = rng.uniform(0.01, 0.99, (t_count, n))
    ids = np.stack([rng.choice(n, k, replace=False) for _ in range(t_count)])
    f, p, loss = O.balance_stats(s, ids, k, seq_len=10, alpha=1e-4)
    assert f.shape == (4, n) and loss.shape == (4,)
    np.testing.assert_allclose(f.sum(axis=1), n, rtol=1e-14)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(loss, 1e-4 * np.sum(f * p, axis=1), rtol=1e-14)


def test_balance_stats_even_split_gives_alpha():
    n, k, t_count = 8, 2, 8   # each expert chosen exactly k * t / n = 2 times
    ids = np.array([[t % n, (t + 4) % n] for t in range(t_count)])
    s = np.random.default_rng(6).uniform(0.1, 0.9, (t_count, n))
    f, p, loss = O.balance_stats(s, ids, k, seq_len=t_count, alpha=1e-4)
    np.testing.assert_array_equal(f, 1.0)
    assert abs(loss[0] - 1e-4) < 1e-18


def test_balance_stats_hand_case():
    # N = 4, K = 1, one sequence of two tokens; affinities in binary fractions
    s = np.array([[0.5, 0.25, 0.125, 0.125], [0.25, 0.25, 0.25, 0.25]])
    ids = np.array([[0], [2]])
    f, p, loss = O.balance_stats(s, ids, 1, seq_len=2, alpha=1e-4)
    assert f[0].tolist() == [2.0, 0.0, 2.0, 0.0]          # 4 / (1 * 2) * counts
    assert p[0].tolist() == [0.375, 0.25, 0.1875, 0.1875]  # column means of s / row sums
    assert abs(loss[0] - 1.125e-4) < 1e-19                # 1e-4 * (2 * .375 + 2 * .1875)


def test_balance_stats_ragged_last_sequence():
    s = np.full((5, 4), 0.5)
    ids = np.array([[0], [1], [2], [3], [3]])
    f, p, loss = O.balance_stats(s, ids, 1, seq_len=2, alpha=1.0)
    assert f.shape == (3, 4)
    assert f[2].tolist() == [0.0, 0.0, 0.0, 4.0]   # one token: 4 / (1 * 1)
    assert p[2].tolist() == [0.25] * 4
    assert abs(loss[2] - 1.0) < 1e-15
