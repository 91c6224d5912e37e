"""The synthetic inputs follow their stated recipe (no GPU).

Sizes of every workload; seeded, reproducible streams; x ~ N(0, 1) rounded
to bf16; the outlier workload's 1% of channels (72 of 7168) scaled by 20; the
skewed workload's mean logits alpha * r_i^-1.2 over a seeded permutation of
the ranks; the bias ranges; weights N(0, 1/fan_in) in 128x128 pool blocks.
"""
import numpy as np
import pytest

from mixture_experts_layer_40_b200 import inputs as I

SIZES = {   # name: (T, H, N, K, I, bias range)
    "tiny": (64, 256, 16, 4, 128, 0.1),
    "v3_prefill": (4096, 7168, 256, 8, 2048, 0.0),
    "skewed": (8192, 7168, 256, 8, 2048, 0.0),
    "large_prefill": (32768, 7168, 256, 8, 2048, 0.05),
    "decode": (128, 7168, 256, 8, 2048, 0.05),
}


@pytest.mark.parametrize("name", sorted(SIZES))
def test_workload_sizes(name):
    w = I.WORKLOADS[name]
    assert (w.T, w.H, w.N, w.K, w.I, w.bias_range) == SIZES[name]
    assert w.H % 256 == 0 and w.I % 128 == 0 and w.K <= w.N


def test_streams_are_seeded_and_distinct():
    w = I.WORKLOADS["tiny"]
    assert np.array_equal(I.make_x(w), I.make_x(w))
    assert not np.array_equal(I.make_x(w, step=0), I.make_x(w, step=1))
    other = I.Workload("tiny", T=64, H=256, N=16, K=4, I=128, bias_range=0.1, seed=1)
    assert not np.array_equal(I.make_x(w), I.make_x(other))
    assert np.array_equal(I.make_gate_w(w), I.make_gate_w(w))
    assert np.array_equal(I.make_bias(w), I.make_bias(w))


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is halfway between bf16 neighbours 1 and 1 + 2^-7: ties to even (1)
    a = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], np.float32)
    back = I.bf16_bits_to_f32(I.f32_to_bf16_bits(a))
    assert back.tolist() == [1.0, 1.0 + 2.0 ** -6, -2.5, 0.0]


def test_x_is_standard_normal_in_bf16():
    w = I.WORKLOADS["v3_prefill"]
    x = I.bf16_bits_to_f32(I.make_x(w, rows=512))
    assert x.shape == (512, w.H)
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1.0) < 0.01
    # every value is a bf16 value: the low 16 bits of its float32 are zero
    assert not np.any(x.view(np.uint32) & np.uint32(0xFFFF))


def test_outlier_channels():
    w = I.WORKLOADS["large_prefill"]
    ch = I.outlier_channels(w)
    assert len(ch) == 72 and len(set(ch.tolist())) == 72 and ch.max() < w.H
    x = I.bf16_bits_to_f32(I.make_x(w, rows=1024)).astype(np.float64)
    rms = np.sqrt(np.mean(x ** 2, axis=0))
    mask = np.zeros(w.H, bool)
    mask[ch] = True
    assert np.all(np.abs(rms[mask] / 20.0 - 1.0) < 0.15)
    assert np.all(np.abs(rms[~mask] - 1.0) < 0.15)


def test_skewed_mean_logits_follow_the_power_law():
    w = I.WORKLOADS["skewed"]
    x = I.bf16_bits_to_f32(I.make_x(w, rows=2048)).astype(np.float64)
    g = I.make_gate_w(w).astype(np.float64)
    mean_logit = (x @ g.T).mean(axis=0)
    ranks = np.random.default_rng([w.seed, 9]).permutation(w.N) + 1
    expect = 4.0 * ranks.astype(np.float64) ** -1.2
    # E[x . e_i] = |d|^2 * alpha r_i^-1.2 = alpha r_i^-1.2 (d a unit vector);
    # the sampling noise of a mean over 2048 tokens is about 1/sqrt(2048)
    assert np.max(np.abs(mean_logit - expect)) < 0.1
    assert np.argmax(mean_logit) == np.argmin(ranks)


def test_bias_ranges():
    for name, (*_, r) in SIZES.items():
        b = I.make_bias(I.WORKLOADS[name])
        assert b.dtype == np.float32 and b.shape == (I.WORKLOADS[name].N,)
        if r == 0:
            assert not b.any()
        else:
            assert np.all(np.abs(b) <= r) and np.abs(b).max() > 0.8 * r


def test_weight_pool_blocks():
    w = I.WORKLOADS["tiny"]
    p = I.make_weight_pool(w)
    ib, hb = w.I // 128, w.H // 128
    assert p.slot_gate.shape == (w.E, ib, hb) and p.slot_down.shape == (w.E, hb, ib)
    # small workloads: every block position has its own pool block
    used = np.concatenate([p.slot_gate.ravel(), p.slot_up.ravel()])
    assert len(set(used.tolist())) == used.size == p.pool13.shape[0]
    assert abs(float(p.pool13.std()) * np.sqrt(w.H) - 1.0) < 0.02
    assert abs(float(p.pool2.std()) * np.sqrt(w.I) - 1.0) < 0.02
    g = I.make_gate_w(w)
    assert abs(float(g.std()) * np.sqrt(w.H) - 1.0) < 0.05
