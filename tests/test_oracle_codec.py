"""Pins for the oracle's E4M3 codec and quantisers.

Each test checks the oracle against something other than itself: values the
FP8 format fixes (largest value 448, three mantissa bits, from "DeepSeek-V3
Technical Report" (deepforge.srivtx.xyz), "Per-tile FP8 scaling"), torch's own
float8_e4m3fn casts, the page's rounding rule restated independently, a
hand-worked example, and the outlier success criteria of the same page's
"Build it yourself" section.
"""
import math
import os

import numpy as np
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_decode_known_codes():
    d = O.E4M3_DECODE
    assert d[0x00] == 0.0 and not math.copysign(1.0, d[0x00]) < 0
    assert d[0x80] == 0.0 and math.copysign(1.0, d[0x80]) < 0
    assert d[0x38] == 1.0               # 0 0111 000: exponent equal to the bias
    assert d[0x7E] == 448.0             # largest finite value
    assert d[0xFE] == -448.0
    assert d[0x08] == 2.0 ** -6         # smallest normal
    assert d[0x01] == 2.0 ** -9         # smallest subnormal
    assert d[0x07] == 7 * 2.0 ** -9     # largest subnormal
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])
    assert np.sum(np.isnan(d)) == 2     # E4M3FN: no infinities, two NaNs
    assert np.nanmax(d) == 448.0


def test_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.e4m3_decode(np.arange(256, dtype=np.uint8))
    both_nan = np.isnan(ref) & np.isnan(ours)
    assert np.all(both_nan | (ref == ours))
    assert np.array_equal(np.signbit(ref[~both_nan]), np.signbit(ours[~both_nan]))


def test_roundtrip_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.e4m3_decode(codes)
    back = O.e4m3_encode(vals)
    finite = ~np.isnan(vals)
    assert finite.sum() == 254
    assert np.array_equal(back[finite], codes[finite])
    assert np.all(back[~finite] == 0x7F)


def test_eight_steps_per_binade():
    # three mantissa bits: each binade [2^k, 2^(k+1)) holds 8 equally spaced values
    pos = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)
    for e in range(1, 16):
        v = pos[(pos >= 2.0 ** (e - 7)) & (pos < 2.0 ** (e - 6))]
        assert len(v) == (8 if e < 15 else 7)
        assert np.allclose(np.diff(v), 2.0 ** (e - 10), rtol=0, atol=0)


def _page_rounding_rule(a):
    """The page's E4M3 rounding rule, restated: binade exponent clamped to
    [-6, 8], step 2^(e-3), magnitude rounded half-to-even to a multiple of
    the step, sign restored."""
    a = np.asarray(a, np.float64)
    mag = np.abs(a)
    e = np.clip(np.floor(np.log2(np.where(mag > 0, mag, 1.0))), -6, 8)
    step = 2.0 ** (e - 3)
    return np.where(mag > 0, np.sign(a) * np.round(mag / step) * step, 0.0)


def test_encode_matches_page_rule():
    rng = np.random.default_rng(11)
    mags = 2.0 ** rng.uniform(-12, math.log2(448.0), 200_000)
    v = (mags * rng.choice([-1.0, 1.0], mags.shape)).astype(np.float32).astype(np.float64)
    ours = O.e4m3_decode(O.e4m3_encode(v))
    assert np.array_equal(ours, _page_rounding_rule(v))


def test_encode_matches_torch_cast_random_and_midpoints():
    rng = np.random.default_rng(12)
    mags = 2.0 ** rng.uniform(-12, math.log2(448.0), 100_000)
    v = (mags * rng.choice([-1.0, 1.0], mags.shape)).astype(np.float32)
    pos = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)      # exact in fp32
    v = np.concatenate([v, mids, -mids, pos.astype(np.float32)])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(v), ref)


def test_encode_ties_to_even():
    # midpoint between 1.0 (0x38, even) and 1.125 (0x39): goes to 1.0;
    # midpoint between 1.125 and 1.25 (0x3A, even): goes to 1.25
    assert O.e4m3_encode(np.array([1.0625]))[0] == 0x38
    assert O.e4m3_encode(np.array([1.1875]))[0] == 0x3A
    # subnormal midpoint between 1*2^-9 (odd) and 2*2^-9 (even)
    assert O.e4m3_encode(np.array([1.5 * 2.0 ** -9]))[0] == 0x02
    # below half the smallest subnormal rounds to zero, exactly half goes to even 0
    assert O.e4m3_encode(np.array([0.5 * 2.0 ** -9]))[0] == 0x00
    assert O.e4m3_encode(np.array([0.51 * 2.0 ** -9]))[0] == 0x01


def test_encode_saturates():
    v = np.array([448.0, 449.0, 464.0, 1e6, np.inf, -500.0, -np.inf, np.nan, -0.0, 0.0])
    c = O.e4m3_encode(v)
    assert list(c) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F, 0x80, 0x00]


def test_half_ulp_bound():
    rng = np.random.default_rng(13)
    v = rng.standard_normal(100_000) * 30.0
    q = O.e4m3_decode(O.e4m3_encode(v))
    normal = np.abs(v) >= 2.0 ** -6
    assert np.all(np.abs(q - v)[normal] <= 2.0 ** -4 * np.abs(v)[normal])
    assert np.all(np.abs(q - v)[~normal] <= 2.0 ** -10)


# ---------------------------------------------------------------- quantisers

def test_per_tile_worked_example():
    rows = np.loadtxt(os.path.join(GOLDEN, "per_tile_example.txt"))
    x = np.zeros((1, 128), np.float32)
    x[0, :4] = rows[:, 0]
    q, s = O.quantize_1x128(x)
    fp8_vals = O.e4m3_decode(q[0, :4])
    assert np.array_equal(fp8_vals, rows[:, 1])
    assert np.all(q[0, 4:] == 0)
    deq = O.dequantize_1x128(q, s)[0, :4]
    # the page's scale is 448/2.5 in exact arithmetic; ours is its fp32 rounding
    assert np.allclose(deq, rows[:, 2], rtol=2e-7, atol=0)
    assert s[0, 0] == np.float32(448.0 / float(np.float32(2.5)))


def test_scale_is_correctly_rounded_fp32_division():
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((64, 512)) * rng.uniform(1e-3, 1e3, (64, 1))).astype(np.float32)
    _, s = O.quantize_1x128(x)
    amax = np.abs(x.reshape(64, 4, 128)).max(axis=2)
    # a double-precision divide of two floats, rounded once to float, is the
    # correctly rounded float quotient
    expect = np.array([[np.float32(448.0 / float(a)) for a in row] for row in amax], np.float32)
    assert np.array_equal(s, expect)


def test_amax_element_maps_to_448_and_zero_tile():
    rng = np.random.default_rng(15)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    x[3, 128:] = 0.0
    q, s = O.quantize_1x128(x)
    for r in range(8):
        for t in range(2):
            tile = x[r, 128 * t:128 * (t + 1)]
            if np.all(tile == 0):
                assert s[r, t] == 1.0 and np.all(q[r, 128 * t:128 * (t + 1)] == 0)
                continue
            j = int(np.argmax(np.abs(tile)))
            assert q[r, 128 * t + j] == (0xFE if tile[j] < 0 else 0x7E)


def test_quantised_error_bound():
    rng = np.random.default_rng(16)
    x = (rng.standard_normal((32, 384)) * 5).astype(np.float32)
    q, s = O.quantize_1x128(x)
    deq = O.dequantize_1x128(q, s)
    scaled = np.abs(x.reshape(32, 3, 128) * s[:, :, None].astype(np.float64)).reshape(32, 384)
    sc = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(deq - x)
    normal = scaled >= 2.0 ** -6
    # half an ulp of E4M3 plus the float32 rounding of x * scale
    assert np.all(err[normal] <= (2.0 ** -4 + 2.0 ** -22) * np.abs(x[normal]))
    assert np.all(err[~normal] <= (2.0 ** -10) / sc[~normal] + 1e-30)


def test_outlier_success_criteria():
    """Per-tensor scaling with one outlier crushes the small values (relative
    error above 0.5 on a tile without the outlier); 128-element tiles bring
    the error below 0.05 ("Build it yourself", success criteria)."""
    rng = np.random.default_rng(17)
    x = (rng.standard_normal(1024) * 1e-5).astype(np.float32)
    x[5] = 1e3
    tile = slice(256, 384)  # a tile without the outlier
    s_tensor = np.float32(448.0) / np.float32(np.abs(x).max())
    deq_tensor = O.e4m3_decode(O.e4m3_encode((x * s_tensor).astype(np.float32))) / float(s_tensor)
    rel_tensor = np.linalg.norm(deq_tensor[tile] - x[tile]) / np.linalg.norm(x[tile])
    q, s = O.quantize_1x128(x[None, :])
    deq_tile = O.dequantize_1x128(q, s)[0]
    rel_tile = np.linalg.norm(deq_tile[tile] - x[tile]) / np.linalg.norm(x[tile])
    assert rel_tensor > 0.5
    assert rel_tile < 0.05


def test_block_quantiser_transpose_symmetry():
    rng = np.random.default_rng(18)
    w = rng.standard_normal((384, 256)).astype(np.float32) * rng.uniform(0.1, 10, (384, 1)).astype(np.float32)
    q, s = O.quantize_128x128(w)
    qt, st = O.quantize_128x128(np.ascontiguousarray(w.T))
    assert s.shape == (3, 2) and st.shape == (2, 3)
    assert np.array_equal(q.T, qt) and np.array_equal(s.T, st)


def test_block_quantiser_block_amax():
    rng = np.random.default_rng(19)
    w = rng.standard_normal((256, 384)).astype(np.float32)
    w[130, 7] = 50.0  # block (1, 0)
    q, s = O.quantize_128x128(w)
    assert s[1, 0] == np.float32(448.0 / 50.0)
    assert q[130, 7] == 0x7E
    # a power-of-two rescaling of one block leaves its codes and moves its scale exactly
    w2 = w.copy()
    w2[:128, 128:256] *= 8.0
    q2, s2 = O.quantize_128x128(w2)
    assert np.array_equal(q2, q)
    assert s2[0, 1] * 8 == s[0, 1]
    assert np.array_equal(np.delete(s2, 1, axis=1), np.delete(s, 1, axis=1))



def test_round_bf16_against_torch_and_ties():
    """bf16 rounding of the expert outputs: torch's float -> bfloat16 cast on
    values exactly representable in float32 (so torch rounds once), the
    even significand on exact midpoints, and one rounding from the exact
    float64 value (no double rounding through float32)."""
    rng = np.random.default_rng(30)
    v = (rng.standard_normal(50_000) * 10 ** rng.uniform(-6, 6, 50_000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(v.astype(np.float64)), ref)
    assert O.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert O.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6
    assert O.round_bf16(np.array([-(1.0 + 3 * 2.0 ** -8)]))[0] == -(1.0 + 2.0 ** -6)
    # just above a midpoint rounds up even where float32 would land on it
    assert O.round_bf16(np.array([1.0 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1.0 + 2.0 ** -7
    assert O.round_bf16(np.array([0.0]))[0] == 0.0
