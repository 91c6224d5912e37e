"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's source (a flipped
sign, a dropped term, a transposed operand or tile, a wrong rounding, a
missing quantisation), loads the copy as a separate module, and runs the pin
that must catch it with the copy in place of the oracle. The planted copy
never replaces the oracle itself; nothing here touches the GPU path. The
pins named are the independent ones (closed forms, worked examples of the
pages, brute-force loops, finite differences, hand-built cases, library
casts), so a pass here shows that each part of the oracle is held by
something other than itself.
"""
import importlib
import os
import types

import pytest

ORACLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "oracle", "moe_oracle.py")

# (mistake, original text, planted text, pin module, pin test)
CASES = [
    ("sigmoid sign", "return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))",
     "return 1.0 / (1.0 + np.exp(np.asarray(z, np.float64)))",
     "test_oracle_router", "test_sigmoid_closed_forms"),
    ("gates from the biased score",
     "    sel = np.take_along_axis(s, ids, axis=1)\n    gates = sel / np.sum(sel, axis=1, keepdims=True)\n    return ids, gates, s, score\n",
     "    sel = np.take_along_axis(score, ids, axis=1)\n    gates = sel / np.sum(sel, axis=1, keepdims=True)\n    return ids, gates, s, score\n",
     "test_oracle_router", "test_hand_built_routing"),
    ("ties to the higher expert id",
     "    order = np.argsort(-score, axis=1, kind=\"stable\")\n    ids = order[:, :k]",
     "    order = score.shape[1] - 1 - np.argsort(-score[:, ::-1], axis=1, kind=\"stable\")\n    ids = order[:, :k]",
     "test_oracle_router", "test_hand_built_routing"),
    ("bias update sign flipped", "    delta = np.sign(np.int64(t_count)", "    delta = -np.sign(np.int64(t_count)",
     "test_oracle_router", "test_bias_update_hand_built_loads"),
    ("bias compared with a rounded mean",
     "    delta = np.sign(np.int64(t_count) * np.int64(k)\n                    - np.int64(n)",
     "    delta = np.sign(np.int64(t_count * k // n) * np.int64(n)\n                    - np.int64(n)",
     "test_oracle_router", "test_bias_update_hand_built_loads"),
    ("permutation with tokens descending",
     "    for t in range(t_count):\n        for j in range(k):",
     "    for t in reversed(range(t_count)):\n        for j in range(k):",
     "test_oracle_router", "test_permutation_definition"),
    ("scale amax / 448", "        s = np.float32(E4M3_MAX) / amax_f32", "        s = amax_f32 / np.float32(E4M3_MAX)",
     "test_oracle_codec", "test_per_tile_worked_example"),
    ("zero tile scaled by 0", "    return np.where(amax_f32 > 0, s, np.float32(1.0)).astype(np.float32)",
     "    return np.where(amax_f32 > 0, s, np.float32(0.0)).astype(np.float32)",
     "test_oracle_codec", "test_amax_element_maps_to_448_and_zero_tile"),
    ("one activation scale per row", "    amax = np.max(np.abs(xt), axis=2)\n",
     "    amax = np.repeat(np.max(np.abs(xt), axis=(1, 2))[:, None], cols // TILE, axis=1)\n",
     "test_oracle_codec", "test_scale_is_correctly_rounded_fp32_division"),
    ("ties away from zero", "    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))", "    take_hi = (d_hi <= d_lo)",
     "test_oracle_codec", "test_encode_matches_torch_cast_random_and_midpoints"),
    ("exponent bias 8",
     "            table[code] = sign * (1.0 + man_field / 8.0) * 2.0 ** (exp_field - 7)",
     "            table[code] = sign * (1.0 + man_field / 8.0) * 2.0 ** (exp_field - 8)",
     "test_oracle_codec", "test_decode_known_codes"),
    ("dequantisation multiplies by the scale",
     "    return (v / np.asarray(scales, np.float64)[:, :, None]).reshape(rows, cols)",
     "    return (v * np.asarray(scales, np.float64)[:, :, None]).reshape(rows, cols)",
     "test_oracle_codec", "test_per_tile_worked_example"),
    ("bf16 rounding truncates", "    return np.ldexp(np.round(m * 256.0) / 256.0, e)",
     "    return np.ldexp(np.trunc(m * 256.0) / 256.0, e)",
     "test_oracle_codec", "test_round_bf16_against_torch_and_ties"),
    ("silu replaced by sigmoid", "    return a / (1.0 + np.exp(-a))", "    return 1.0 / (1.0 + np.exp(-a))",
     "test_oracle_experts", "test_swiglu_brute_force_loops"),
    ("SwiGLU operands swapped",
     "    h = silu(g) * u\n    hq, hs = quantize_1x128(h.astype(np.float32))",
     "    h = silu(u) * g\n    hq, hs = quantize_1x128(h.astype(np.float32))",
     "test_oracle_experts", "test_h_requantisation_seen_through_identity_down_weights"),
    ("h not re-quantised",
     "    _, hq, hs = expert_up_q(xq, xs, wg_deq, wu_deq)\n    return round_bf16(expert_down_q(hq, hs, wd_deq)), hq, hs",
     "    h, hq, hs = expert_up_q(xq, xs, wg_deq, wu_deq)\n    return round_bf16(h @ wd_deq.T), hq, hs",
     "test_oracle_experts", "test_h_requantisation_seen_through_identity_down_weights"),
    ("expert output not rounded to bf16",
     "    return round_bf16(expert_down_q(hq, hs, wd_deq)), hq, hs", "    return expert_down_q(hq, hs, wd_deq), hq, hs",
     "test_oracle_experts", "test_h_requantisation_seen_through_identity_down_weights"),
    ("combine without the shared expert", "    out = np.array(y_shared, dtype=np.float64, copy=True)",
     "    out = np.zeros_like(np.asarray(y_shared, dtype=np.float64))",
     "test_oracle_experts", "test_sparse_equals_dense_then_mask"),
    ("combine without the gates", "            out[t] += gates[t, j] * y_routed[t, j]", "            out[t] += y_routed[t, j]",
     "test_oracle_experts", "test_sparse_equals_dense_then_mask"),
    ("forced routing gated by biased scores",
     "        sel = np.take_along_axis(s, ids, axis=1)\n        gates = sel / np.sum(sel, axis=1, keepdims=True)\n    counts = expert_counts(ids, n)",
     "        sel = np.take_along_axis(s + np.asarray(bias, np.float32), ids, axis=1)\n        gates = sel / np.sum(sel, axis=1, keepdims=True)\n    counts = expert_counts(ids, n)",
     "test_oracle_experts", "test_forced_routing_keeps_the_unbiased_gates"),
    ("group score from unbiased affinities", "    grouped = score.reshape(t_count, n_groups, size)",
     "    grouped = s.reshape(t_count, n_groups, size)",
     "test_oracle_routing_ext", "node_limited_golden_cases"),
    ("load fraction without N / K", "        f[q] = n * counts / (k * t_seq)", "        f[q] = counts / t_seq",
     "test_oracle_routing_ext", "test_balance_stats_closed_forms"),
    ("silu' wrong", "    return sg * (1.0 + g * (1.0 - sg))", "    return sg * (1.0 - sg)",
     "test_oracle_backward", "test_dx_matches_finite_differences"),
    ("Dgrad on the unquantised dy", "    dh = dequantize_1x128(dyq, dys) @ wd", "    dh = np.asarray(dy, np.float64) @ wd",
     "test_oracle_backward", "test_dgrad_quantises_dy_and_dg_du_in_row_tiles"),
    ("Dgrad on the unquantised dG",
     "    dx = dequantize_1x128(dgq, dgs) @ wg + dequantize_1x128(duq, dus) @ wu",
     "    dx = d_g @ wg + dequantize_1x128(duq, dus) @ wu",
     "test_oracle_backward", "test_dgrad_quantises_dy_and_dg_du_in_row_tiles"),
    ("Wgrad with h tiled along the rows",
     "    dwd = q(np.asarray(dy, np.float32)).T @ q(h.astype(np.float32))",
     "    dwd = q(np.asarray(dy, np.float32)).T @ dequantize_1x128(*quantize_1x128(h.astype(np.float32)))",
     "test_oracle_backward", "test_wgrad_down_uses_h_quantised_down_its_columns"),
    ("Wgrad on the dequantised x_hat", "    dwg = q(d_g.astype(np.float32)).T @ q(x32)",
     "    dwg = q(d_g.astype(np.float32)).T @ q(x_hat.astype(np.float32))",
     "test_oracle_backward", "test_wgrad_up_uses_x_quantised_down_its_columns"),
    ("routed dY not scaled by the gate",
     "            dy_rows = gates[rr, kk][:, None] * dy[rr].astype(np.float64)",
     "            dy_rows = dy[rr].astype(np.float64)",
     "test_oracle_backward", "test_dx_matches_finite_differences"),
    ("gate gradient times the gate",
     "            dgates[rr, kk] = np.sum(dy[rr].astype(np.float64) * y_e, axis=1)",
     "            dgates[rr, kk] = gates[rr, kk] * np.sum(dy[rr].astype(np.float64) * y_e, axis=1)",
     "test_oracle_backward", "test_gate_gradients_are_dy_dot_expert_output"),
    ("gate logits in float32",
     "    return np.asarray(x, np.float64) @ np.asarray(gate_w, np.float64).T",
     "    return (np.asarray(x, np.float32) @ np.asarray(gate_w, np.float32).T).astype(np.float64)",
     "test_oracle_router", "test_logits_exact_on_small_case"),
    ("counts off by one for expert 0",
     "    return np.bincount(np.asarray(ids).ravel(), minlength=n_experts).astype(np.int32)",
     "    return (np.bincount(np.asarray(ids).ravel(), minlength=n_experts) + (np.arange(n_experts) == 0)).astype(np.int32)",
     "test_oracle_router", "test_route_invariants_tiny"),
    ("bias update in float64", "    return (bias + step).astype(np.float32)",
     "    return (bias.astype(np.float64) + float(gamma) * delta).astype(np.float32)",
     "test_oracle_router", "test_bias_update_float32_rounding"),
    ("negative zero loses its sign", "    codes = np.where(neg, mag | 0x80, mag).astype(np.uint8)",
     "    codes = np.where(neg & (mag > 0), mag | 0x80, mag).astype(np.uint8)",
     "test_oracle_codec", "test_roundtrip_all_codes"),
    ("subnormal exponent off by one",
     "            table[code] = sign * (man_field / 8.0) * 2.0 ** (1 - 7)",
     "            table[code] = sign * (man_field / 8.0) * 2.0 ** (0 - 7)",
     "test_oracle_codec", "test_decode_known_codes"),
    ("weight blocks assembled transposed",
     "        return m.transpose(0, 2, 1, 3).reshape(nb * TILE, kb * TILE)",
     "        return m.transpose(0, 3, 1, 2).reshape(nb * TILE, kb * TILE)",
     "test_oracle_experts", "test_assembly_places_pool_blocks"),
    ("gate mass not normalised",
     "        p[q] = np.sum(s[lo:hi] / np.sum(s[lo:hi], axis=1, keepdims=True), axis=0) / t_seq",
     "        p[q] = np.sum(s[lo:hi], axis=0) / t_seq",
     "test_oracle_routing_ext", "test_balance_stats_closed_forms"),
    ("balance loss without alpha", "        loss[q] = alpha * np.sum(f[q] * p[q])",
     "        loss[q] = np.sum(f[q] * p[q])",
     "test_oracle_routing_ext", "test_balance_stats_closed_forms"),
    ("dU from U instead of silu(G)", "    d_u = dh * silu(g)\n    dgq", "    d_u = dh * u\n    dgq",
     "test_oracle_backward", "test_dgrad_quantises_dy_and_dg_du_in_row_tiles"),
    ("dW_up from dG", "    dwu = q(d_u.astype(np.float32)).T @ q(x32)",
     "    dwu = q(d_g.astype(np.float32)).T @ q(x32)",
     "test_oracle_backward", "test_wgrad_up_uses_x_quantised_down_its_columns"),
    ("128x1 tiles run along the columns",
     "    return quantize_1x128(np.ascontiguousarray(pad.T))",
     "    c2, s2 = quantize_1x128(np.ascontiguousarray(pad))\n    return quantize_1x128(np.ascontiguousarray(dequantize_1x128(c2, s2).astype(np.float32).T))",
     "test_oracle_backward", "test_quantize_128x1_tiles_run_down_the_rows"),
    ("backward without the shared expert", "    for e in list(np.unique(ids[keep])) + [n]:",
     "    for e in list(np.unique(ids[keep])):",
     "test_oracle_backward", "test_dx_matches_finite_differences"),
]


def _planted(old: str, new: str) -> types.ModuleType:
    src = open(ORACLE).read()
    assert src.count(old) == 1, "the planted text must match one place in the oracle"
    mod = types.ModuleType("moe_oracle_planted")
    mod.__file__ = ORACLE
    exec(compile(src.replace(old, new), ORACLE + " (planted)", "exec"), mod.__dict__)
    return mod


def _all_golden_cases(tmod):
    """Every hand-built node-limited case of the golden file, as one pin."""
    def run():
        for case in tmod._golden_cases():
            tmod.test_node_limited_hand_cases(case)
    return run


@pytest.mark.parametrize("name,old,new,pin_module,pin", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_fails_its_pin(name, old, new, pin_module, pin, monkeypatch):
    tmod = importlib.import_module("tests." + pin_module)
    pin_fn = _all_golden_cases(tmod) if pin == "node_limited_golden_cases" else getattr(tmod, pin)
    pin_fn()                                   # the pin holds for the oracle itself
    monkeypatch.setattr(tmod, "O", _planted(old, new))
    with pytest.raises(Exception):
        pin_fn()
