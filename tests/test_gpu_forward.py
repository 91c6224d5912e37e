"""GPU parity of the whole layer forward (moe_forward through the C ABI)
against the oracle: intermediates that are integer or byte work are compared
bit-exactly (x codes and scales, counts, offsets, the permutation), routing
with the near-tie rule, the expert path stage by stage (h codes, the bf16
expert outputs, the combine; tests/helpers.py expert_path_parity) and the
output rows within 2e-2 of their RMS. Small workloads are checked on every
token; the V3-shape ones on a seeded sample of 512 tokens (routing, counts
and the permutation always on every token)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I
from mixture_experts_layer_40_b200.layer import MoELayer, device_weights
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from __graft_entry__ import build
    build()
    assert torch.cuda.is_available()


def run_forward(w: I.Workload, case: H.Case | None = None, bias_override=None):
    case = case or H.make_case(w)
    bias = case.bias if bias_override is None else bias_override
    layer = MoELayer(w.T, w.H, w.N, w.K, w.I, device_weights(w, case.pool, case.gate_w, "cuda"))
    xd = H.x_to_device(case.x_bits)
    bd = torch.from_numpy(bias).cuda()
    y = layer.forward(xd, bd)
    assert layer.status() == 0
    return case, layer, bias, H.bf16_to_f32(y)


def check_intermediates(w, case, layer, bias, sample_rows=None):
    L = layer.layout
    ids = layer.ids.cpu().numpy()
    r_ids, _, s, score = O.route(case.x, case.gate_w, bias, w.K)
    use_ids, ndiff, nnear = H.reconcile_ids(ids, r_ids, score, w.K)
    counts = layer.counts.cpu().numpy()
    assert np.array_equal(counts, O.expert_counts(use_ids, w.N))
    # x codes and scales sit in the shared-expert GEMM rows
    rows = np.arange(w.T) if sample_rows is None else np.asarray(sample_rows)
    a_q = layer.view("a_q", torch.uint8, (L.rows_total, w.H))
    a_s = layer.view("a_s", torch.float32, (L.rows_total, w.H // 128))
    idx = torch.from_numpy(L.routed_cap + rows).cuda()
    rq, rs = O.quantize_1x128(case.x[rows])
    assert np.array_equal(a_q[idx].cpu().numpy(), rq)
    assert np.array_equal(a_s[idx].cpu().numpy().view(np.uint32), rs.view(np.uint32))
    # offsets, group table, permutation: bit-exact against the oracle's order
    offsets, tokens, rank = O.permutation(use_ids, w.N)
    assert np.array_equal(layer.view("offsets", torch.int32, (w.N + 1,)).cpu().numpy(), offsets)
    gr = layer.view("group_rows", torch.int32, (w.N + 1,)).cpu().numpy()
    st = layer.view("row_start", torch.int32, (w.N + 1,)).cpu().numpy()
    assert np.array_equal(gr[:w.N], counts) and gr[w.N] == w.T
    padded = (counts + 127) // 128 * 128
    assert np.array_equal(st[:w.N], np.concatenate([[0], np.cumsum(padded)[:-1]]))
    assert st[w.N] == L.routed_cap
    row_token = layer.view("row_token", torch.int32, (L.routed_cap,)).cpu().numpy()
    token_row = layer.view("token_row", torch.int32, (w.T, w.K)).cpu().numpy()
    expect_rt = np.full(L.routed_cap, -1, np.int32)
    for e in range(w.N):
        seg = tokens[offsets[e]:offsets[e + 1]]
        expect_rt[st[e]:st[e] + len(seg)] = seg
    assert np.array_equal(row_token, expect_rt)
    expect_tr = st[use_ids] + rank
    assert np.array_equal(token_row, expect_tr)
    # routed GEMM rows hold the token's codes
    some = np.nonzero(row_token >= 0)[0][:: max(1, (row_token >= 0).sum() // 64)]
    got = a_q[torch.from_numpy(some).cuda()].cpu().numpy()
    want = a_q[torch.from_numpy(L.routed_cap + row_token[some]).cuda()].cpu().numpy()
    assert np.array_equal(got, want)
    return use_ids, ndiff


def check_output(w, case, layer, bias, y, use_ids, tokens=None):
    tokens = np.arange(w.T) if tokens is None else np.asarray(tokens)
    stats = H.expert_path_parity(w, case, layer, y[tokens], use_ids, tokens)
    # gates of the GPU's ids from the oracle's unbiased affinities
    s = O.sigmoid(O.gate_logits(case.x, case.gate_w))
    sel = np.take_along_axis(s, use_ids.astype(np.int64), axis=1)
    ref_gates = sel / sel.sum(axis=1, keepdims=True)
    assert np.max(np.abs(layer.gates.cpu().numpy() - ref_gates)) < 1e-5
    return stats


def test_forward_tiny_all_tokens():
    w = I.WORKLOADS["tiny"]
    case, layer, bias, y = run_forward(w)
    use_ids, _ = check_intermediates(w, case, layer, bias)
    check_output(w, case, layer, bias, y, use_ids)


def test_forward_tiny_bias_update_bit_exact():
    w = I.WORKLOADS["tiny"]
    case, layer, bias, y = run_forward(w)
    bd = torch.from_numpy(bias).cuda()
    layer.update_bias(bd, w.gamma)
    nb = O.update_bias(bias, layer.counts.cpu().numpy(), w.T, w.K, w.gamma)
    assert np.array_equal(bd.cpu().numpy(), nb)


@pytest.mark.parametrize("t", [1, 7, 200, 513])
def test_forward_ragged_token_counts(t):
    w = I.Workload(f"ragged{t}", T=t, H=512, N=32, K=4, I=256, bias_range=0.1, seed=t)
    case, layer, bias, y = run_forward(w)
    use_ids, _ = check_intermediates(w, case, layer, bias)
    check_output(w, case, layer, bias, y, use_ids)


def test_forward_all_tokens_to_the_same_experts():
    w = I.Workload("hot", T=300, H=256, N=16, K=4, I=128, bias_range=0.1, seed=5)
    case = H.make_case(w)
    bias = case.bias.copy()
    bias[[0, 5, 6, 15]] = 4.0
    case, layer, bias, y = run_forward(w, case, bias_override=bias)
    counts = layer.counts.cpu().numpy()
    assert counts[0] == w.T and counts[1] == 0
    use_ids, _ = check_intermediates(w, case, layer, bias)
    check_output(w, case, layer, bias, y, use_ids)


def test_forward_run_to_run_identical():
    w = I.Workload("det", T=777, H=512, N=32, K=4, I=256, bias_range=0.1, seed=9)
    case, layer, bias, y1 = run_forward(w)
    xd = H.x_to_device(case.x_bits)
    bd = torch.from_numpy(bias).cuda()
    y2 = H.bf16_to_f32(layer.forward(xd, bd))
    assert np.array_equal(y1, y2)


def test_forward_decode_v3_shape():
    w = I.WORKLOADS["decode"]
    case, layer, bias, y = run_forward(w)
    use_ids, _ = check_intermediates(w, case, layer, bias)
    check_output(w, case, layer, bias, y, use_ids)


def _sampled(w, seed, n=512):
    return np.sort(np.random.default_rng(seed).choice(w.T, min(n, w.T), replace=False))


def test_forward_v3_prefill_sampled():
    w = I.WORKLOADS["v3_prefill"]
    case, layer, bias, y = run_forward(w)
    use_ids, _ = check_intermediates(w, case, layer, bias, sample_rows=_sampled(w, 1))
    check_output(w, case, layer, bias, y, use_ids, tokens=_sampled(w, 2))


def test_forward_large_prefill_outliers_sampled():
    """T = 32768 with 1% of the channels scaled x20 (the outliers that stress
    the 1x128 tiles): routing, counts and the permutation on every token; x
    codes and scales, h codes, expert outputs and y on 512 seeded tokens."""
    w = I.WORKLOADS["large_prefill"]
    case, layer, bias, y = run_forward(w)
    use_ids, _ = check_intermediates(w, case, layer, bias, sample_rows=_sampled(w, 3))
    check_output(w, case, layer, bias, y, use_ids, tokens=_sampled(w, 4))


def test_forward_skewed_sampled():
    """T = 8192 with Zipf-ranked gate logits: a few experts receive most of
    the tokens (the largest groups of the grouped GEMMs)."""
    w = I.WORKLOADS["skewed"]
    case, layer, bias, y = run_forward(w)
    counts = layer.counts.cpu().numpy()
    assert counts.max() > 4 * counts.mean()
    use_ids, _ = check_intermediates(w, case, layer, bias, sample_rows=_sampled(w, 5))
    check_output(w, case, layer, bias, y, use_ids, tokens=_sampled(w, 6))


def test_forward_with_and_without_presplit_gate():
    """The centroids' bf16 terms made once (moe_split_gate, moe_weights.gate_split)
    or on every call give the same routing and output bits; after the
    centroids change, resplit_gate follows them."""
    w = I.Workload("split", T=333, H=512, N=32, K=4, I=256, bias_range=0.1, seed=17)
    case = H.make_case(w)
    dw = device_weights(w, case.pool, case.gate_w, "cuda")
    xd = H.x_to_device(case.x_bits)
    bd = torch.from_numpy(case.bias).cuda()
    a = MoELayer(w.T, w.H, w.N, w.K, w.I, dw, presplit_gate=True)
    b = MoELayer(w.T, w.H, w.N, w.K, w.I, dw, presplit_gate=False)
    ya, yb = a.forward(xd, bd), b.forward(xd, bd)
    assert a.status() == 0 and b.status() == 0
    assert torch.equal(ya, yb) and torch.equal(a.ids, b.ids) and torch.equal(a.gates, b.gates)
    # the split terms sum back to the centroids exactly
    t = a.gate_split.double()
    assert torch.equal(t[0] + t[1] + t[2], dw.gate_w.double())
    dw.gate_w.mul_(-1.0)
    a.resplit_gate()
    ya, yb = a.forward(xd, bd), b.forward(xd, bd)
    assert torch.equal(ya, yb) and torch.equal(a.ids, b.ids)
