"""GPU parity of the single kernels through the C ABI: quantisers (bit-exact),
bias update (bit-exact), routing (ids with the near-tie rule, counts exact,
gates to fp32 accuracy) and the grouped FP8 expert GEMMs (against float64
sums of the same dequantised operands)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import inputs as I
from tests import helpers as H

pytestmark = pytest.mark.gpu
GATE_TOL = 1e-5


@pytest.fixture(scope="module")
def capi():
    from __graft_entry__ import build
    build()
    from mixture_experts_layer_40_b200 import capi as c
    assert torch.cuda.is_available()
    return c


def _bf16_rows(rng, rows, cols, outliers=False):
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x *= rng.uniform(1e-3, 1e2, (rows, 1)).astype(np.float32)
    if outliers:
        ch = rng.choice(cols, size=max(1, cols // 100), replace=False)
        x[:, ch] *= 20
    if rows > 2:
        x[1, :128] = 0.0          # an all-zero tile
        x[2, 128:256] = 1e-30     # tiny values (bf16 keeps them normal)
    return I.f32_to_bf16_bits(x)


@pytest.mark.parametrize("rows,cols", [(1, 128), (3, 256), (130, 7168), (1000, 384)])
def test_quantize_1x128_bit_exact(capi, rows, cols):
    rng = np.random.default_rng(rows * 7 + cols)
    xb = _bf16_rows(rng, rows, cols, outliers=True)
    xd = H.x_to_device(xb)
    q = torch.full((rows, cols), 0xAB, dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, cols // 128), dtype=torch.float32, device="cuda")
    capi.moe_quantize_1x128(xd, q, s)
    rq, rs = O.quantize_1x128(I.bf16_bits_to_f32(xb))
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_quantize_1x128_empty(capi):
    xd = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((0, 256), dtype=torch.uint8, device="cuda")
    s = torch.empty((0, 2), dtype=torch.float32, device="cuda")
    capi.moe_quantize_1x128(xd, q, s)
    torch.cuda.synchronize()


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (512, 1024)])
def test_quantize_128x128_bit_exact(capi, rows, cols):
    rng = np.random.default_rng(rows + cols)
    w = (rng.standard_normal((rows, cols)) * rng.uniform(1e-3, 10, (rows, 1))).astype(np.float32)
    w[:128, :128] = 0.0
    wd = torch.from_numpy(w).cuda()
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows // 128, cols // 128), dtype=torch.float32, device="cuda")
    capi.moe_quantize_128x128(wd, q, s)
    rq, rs = O.quantize_128x128(w)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_update_bias_bit_exact(capi):
    rng = np.random.default_rng(3)
    n, t, k = 256, 4096, 8
    b = rng.uniform(-0.1, 0.1, n).astype(np.float32)
    c = rng.integers(100, 160, n).astype(np.int32)
    c[:5] = 128  # exactly at the mean load T*K/N
    bd = torch.from_numpy(b).cuda()
    cd = torch.from_numpy(c).cuda()
    capi.moe_update_bias(bd, cd, n, t, k, 1e-3)
    assert np.array_equal(bd.cpu().numpy(), O.update_bias(b, c, t, k, 1e-3))
    capi.moe_update_bias(bd, cd, n, t, k, 0.0)
    assert np.array_equal(bd.cpu().numpy(), O.update_bias(b, c, t, k, 1e-3))


def _route(capi, w, x_bits, gate_w, bias):
    sh = capi.shape_of(w.T, w.H, w.N, w.K, w.I)
    ws = torch.empty(capi.moe_workspace_size(sh), dtype=torch.uint8, device="cuda")
    ids = torch.empty((w.T, w.K), dtype=torch.int32, device="cuda")
    gates = torch.empty((w.T, w.K), dtype=torch.float32, device="cuda")
    counts = torch.empty((w.N,), dtype=torch.int32, device="cuda")
    capi.moe_route(sh, torch.from_numpy(gate_w).cuda(), H.x_to_device(x_bits),
                   torch.from_numpy(bias).cuda(), ids, gates, counts, ws)
    assert capi.moe_get_status(ws) == 0
    return ids.cpu().numpy(), gates.cpu().numpy(), counts.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "decode", "v3_prefill", "skewed", "large_prefill"])
def test_route_parity(capi, name):
    """large_prefill (T = 32768) takes the wide-tile logits kernel (256 tokens x
    256 experts per CTA), the others the 128 x 64 tiles."""
    w = I.WORKLOADS[name]
    xb = I.make_x(w)
    gate_w, bias = I.make_gate_w(w), I.make_bias(w)
    ids, gates, counts = _route(capi, w, xb, gate_w, bias)
    r_ids, r_gates, s, score = O.route(I.bf16_bits_to_f32(xb), gate_w, bias, w.K)
    use_ids, ndiff, nnear = H.reconcile_ids(ids, r_ids, score, w.K)
    assert np.array_equal(counts, O.expert_counts(use_ids, w.N))
    assert counts.sum() == w.T * w.K
    # gates of the GPU's ids from the oracle's unbiased affinities; the fp32
    # logits are within ~1e-6 of the float64 ones (|z| up to ~10 in the skewed
    # workload), which moves a gate by at most a few 1e-6
    sel = np.take_along_axis(s, ids.astype(np.int64), axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    assert np.max(np.abs(gates - ref)) < GATE_TOL
    assert np.allclose(gates.sum(axis=1), 1.0, atol=GATE_TOL)


@pytest.mark.parametrize("t,n,h", [(333, 512, 2048), (1, 256, 7168), (700, 256, 1024)])
def test_route_parity_split_reduction(capi, t, n, h):
    """Batches too small for whole-depth tiles to fill the GPU split the gate
    GEMM's reduction into slices (8 for T=333 at N=512 over two 256-expert
    column tiles, 28 for one token, 4 for T=700 at H=1024) and sum the
    slices in order before the top-K."""
    w = I.Workload("split", T=t, H=h, N=n, K=8, I=256, bias_range=0.05, seed=22)
    xb = I.make_x(w)
    gate_w, bias = I.make_gate_w(w), I.make_bias(w)
    ids, gates, counts = _route(capi, w, xb, gate_w, bias)
    r_ids, _, s, score = O.route(I.bf16_bits_to_f32(xb), gate_w, bias, w.K)
    use_ids, _, _ = H.reconcile_ids(ids, r_ids, score, w.K)
    assert np.array_equal(counts, O.expert_counts(use_ids, w.N))
    sel = np.take_along_axis(s, ids.astype(np.int64), axis=1)
    assert np.max(np.abs(gates - sel / sel.sum(axis=1, keepdims=True))) < GATE_TOL


@pytest.mark.parametrize("k", [1, 4])
def test_route_parity_wide_tiles_fewer_slots(capi, k):
    """The selection fused into the wide logits tiles keeps a sorted list of
    eight; with K < 8 its first K entries are the choices. T = 16384 with a
    ragged last tile (T - 100)."""
    w = I.Workload("wide", T=16384 - 100, H=7168, N=256, K=k, I=2048, bias_range=0.05,
                   seed=21)
    xb = I.make_x(w)
    gate_w, bias = I.make_gate_w(w), I.make_bias(w)
    ids, gates, counts = _route(capi, w, xb, gate_w, bias)
    r_ids, _, s, score = O.route(I.bf16_bits_to_f32(xb), gate_w, bias, w.K)
    use_ids, _, _ = H.reconcile_ids(ids, r_ids, score, w.K)
    assert np.array_equal(counts, O.expert_counts(use_ids, w.N))
    sel = np.take_along_axis(s, ids.astype(np.int64), axis=1)
    assert np.max(np.abs(gates - sel / sel.sum(axis=1, keepdims=True))) < GATE_TOL


def test_route_ragged_tokens_and_hot_expert(capi):
    w = I.Workload("hot", T=333, H=512, N=32, K=4, I=128, bias_range=0.1)
    xb = I.make_x(w)
    gate_w = I.make_gate_w(w)
    bias = I.make_bias(w)
    bias[[3, 7, 11, 30]] = 5.0  # every token picks these four
    ids, gates, counts = _route(capi, w, xb, gate_w, bias)
    assert np.array_equal(np.sort(ids, 1), np.tile([3, 7, 11, 30], (w.T, 1)))
    assert counts[3] == w.T and counts.sum() == w.T * w.K
    r_ids, _, s, score = O.route(I.bf16_bits_to_f32(xb), gate_w, bias, w.K)
    H.reconcile_ids(ids, r_ids, score, w.K)


# ----------------------------------------------------------- grouped GEMMs

def _gemm_case(h_dim, i_dim, group_rows, seed=0):
    """Seeded rows + per-group weights for the stage entry points."""
    rng = np.random.default_rng(seed)
    starts, r = [], 0
    for c in group_rows:
        starts.append(r)
        r += (c + 127) // 128 * 128 + 128  # a padding tile between groups
    rows = r
    n_groups = len(group_rows)
    a = rng.standard_normal((rows, h_dim)).astype(np.float32)
    a *= rng.uniform(0.1, 10, (rows, 1)).astype(np.float32)
    a_q, a_s = O.quantize_1x128(a)
    w13 = (rng.standard_normal((n_groups, 2 * i_dim, h_dim)) / np.sqrt(h_dim)).astype(np.float32)
    w2 = (rng.standard_normal((n_groups, h_dim, i_dim)) / np.sqrt(i_dim)).astype(np.float32)
    q13 = np.empty(w13.shape, np.uint8)
    s13 = np.empty((n_groups, 2 * i_dim // 128, h_dim // 128), np.float32)
    q2 = np.empty(w2.shape, np.uint8)
    s2 = np.empty((n_groups, h_dim // 128, i_dim // 128), np.float32)
    for g in range(n_groups):
        q13[g], s13[g] = O.quantize_128x128(w13[g])
        q2[g], s2[g] = O.quantize_128x128(w2[g])
    return dict(rows=rows, starts=np.array(starts, np.int32), counts=np.array(group_rows, np.int32),
                a_q=a_q, a_s=a_s, q13=q13, s13=s13, q2=q2, s2=s2)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


# Group sizes: empty groups, whole 128-row tiles, last row tiles of 1, 3, 5,
# 44, 64 and 65 rows.
TAIL_CASES = [
    (256, 128, [5, 0, 128, 129, 300, 1]),
    (256, 128, [64, 65, 192, 3, 0, 0, 64]),
    (7168, 2048, [130, 0, 7, 256]),
]


@pytest.mark.parametrize("h_dim,i_dim,group_rows", TAIL_CASES)
def test_expert_up_parity(capi, h_dim, i_dim, group_rows):
    c = _gemm_case(h_dim, i_dim, group_rows, seed=h_dim)
    n_groups, rows = len(group_rows), c["rows"]
    h_q = torch.full((rows, i_dim), 0x5A, dtype=torch.uint8, device="cuda")
    h_s = torch.full((rows, i_dim // 128), -7.0, dtype=torch.float32, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    capi.moe_expert_up(h_dim, i_dim, n_groups, _dev(c["counts"]), _dev(c["starts"]), rows,
                       _dev(c["a_q"]), _dev(c["a_s"]), _dev(c["q13"]), _dev(c["s13"]), h_q, h_s,
                       status)
    assert capi.moe_get_status(status) == 0
    hq, hs = h_q.cpu().numpy(), h_s.cpu().numpy()
    x_hat = O.dequantize_1x128(c["a_q"], c["a_s"])
    written = np.zeros(rows, bool)
    match = total = 0
    for g in range(n_groups):
        st, n = c["starts"][g], c["counts"][g]
        written[st:st + n] = True
        if n == 0:
            continue
        w13 = O.dequantize_128x128(c["q13"][g], c["s13"][g])
        gate = np.concatenate([w13[256 * j:256 * j + 128] for j in range(i_dim // 128)])
        up = np.concatenate([w13[256 * j + 128:256 * j + 256] for j in range(i_dim // 128)])
        xr = x_hat[st:st + n]
        h = O.silu(xr @ gate.T) * (xr @ up.T)
        # the GPU code of every element is the E4M3 rounding of h * scale up to
        # the fp32 accumulation error: within one code step of the oracle's
        rq, rs = O.quantize_1x128(h.astype(np.float32))
        assert np.allclose(hs[st:st + n], rs, rtol=2e-5, atol=0)
        deq = O.dequantize_1x128(hq[st:st + n], hs[st:st + n])
        step = np.abs(O.dequantize_1x128(rq, rs)) * 2.0 ** -3 + 2.0 ** -9 / np.repeat(rs, 128, 1)
        assert np.all(np.abs(deq - h) <= step + 1e-6 * np.abs(h).max())
        match += np.sum(hq[st:st + n] == rq)
        total += rq.size
    assert match / total > 0.995, match / total
    # rows outside every segment are untouched
    assert np.all(hq[~written] == 0x5A) and np.all(hs[~written] == -7.0)


@pytest.mark.parametrize("h_dim,i_dim,group_rows", TAIL_CASES)
def test_expert_down_parity(capi, h_dim, i_dim, group_rows):
    rng = np.random.default_rng(h_dim + 1)
    starts, r = [], 0
    for n in group_rows:
        starts.append(r)
        r += (n + 127) // 128 * 128 + 128
    rows, n_groups = r, len(group_rows)
    h = (rng.standard_normal((rows, i_dim)) * rng.uniform(0.1, 10, (rows, 1))).astype(np.float32)
    h_q, h_s = O.quantize_1x128(h)
    w2 = (rng.standard_normal((n_groups, h_dim, i_dim)) / np.sqrt(i_dim)).astype(np.float32)
    q2 = np.empty(w2.shape, np.uint8)
    s2 = np.empty((n_groups, h_dim // 128, i_dim // 128), np.float32)
    for g in range(n_groups):
        q2[g], s2[g] = O.quantize_128x128(w2[g])
    y = torch.full((rows, h_dim), 3.0, dtype=torch.float32, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    capi.moe_expert_down(h_dim, i_dim, n_groups, _dev(np.array(group_rows, np.int32)),
                         _dev(np.array(starts, np.int32)), rows, _dev(h_q), _dev(h_s), _dev(q2),
                         _dev(s2), y, status)
    assert capi.moe_get_status(status) == 0
    yg = y.cpu().numpy().astype(np.float64)
    h_hat = O.dequantize_1x128(h_q, h_s)
    written = np.zeros(rows, bool)
    for g in range(n_groups):
        st, n = starts[g], group_rows[g]
        written[st:st + n] = True
        if n == 0:
            continue
        ref = h_hat[st:st + n] @ O.dequantize_128x128(q2[g], s2[g]).T
        got = yg[st:st + n]
        # fp32 outputs of exact E4M3 products: only the fp32 accumulation
        # error remains, which the per-128 promotion keeps below 1e-5 of the
        # row's scale (a 14-bit accumulator at this depth would be ~1e-2 off)
        scale = np.sqrt(np.mean(ref ** 2, axis=1, keepdims=True))
        assert np.all(np.abs(got - ref) <= 1e-5 * scale)
        rel = np.sqrt(np.mean((got - ref) ** 2) / np.mean(ref ** 2))
        assert rel < 1e-6, rel
    assert np.all(yg[~written] == 3.0)


@pytest.mark.parametrize("h_dim,i_dim,group_rows", [
    (256, 128, [5, 0, 128, 129, 300, 1, 31, 32, 33]),
    (256, 128, [64, 65, 192, 3, 0, 0, 64]),
    (7168, 2048, [130, 0, 7, 256]),
])
def test_expert_down_bf16_is_the_rounded_fp32_gemm(capi, h_dim, i_dim, group_rows):
    """The layer's down GEMM writes bf16 expert outputs ("DeepSeek-V3:
    Auxiliary-Loss-Free MoE Load Balancing...", section V, Figure 6): bit for
    bit the round-to-nearest-even of the fp32 GEMM's totals (same kernel,
    other epilogue), and the bf16 rounding of the float64 sums of the same
    operands up to the near-midpoint rule. Groups of 31, 32 and 33 rows cover
    the direct stores of a partial 32-row quarter and the staged TMA stores."""
    rng = np.random.default_rng(h_dim + 2)
    starts, r = [], 0
    for n in group_rows:
        starts.append(r)
        r += (n + 127) // 128 * 128 + 128
    rows, n_groups = r, len(group_rows)
    h = (rng.standard_normal((rows, i_dim)) * rng.uniform(0.1, 10, (rows, 1))).astype(np.float32)
    h_q, h_s = O.quantize_1x128(h)
    w2 = (rng.standard_normal((n_groups, h_dim, i_dim)) / np.sqrt(i_dim)).astype(np.float32)
    q2 = np.empty(w2.shape, np.uint8)
    s2 = np.empty((n_groups, h_dim // 128, i_dim // 128), np.float32)
    for g in range(n_groups):
        q2[g], s2[g] = O.quantize_128x128(w2[g])
    args = (h_dim, i_dim, n_groups, _dev(np.array(group_rows, np.int32)),
            _dev(np.array(starts, np.int32)), rows, _dev(h_q), _dev(h_s), _dev(q2), _dev(s2))
    y32 = torch.full((rows, h_dim), 3.0, dtype=torch.float32, device="cuda")
    y16 = torch.full((rows, h_dim), 3.0, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    capi.moe_expert_down(*args, y32, status)
    capi.moe_expert_down_bf16(*args, y16, status)
    assert capi.moe_get_status(status) == 0
    assert torch.equal(y16, y32.to(torch.bfloat16))
    got = y16.float().cpu().numpy().astype(np.float64)
    h_hat = O.dequantize_1x128(h_q, h_s)
    written = np.zeros(rows, bool)
    flips = 0
    for g in range(n_groups):
        st, n = starts[g], group_rows[g]
        written[st:st + n] = True
        if n == 0:
            continue
        ref = h_hat[st:st + n] @ O.dequantize_128x128(q2[g], s2[g]).T
        flips += H.check_bf16(got[st:st + n], ref, f"group {g}")
    assert np.all(got[~written] == 3.0)
