"""GPU parity of the expert-parallel layer (the moe_ep_* calls through the C
ABI). W ranks are emulated one after another on one GPU: every rank's
dispatch, then the exchange done by slicing (what an all-to-all delivers:
rows source-major, each source's rows in its send order), every rank's
experts, the exchange back, every rank's combine. No kernel waits on another
rank's work.

Checks, per rank:
  * routing, gates and counts identical to moe_forward's on the same tokens;
  * the send plan (row counts, pair counts, slots: destination-major, tokens
    ascending) and every packed row's local ids and gates, bit-exact against
    their definition; the packed codes and scales bit-exact against the
    oracle's 1x128 quantisation;
  * the output against moe_forward with all experts on one GPU: each expert
    output is the same GEMM result, only the order of the fp32 additions in
    the combine differs, so values agree to one bf16 ulp (plus a 4e-6 RMS
    allowance for cancellation) and almost all are identical;
  * the output against the oracle (small shapes): the one-GPU layer on the
    rank's tokens stage by stage (tests/helpers.py expert_path_parity), and
    the expert-parallel output the rounding of the oracle's combine of those
    expert outputs, up to near ties, within the layer output's tier.
The product's ExpertParallelMoE is also run over a real one-rank NCCL group."""
import dataclasses
import socket

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200 import capi, ep
from mixture_experts_layer_40_b200 import inputs as I
from mixture_experts_layer_40_b200.layer import MoELayer, device_weights
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from __graft_entry__ import build
    build()
    assert torch.cuda.is_available()


def rank_x(w: I.Workload, rank: int, T: int) -> np.ndarray:
    return I.make_x(I.Workload(w.name, T=T, H=w.H, N=w.N, K=w.K, I=w.I, seed=w.seed + 101 * (rank + 1)))


def emulate(w: I.Workload, W: int, xs_bits, dw, bias: np.ndarray, G: int = 0, M: int = 0):
    """One expert-parallel step over W emulated ranks; returns per-rank dicts."""
    N, K, Hd = w.N, w.K, w.H
    el = N // W
    bd = torch.from_numpy(bias).cuda()
    wl_t = [ep.local_weights(dw.w13, dw.s13, dw.w2, dw.s2, N, W, r) for r in range(W)]
    wl = [capi.make_weights(dw.gate_w, *t) for t in wl_t]
    rb = capi.moe_ep_row_bytes(capi.shape_of(1, Hd, N, K, w.I, G, M))
    # odd ranks route with the centroids split once beforehand, even ranks
    # split them in the call: both must route as moe_forward does
    gs = torch.empty((3, N, Hd), dtype=torch.bfloat16, device="cuda")
    capi.moe_split_gate(dw.gate_w, gs)
    ranks = []
    for r, xb in enumerate(xs_bits):
        T = xb.shape[0]
        sh = capi.shape_of(T, Hd, N, K, w.I, G, M)
        st = {"T": T, "sh": sh, "x_bits": xb}
        st["xd"] = H.x_to_device(xb) if T else torch.empty(0, Hd, dtype=torch.bfloat16,
                                                             device="cuda")
        st["send"] = torch.zeros(max(T * min(W, K), 1), rb, dtype=torch.uint8, device="cuda")
        st["sc"] = torch.full((W, 2), -7, dtype=torch.int32, device="cuda")
        st["ws"] = torch.empty(capi.moe_ep_dispatch_workspace_size(sh, W), dtype=torch.uint8,
                               device="cuda")
        st["ids"] = torch.empty(T, K, dtype=torch.int32, device="cuda")
        st["gates"] = torch.empty(T, K, dtype=torch.float32, device="cuda")
        st["counts"] = torch.full((N,), -1, dtype=torch.int32, device="cuda")
        capi.moe_ep_dispatch(sh, W, dw.gate_w, st["xd"], bd, st["send"], st["sc"], st["ws"],
                             topk_ids=st["ids"] if T else None,
                             topk_gates=st["gates"] if T else None, counts=st["counts"],
                             gate_split=gs if r % 2 else None)
        capi.moe_ep_shared(sh, W, wl[r], st["ws"])
        ranks.append(st)
    torch.cuda.synchronize()
    rows = np.stack([st["sc"].cpu().numpy()[:, 0] for st in ranks])   # [src, dst]
    pairs = np.stack([st["sc"].cpu().numpy()[:, 1] for st in ranks])
    off = np.concatenate([np.zeros((W, 1), np.int64), np.cumsum(rows, axis=1)], axis=1)
    outs = []
    for d in range(W):
        recv = torch.cat([ranks[s]["send"][off[s, d]:off[s, d + 1]] for s in range(W)])
        R, P = int(rows[:, d].sum()), int(pairs[:, d].sum())
        sh = ranks[0]["sh"]
        ews = torch.empty(capi.moe_ep_expert_workspace_size(sh, W, R, P), dtype=torch.uint8,
                          device="cuda")
        out = torch.empty(R, Hd, dtype=torch.float32, device="cuda")
        capi.moe_ep_experts(sh, W, wl[d], recv, R, P, out, ews)
        assert capi.moe_get_status(ews) == 0
        outs.append(out)
    for s, st in enumerate(ranks):
        # rank d's output rows from source s sit after those of sources < s
        parts = []
        for d in range(W):
            start = int(rows[:s, d].sum())
            parts.append(outs[d][start:start + rows[s, d]])
        ret = torch.cat(parts)
        y = torch.empty(st["T"], Hd, dtype=torch.bfloat16, device="cuda")
        capi.moe_ep_combine(st["sh"], W, ret, int(rows[s].sum()), st["ws"], y)
        assert capi.moe_get_status(st["ws"]) == 0
        st["y"] = y
        st["rows"], st["pairs"] = rows[s], pairs[s]
    torch.cuda.synchronize()
    return ranks


def check_plan(w: I.Workload, W: int, st):
    T, K, el = st["T"], w.K, w.N // W
    rows, pairs = st["rows"], st["pairs"]
    if T == 0:
        assert not rows.any() and not pairs.any()
        return
    ids = st["ids"].cpu().numpy()
    gates = st["gates"].cpu().numpy()
    dest = ids // el
    expect_rows = [int(np.any(dest == d, axis=1).sum()) for d in range(W)]
    expect_pairs = [int((dest == d).sum()) for d in range(W)]
    assert list(rows) == expect_rows and list(pairs) == expect_pairs
    send = st["send"].cpu().numpy()
    hd = w.H
    q, s = O.quantize_1x128(I.bf16_bits_to_f32(st["x_bits"]))
    slot = 0
    for d in range(W):
        for t in np.nonzero(np.any(dest == d, axis=1))[0]:
            row = send[slot]
            assert np.array_equal(row[:hd], q[t])
            assert np.array_equal(row[hd:hd + 4 * (hd // 128)].view(np.uint32), s[t].view(np.uint32))
            meta = row[hd + 4 * (hd // 128):hd + 4 * (hd // 128) + 8 * K]
            lid = meta[:4 * K].view(np.int32)
            g = meta[4 * K:].view(np.float32)
            here = dest[t] == d
            assert np.array_equal(lid, np.where(here, ids[t] - d * el, -1))
            assert np.array_equal(g.view(np.uint32), np.where(here, gates[t], 0.0).astype(np.float32).view(np.uint32))
            slot += 1
    assert slot == sum(expect_rows)


def check_against_forward(w: I.Workload, st, dw, bias, G=0, M=0):
    T = st["T"]
    if T == 0:
        return None
    layer = MoELayer(T, w.H, w.N, w.K, w.I, dw, groups=G, topk_groups=M)
    y_f = layer.forward(st["xd"], torch.from_numpy(bias).cuda())
    assert layer.status() == 0
    assert torch.equal(layer.ids, st["ids"]) and torch.equal(layer.gates, st["gates"])
    assert torch.equal(layer.counts, st["counts"])
    a = st["y"].float().cpu().numpy()
    b = y_f.float().cpu().numpy()
    rms = float(np.sqrt(np.mean(b.astype(np.float64) ** 2)))
    _, e = np.frexp(np.maximum(np.abs(a), np.abs(b)))
    ulp = np.ldexp(1.0, e - 8)  # bf16: 8 significant bits
    diff = np.abs(a - b)
    assert np.all(diff <= ulp + 4e-6 * rms), float(np.max(diff / (ulp + 4e-6 * rms)))
    assert np.mean(a == b) >= 0.95
    return layer, b


def check_against_oracle(w: I.Workload, st, case, one_gpu):
    if st["T"] == 0:
        return
    layer, y_one = one_gpu
    wr = dataclasses.replace(w, T=st["T"])
    x = I.bf16_bits_to_f32(st["x_bits"])
    rcase = dataclasses.replace(case, w=wr, x_bits=st["x_bits"], x=x)
    r_ids, _, _, score = O.route(x, case.gate_w, case.bias, w.K)
    use, _, _ = H.reconcile_ids(st["ids"].cpu().numpy(), r_ids, score, w.K)
    stats = H.expert_path_parity(wr, rcase, layer, y_one, use, np.arange(st["T"]))
    y_ep = st["y"].float().cpu().numpy().astype(np.float64)
    H.check_bf16(y_ep, stats["y_ref"], "expert-parallel combine")
    H.check_rows(y_ep, stats["y_ref"])


def _setup(w: I.Workload):
    case = H.make_case(w)
    dw = device_weights(w, case.pool, case.gate_w, "cuda")
    return case, dw


@pytest.mark.parametrize("W,Ts", [(2, [300, 171]), (2, [77, 0]), (2, [2500, 1025])])
def test_ep_two_ranks(W, Ts):
    w = I.Workload("ep2", T=max(Ts), H=512, N=32, K=4, I=256, bias_range=0.1, seed=21)
    case, dw = _setup(w)
    xs = [rank_x(w, r, t) for r, t in enumerate(Ts)]
    ranks = emulate(w, W, xs, dw, case.bias)
    for st in ranks:
        check_plan(w, W, st)
        one = check_against_forward(w, st, dw, case.bias)
        check_against_oracle(w, st, case, one)


def test_ep_four_ranks_node_limited():
    # groups = ranks: every token reaches at most 2 of the 4 ranks
    w = I.Workload("ep4", T=200, H=256, N=64, K=4, I=128, bias_range=0.1, seed=22)
    case, dw = _setup(w)
    Ts = [200, 1, 0, 129]
    xs = [rank_x(w, r, t) for r, t in enumerate(Ts)]
    ranks = emulate(w, 4, xs, dw, case.bias, G=4, M=2)
    for st in ranks:
        check_plan(w, 4, st)
        if st["T"]:
            dest = st["ids"].cpu().numpy() // 16
            assert max(len(set(r)) for r in dest) <= 2
        check_against_forward(w, st, dw, case.bias, G=4, M=2)


def test_ep_all_tokens_on_one_rank():
    # the bias sends every token to experts 0..3, all on rank 0: rank 1 gets no rows
    w = I.Workload("ep1", T=150, H=256, N=32, K=4, I=128, bias_range=0.1, seed=23)
    case, dw = _setup(w)
    bias = case.bias.copy()
    bias[:4] = 5.0
    xs = [rank_x(w, r, 150) for r in range(2)]
    ranks = emulate(w, 2, xs, dw, bias)
    for st in ranks:
        assert list(st["rows"]) == [150, 0] and list(st["pairs"]) == [600, 0]
        check_plan(w, 2, st)
        check_against_forward(w, st, dw, bias)


def test_ep_v3_shape_eight_ranks():
    w = I.WORKLOADS["v3_prefill"]
    case, dw = _setup(w)
    Ts = [96, 130, 64, 1, 128, 100, 37, 96]
    xs = [rank_x(w, r, t) for r, t in enumerate(Ts)]
    ranks = emulate(w, 8, xs, dw, case.bias)
    for st in ranks:
        check_plan(w, 8, st)
        check_against_forward(w, st, dw, case.bias)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_expert_parallel_layer_one_rank_nccl():
    import torch.distributed as dist
    w = I.Workload("ep_nccl", T=256, H=512, N=32, K=4, I=256, bias_range=0.1, seed=24)
    case, dw = _setup(w)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        w13, s13, w2, s2 = ep.local_weights(dw.w13, dw.s13, dw.w2, dw.s2, w.N, 1, 0)
        layer = ep.ExpertParallelMoE(w.T, w.H, w.N, w.K, w.I, 1, 0, dw.gate_w, w13, s13, w2, s2)
        xb = rank_x(w, 0, 200)
        xd = H.x_to_device(xb)
        bd = torch.from_numpy(case.bias).cuda()
        y = layer.forward(xd, bd)
        torch.cuda.synchronize()
        assert layer.status() == 0
        assert layer.last["send_rows"] == [200] and layer.last["pairs"] == 800
        st = {"T": 200, "xd": xd, "y": y, "ids": layer.ids[:200], "gates": layer.gates[:200],
              "counts": layer.counts}
        check_against_forward(w, st, dw, case.bias)
        total = layer.batch_counts()
        assert int(total.sum()) == 800
        # new centroids: resplit_gate makes the layer route as one that splits
        # them in every dispatch
        ids0 = layer.ids[:200].clone()
        dw.gate_w.mul_(-1.0)
        layer.resplit_gate()
        fresh = ep.ExpertParallelMoE(w.T, w.H, w.N, w.K, w.I, 1, 0, dw.gate_w, w13, s13, w2, s2,
                                     presplit_gate=False)
        ya, yb = layer.forward(xd, bd), fresh.forward(xd, bd)
        torch.cuda.synchronize()
        assert layer.status() == 0 and fresh.status() == 0
        assert torch.equal(ya, yb) and torch.equal(layer.ids[:200], fresh.ids[:200])
        assert not torch.equal(layer.ids[:200], ids0)   # the routing did change
    finally:
        dist.destroy_process_group()


def _dispatch_one(w, W, xb, dw, bias, send_cap=None, guard=0):
    T = xb.shape[0]
    sh = capi.shape_of(T, w.H, w.N, w.K, w.I)
    rb = capi.moe_ep_row_bytes(sh)
    cap = T * min(W, w.K) if send_cap is None else send_cap
    send = torch.zeros(cap + guard, rb, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(W, 2, dtype=torch.int32, device="cuda")
    ws = torch.empty(capi.moe_ep_dispatch_workspace_size(sh, W), dtype=torch.uint8, device="cuda")
    capi.moe_ep_dispatch(sh, W, dw.gate_w, H.x_to_device(xb), torch.from_numpy(bias).cuda(),
                         send[:cap], sc, ws)
    return sh, send, sc, ws


def test_ep_wrong_pair_count_is_reported():
    # a receiver told the wrong number of (row, slot) pairs reports MOE_ERR_BOUNDS
    # through its status word; every index is checked before use, so no access
    # leaves its buffer, and a call with the right count afterwards is clean
    w = I.Workload("ep_err", T=200, H=256, N=32, K=4, I=128, bias_range=0.1, seed=25)
    case, dw = _setup(w)
    sh, send, sc, ws = _dispatch_one(w, 2, rank_x(w, 0, 200), dw, case.bias)
    torch.cuda.synchronize()
    assert capi.moe_get_status(ws) == 0
    rows, pairs = sc.cpu().numpy()[0]
    wl_t = ep.local_weights(dw.w13, dw.s13, dw.w2, dw.s2, w.N, 2, 0)
    wl = capi.make_weights(dw.gate_w, *wl_t)
    recv = send[:rows]
    out = torch.empty(rows, w.H, dtype=torch.float32, device="cuda")
    for p in (pairs - 1, pairs + 1, pairs):
        ews = torch.empty(capi.moe_ep_expert_workspace_size(sh, 2, int(rows), int(p)),
                          dtype=torch.uint8, device="cuda")
        capi.moe_ep_experts(sh, 2, wl, recv, int(rows), int(p), out, ews)
        assert capi.moe_get_status(ews) == (0 if p == pairs else -5)


def test_ep_send_buffer_too_small_is_reported():
    # rows beyond send_cap are dropped and flagged; the guard rows after the
    # buffer stay untouched
    w = I.Workload("ep_cap", T=200, H=256, N=32, K=4, I=128, bias_range=0.1, seed=26)
    case, dw = _setup(w)
    sh, send, sc, ws = _dispatch_one(w, 2, rank_x(w, 0, 200), dw, case.bias, send_cap=150,
                                     guard=64)
    torch.cuda.synchronize()
    assert capi.moe_get_status(ws) == -5
    assert int(sc.cpu()[:, 0].sum()) > 150     # the plan still counts every row
    assert not send[150:].any().item()


def emulate_peer(w: I.Workload, W: int, T_cap: int, steps, dw, bias: np.ndarray, G=0, M=0):
    """Steps of the peer mode over W emulated ranks on one GPU. Every rank's
    receive, count and return buffers are ordinary allocations here and the
    pointer arrays hold their addresses; the barriers of a real run are the
    order of the calls (all dispatches, then all experts, then all combines).
    Returns, per step, the list of per-rank outputs."""
    N, K, Hd = w.N, w.K, w.H
    bd = torch.from_numpy(bias).cuda()
    wl_t = [ep.local_weights(dw.w13, dw.s13, dw.w2, dw.s2, N, W, r) for r in range(W)]
    wl = [capi.make_weights(dw.gate_w, *t) for t in wl_t]
    sh_cap = capi.shape_of(T_cap, Hd, N, K, w.I, G, M)
    rb = capi.moe_ep_row_bytes(sh_cap)
    recv = [torch.zeros(W * T_cap, rb, dtype=torch.uint8, device="cuda") for _ in range(W)]
    cnt = [torch.full((W,), -3, dtype=torch.int32, device="cuda") for _ in range(W)]
    ret = [torch.zeros(W * T_cap, Hd, dtype=torch.float32, device="cuda") for _ in range(W)]
    ptrs = lambda ts: torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device="cuda")
    p_recv, p_cnt, p_ret = ptrs(recv), ptrs(cnt), ptrs(ret)
    ws = [torch.empty(capi.moe_ep_dispatch_workspace_size(sh_cap, W), dtype=torch.uint8,
                      device="cuda") for _ in range(W)]
    ews = [torch.empty(capi.moe_ep_peer_expert_workspace_size(sh_cap, W, T_cap),
                       dtype=torch.uint8, device="cuda") for _ in range(W)]
    gs = torch.empty((3, N, Hd), dtype=torch.bfloat16, device="cuda")
    capi.moe_split_gate(dw.gate_w, gs)
    outs = []
    for xs_bits in steps:
        shs = [capi.shape_of(xb.shape[0], Hd, N, K, w.I, G, M) for xb in xs_bits]
        for r, xb in enumerate(xs_bits):
            T = xb.shape[0]
            xd = H.x_to_device(xb) if T else torch.empty(0, Hd, dtype=torch.bfloat16, device="cuda")
            capi.moe_ep_dispatch_peer(shs[r], W, r, T_cap, dw.gate_w, xd, bd, p_recv, p_cnt, ws[r],
                                      gate_split=gs if r % 2 == 0 else None)
            capi.moe_ep_shared(shs[r], W, wl[r], ws[r])
        for d in range(W):
            capi.moe_ep_experts_peer(shs[d], W, d, T_cap, wl[d], recv[d], cnt[d], p_ret, ews[d])
        ys = []
        for s in range(W):
            y = torch.empty(xs_bits[s].shape[0], Hd, dtype=torch.bfloat16, device="cuda")
            capi.moe_ep_combine_peer(shs[s], W, T_cap, ret[s], ws[s], y)
            ys.append(y)
        torch.cuda.synchronize()
        for r in range(W):
            assert capi.moe_get_status(ws[r]) == 0 and capi.moe_get_status(ews[r]) == 0
        outs.append(ys)
    return outs


@pytest.mark.parametrize("W,Ts,GM", [(2, [300, 171], (0, 0)), (4, [200, 1, 0, 129], (4, 2))])
def test_ep_peer_mode_equals_all_to_all_mode(W, Ts, GM):
    # the same rows, the same per-row sums and the same combine order: identical bits
    w = I.Workload("ep_peer", T=max(Ts), H=256, N=16 * W, K=4, I=128, bias_range=0.1, seed=27)
    case, dw = _setup(w)
    xs = [rank_x(w, r, t) for r, t in enumerate(Ts)]
    a2a = emulate(w, W, xs, dw, case.bias, G=GM[0], M=GM[1])
    (peer,) = emulate_peer(w, W, max(Ts), [xs], dw, case.bias, G=GM[0], M=GM[1])
    for st, y in zip(a2a, peer):
        assert torch.equal(st["y"], y)


def test_ep_peer_mode_second_step_reuses_the_buffers():
    # step 2 sends different batches through the same buffers, rank 1 sending
    # nothing (its count must read 0 everywhere, not step 1's)
    w = I.Workload("ep_peer2", T=240, H=256, N=32, K=4, I=128, bias_range=0.1, seed=28)
    case, dw = _setup(w)
    step1 = [rank_x(w, 0, 240), rank_x(w, 1, 200)]
    step2 = [rank_x(w, 5, 120), np.zeros((0, w.H), np.uint16)]
    outs = emulate_peer(w, 2, 240, [step1, step2], dw, case.bias)
    for step, ys in zip([step1, step2], outs):
        ref = emulate(w, 2, step, dw, case.bias)
        for st, y in zip(ref, ys):
            assert torch.equal(st["y"], y)


def test_expert_parallel_layer_peer_mode_one_rank_nccl():
    import torch.distributed as dist
    w = I.Workload("ep_nccl_peer", T=256, H=512, N=32, K=4, I=256, bias_range=0.1, seed=29)
    case, dw = _setup(w)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        loc = ep.local_weights(dw.w13, dw.s13, dw.w2, dw.s2, w.N, 1, 0)
        a2a = ep.ExpertParallelMoE(w.T, w.H, w.N, w.K, w.I, 1, 0, dw.gate_w, *loc)
        peer = ep.ExpertParallelMoE(w.T, w.H, w.N, w.K, w.I, 1, 0, dw.gate_w, *loc, peer=True)
        bd = torch.from_numpy(case.bias).cuda()
        for t in (200, 256, 17):
            xd = H.x_to_device(rank_x(w, 0, t))
            y_a = a2a.forward(xd, bd)
            y_p = peer.forward(xd, bd)
            torch.cuda.synchronize()
            assert a2a.status() == 0 and peer.status() == 0
            assert torch.equal(y_a, y_p)
    finally:
        dist.destroy_process_group()
