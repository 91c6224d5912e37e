"""Expert parallelism on the CPU: the exchanges of mixture_experts_layer_40_b200.ep
over gloo (world sizes 2 and 3), and the whole expert-parallel decomposition
of the layer ("DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ...",
section V, "Custom all-to-all kernels": a token goes once to each rank that
holds one of its experts) composed from those exchanges with the oracle as
the per-rank compute: every rank's output must equal the oracle's
single-process layer on its tokens. The GPU kernels of the same steps are
checked in test_gpu_ep.py."""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)


def _exchange_main(rank, world, port, out_dir):
    _init(rank, world, port)
    try:
        from mixture_experts_layer_40_b200 import ep
        # rank s sends (s + d) % 3 + d rows to rank d, each row tagged (s, d, i)
        rows = [(rank + d) % 3 + d for d in range(world)]
        send = torch.tensor([[rank, d, i] for d in range(world) for i in range(rows[d])],
                            dtype=torch.int32).reshape(-1, 3)
        counts = torch.tensor([[r, 10 * r] for r in rows], dtype=torch.int32)
        recv_counts = ep.exchange_counts(counts)
        recv_rows = recv_counts[:, 0].tolist()
        recv, _ = ep.exchange_rows(send, rows, recv_rows)
        # the way back: every row returns to its source in the source's order
        back, _ = ep.exchange_rows(recv * 2, recv_rows, rows)
        with open(os.path.join(out_dir, f"x{rank}.json"), "w") as fh:
            json.dump({"recv_counts": recv_counts.tolist(), "recv": recv.tolist(),
                       "back": back.tolist(), "send": send.tolist()}, fh)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchanges_are_source_major_and_return_in_send_order(tmp_path, world):
    mp.start_processes(_exchange_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"x{r}.json")) for r in range(world)]
    for d in range(world):
        rows_from = [(s + d) % 3 + d for s in range(world)]
        assert res[d]["recv_counts"] == [[r, 10 * r] for r in rows_from]
        expect = [[s, d, i] for s in range(world) for i in range(rows_from[s])]
        assert res[d]["recv"] == expect
    for s in range(world):
        assert res[s]["back"] == [[2 * v for v in row] for row in res[s]["send"]]


def _plan(ids, gates, n, w):
    """Send rows of one source: destination-major, tokens ascending; each row
    (token, local ids, gates) with -1 / 0 for slots whose expert is elsewhere."""
    el = n // w
    rows, slot = [], np.full((ids.shape[0], w), -1, np.int64)
    for d in range(w):
        for t in range(ids.shape[0]):
            here = ids[t] // el == d
            if here.any():
                slot[t, d] = len(rows)
                rows.append((d, t, np.where(here, ids[t] - d * el, -1),
                             np.where(here, gates[t], 0.0)))
    return rows, slot


def _ep_main(rank, world, port, out_dir, node_limited):
    _init(rank, world, port)
    try:
        from oracle import moe_oracle as O
        from mixture_experts_layer_40_b200 import ep
        from mixture_experts_layer_40_b200 import inputs as I
        w = I.Workload("ep", T=24, H=256, N=16 * world, K=4, I=128, bias_range=0.1, seed=3)
        wr = I.Workload("ep", T=24 - 7 * rank, H=256, N=16 * world, K=4, I=128, bias_range=0.1,
                        seed=40 + rank)
        pool = I.make_weight_pool(w)
        ew = O.ExpertWeights(pool.pool13, pool.pool2, pool.slot_gate, pool.slot_up,
                             pool.slot_down)
        x = I.bf16_bits_to_f32(I.make_x(wr))
        gate_w, bias = I.make_gate_w(w), I.make_bias(w)
        if node_limited:  # groups = ranks, one of them per token
            ids, gates, _, _, _ = O.route_grouped(x, gate_w, bias, w.K, world, 1)
        else:
            ids, gates, _, _ = O.route(x, gate_w, bias, w.K)
        rows, slot = _plan(ids, gates, w.N, world)
        send_rows = [sum(1 for r in rows if r[0] == d) for d in range(world)]
        pairs = [int(sum((r[2] >= 0).sum() for r in rows if r[0] == d)) for d in range(world)]
        xq, xs = O.quantize_1x128(x)
        codes = torch.from_numpy(np.stack([xq[r[1]] for r in rows]).reshape(-1, w.H)
                                 if rows else np.zeros((0, w.H), np.uint8))
        scales = torch.from_numpy(np.stack([xs[r[1]] for r in rows]).reshape(-1, w.H // 128)
                                  if rows else np.zeros((0, w.H // 128), np.float32))
        lids = torch.tensor(np.array([r[2] for r in rows], np.int32).reshape(-1, w.K))
        gts = torch.tensor(np.array([r[3] for r in rows], np.float64).reshape(-1, w.K))
        recv_counts = ep.exchange_counts(torch.tensor([[a, b] for a, b in zip(send_rows, pairs)],
                                                      dtype=torch.int32))
        recv_rows = recv_counts[:, 0].tolist()
        r_codes, _ = ep.exchange_rows(codes, send_rows, recv_rows)
        r_scales, _ = ep.exchange_rows(scales, send_rows, recv_rows)
        r_lids, _ = ep.exchange_rows(lids, send_rows, recv_rows)
        r_gates, _ = ep.exchange_rows(gts, send_rows, recv_rows)
        assert int((r_lids >= 0).sum()) == int(recv_counts[:, 1].sum())
        # this rank's experts on the received rows: fp64 partial sums, ascending id
        el = w.N // world
        part = np.zeros((r_codes.shape[0], w.H))
        rl, rg = r_lids.numpy(), r_gates.numpy()
        for e in range(el):
            rr, kk = np.nonzero(rl == e)
            if len(rr) == 0:
                continue
            wg, wu, wd = ew.dequantised(rank * el + e)
            y_e, _, _ = O.expert_ffn_q(r_codes.numpy()[rr], r_scales.numpy()[rr], wg, wu, wd)
            part[rr] += rg[rr, kk][:, None] * y_e
        ret, _ = ep.exchange_rows(torch.from_numpy(part), recv_rows, send_rows)
        wg, wu, wd = ew.dequantised(w.N)
        y, _, _ = O.expert_ffn_q(xq, xs, wg, wu, wd)
        for d in range(world):
            on = slot[:, d] >= 0
            y[on] += ret.numpy()[slot[on, d]]
        ref = O.moe_forward(x, gate_w, bias, w.K, ew, mode="Q", ids=ids)["y"]
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
        np.save(os.path.join(out_dir, f"ref{rank}.npy"), ref)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,node_limited", [(2, False), (3, False), (2, True)])
def test_expert_parallel_layer_equals_the_oracle_layer(tmp_path, world, node_limited):
    mp.start_processes(_ep_main, args=(world, _free_port(), str(tmp_path), node_limited),
                       nprocs=world, start_method="spawn")
    for r in range(world):
        y, ref = np.load(tmp_path / f"y{r}.npy"), np.load(tmp_path / f"ref{r}.npy")
        assert y.shape == ref.shape == (24 - 7 * r, 256)
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


@pytest.fixture(scope="module")
def capi():
    from __graft_entry__ import build
    build()
    from mixture_experts_layer_40_b200 import capi as c
    return c


def test_row_bytes_and_workspace_sizes(capi):
    sh = capi.shape_of(4096, 7168, 256, 8, 2048)
    # codes + 56 scales + 8 ids + 8 gates = 7456 bytes, a multiple of 16
    assert capi.moe_ep_row_bytes(sh) == 7168 + 56 * 4 + 8 * 8
    # 256 codes + 2 scales + 3 ids + 3 gates = 288, already a multiple of 16
    assert capi.moe_ep_row_bytes(capi.shape_of(10, 256, 16, 3, 128)) == 288
    # 256 + 8 + 5 * 8 = 304
    assert capi.moe_ep_row_bytes(capi.shape_of(10, 256, 16, 5, 128)) == 304
    # at least the shared expert's bf16 output rows
    assert capi.moe_ep_dispatch_workspace_size(sh, 8) > 4096 * 7168 * 2
    for bad_w in [0, 3, 17, 32]:  # 256/3 not whole; more than 16 ranks; 256/32 < 16
        assert capi.moe_ep_dispatch_workspace_size(sh, bad_w) == 0
    assert capi.moe_ep_expert_workspace_size(sh, 8, 100, 801) == 0  # pairs > R K
    small = capi.moe_ep_expert_workspace_size(sh, 8, 100, 100)
    big = capi.moe_ep_expert_workspace_size(sh, 8, 100, 800)
    assert 0 < small < big
    assert capi.moe_ep_expert_workspace_size(sh, 8, 0, 0) > 0


def test_ep_calls_reject_bad_arguments_on_the_host(capi):
    import ctypes
    lib = capi.LIB
    sh = capi.shape_of(64, 256, 32, 4, 128)
    null = ctypes.c_void_p(0)
    # W = 3 does not divide N; W = 4 leaves 8 experts per rank (< 16)
    for w_bad in (3, 4):
        assert lib.moe_ep_dispatch(sh, w_bad, null, null, null, null, null, null, null, null, 0,
                                   null, null, 0, null) == -1
        assert lib.moe_ep_experts(sh, w_bad, None, null, 0, 0, null, null, 0, null) == -1
        assert lib.moe_ep_combine(sh, w_bad, null, 0, null, 0, null, null) == -1
    assert lib.moe_ep_dispatch(sh, 2, null, null, null, null, null, null, null, null, 0, null,
                               null, 0, null) == -2
    assert lib.moe_ep_experts(sh, 2, None, null, 10, 41, null, null, 0, null) == -1
    assert lib.moe_ep_experts(sh, 2, None, null, -1, 0, null, null, 0, null) == -1
    assert lib.moe_ep_combine(sh, 2, null, -1, null, 0, null, null) == -1
    buf = ctypes.create_string_buffer(4096 + 256)
    addr = (ctypes.addressof(buf) + 255) // 256 * 256
    assert lib.moe_ep_shared(sh, 2, None, ctypes.c_void_p(addr), 256, null) == -6
    assert lib.moe_ep_combine(sh, 2, null, 0, ctypes.c_void_p(addr + 8), 1 << 40, null,
                              null) == -7
    # a pre-split gate off its 16-byte alignment (checked before any CUDA call);
    # the buffers are never dereferenced
    ws_ok, split_bad = ctypes.c_void_p(addr), ctypes.c_void_p(addr + 8)
    big = capi.moe_ep_dispatch_workspace_size(sh, 2)
    assert lib.moe_ep_dispatch(sh, 2, null, split_bad, null, null, null, null, null, ws_ok, 1,
                               ws_ok, ws_ok, big, null) == -7
    assert lib.moe_ep_dispatch_peer(sh, 2, 0, 64, null, split_bad, null, null, null, null, null,
                                    ws_ok, ws_ok, null, ws_ok, big, null) == -7


def test_peer_mode_calls_reject_bad_arguments_on_the_host(capi):
    import ctypes
    lib = capi.LIB
    sh = capi.shape_of(64, 256, 32, 4, 128)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(256)  # never dereferenced: every call below fails its checks first
    # rank outside [0, W), T above T_cap, T_cap < 1, W not dividing N into >= 16 experts
    for W, rank, T_cap in [(2, 2, 64), (2, -1, 64), (2, 0, 63), (2, 0, 0), (4, 0, 64)]:
        assert lib.moe_ep_dispatch_peer(sh, W, rank, T_cap, null, null, null, null, null, null,
                                        null, fake, fake, null, null, 0, null) == -1
        assert lib.moe_ep_experts_peer(sh, W, rank, T_cap, None, null, fake, fake, null, 0,
                                       null) == -1
    assert lib.moe_ep_combine_peer(sh, 2, 63, null, null, 0, null, null) == -1
    # missing pointer arrays
    assert lib.moe_ep_dispatch_peer(sh, 2, 0, 64, null, null, null, null, null, null, null, null,
                                    fake, null, null, 0, null) == -2
    assert lib.moe_ep_experts_peer(sh, 2, 1, 64, None, null, null, fake, null, 0, null) == -2
    assert lib.moe_ep_experts_peer(sh, 2, 1, 64, None, null, fake, null, null, 0, null) == -2
    # workspace sizes: W T_cap rows of min(K, N/W) slots each, growing with T_cap
    a = capi.moe_ep_peer_expert_workspace_size(sh, 2, 64)
    b = capi.moe_ep_peer_expert_workspace_size(sh, 2, 128)
    assert 0 < a < b
    assert capi.moe_ep_peer_expert_workspace_size(sh, 2, 0) == 0
    assert capi.moe_ep_peer_expert_workspace_size(sh, 3, 64) == 0
    # the receiver's buffer for W T_cap rows holds at least its codes and the fp32 rows
    assert a > 2 * 64 * 4 * (256 + 256 * 4)


def _layout_main(rank, world, port, out_dir):
    _init(rank, world, port)
    try:
        from mixture_experts_layer_40_b200 import ep
        res = {}
        T = 100 + rank  # different batch sizes: fine for all-to-all, not for peer mode
        for name, sizes, peer in [("a2a_T", (T, 256, 32, 4, 128, 0, 0), False),
                                  ("peer_T", (T, 256, 32, 4, 128, 0, 0), True),
                                  ("a2a_K", (100, 256, 32, 4 + rank, 128, 0, 0), False),
                                  ("peer_same", (100, 256, 32, 4, 128, 0, 0), True)]:
            try:
                ep.check_same_layout(sizes, world, peer)
                res[name] = "ok"
            except ValueError:
                res[name] = "refused"
        with open(os.path.join(out_dir, f"l{rank}.json"), "w") as fh:
            json.dump(res, fh)
    finally:
        dist.destroy_process_group()


def test_ranks_with_different_layouts_are_refused(tmp_path):
    world = 2
    mp.start_processes(_layout_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    for r in range(world):
        res = json.load(open(tmp_path / f"l{r}.json"))
        assert res == {"a2a_T": "ok", "peer_T": "refused", "a2a_K": "refused", "peer_same": "ok"}
