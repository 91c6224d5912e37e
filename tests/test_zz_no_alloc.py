"""moe_route_noalloc: routing for callers that cannot give the library any
device memory (for example a host that owns every allocation through its own
pool, or a loop where cudaMalloc's device synchronisation is not allowed).

It keeps its logits scratch in a fixed 4 MiB array inside the library and
computes the logits with the fp32 SIMT kernel, not moe_route's tensor-core
kernel. This file checks, through the C ABI, that two calls in a row route
as the oracle does (ids up to near ties, counts exact for the ids chosen,
gates within 1e-5) and agree with moe_route (which uses a caller workspace)
on the same inputs, that the second call is not disturbed by what the first
left in the shared array, that node-limited routing runs through it too, and
that sizes beyond the array are refused before any work is queued. The file
is named to run last, so a run that stops at its first failure has already
run every other test."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_40_b200 import inputs as I
from oracle import moe_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def capi():
    from __graft_entry__ import build
    build()
    from mixture_experts_layer_40_b200 import capi as c
    assert torch.cuda.is_available()
    return c


def _inputs(w):
    xb = I.make_x(w)
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    return x, torch.from_numpy(I.make_gate_w(w)).cuda(), torch.from_numpy(I.make_bias(w)).cuda()


def _outputs(w):
    return (torch.empty((w.T, w.K), dtype=torch.int32, device="cuda"),
            torch.empty((w.T, w.K), dtype=torch.float32, device="cuda"),
            torch.full((w.N,), 12345, dtype=torch.int32, device="cuda"))


def _reference(capi, w, x, gw, b):
    sh = capi.shape_of(w.T, w.H, w.N, w.K, w.I)
    ws = torch.empty(capi.moe_workspace_size(sh), dtype=torch.uint8, device="cuda")
    ids, gates, counts = _outputs(w)
    capi.moe_route(sh, gw, x, b, ids, gates, counts, ws)
    return ids, gates, counts


def _noalloc(capi, w, x, gw, b, groups=0, top=0):
    sh = capi.shape_of(w.T, w.H, w.N, w.K, w.I, groups, top)
    ids, gates, counts = _outputs(w)
    rc = capi.LIB.moe_route_noalloc(sh, gw.data_ptr(), x.data_ptr(), b.data_ptr(), ids.data_ptr(),
                                    gates.data_ptr(), counts.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    return ids, gates, counts


def test_two_calls_match_the_workspace_entry_point(capi):
    # first call: the V3 prefill shape fills the whole scratch (T * N = 4096 * 256);
    # second call: a smaller batch with different data and bias, reading an array
    # that still holds the first call's logits
    big = I.WORKLOADS["v3_prefill"]
    small = I.Workload("second", T=1000, H=7168, N=256, K=8, I=2048, bias_range=0.05, seed=7)
    for w in (big, small):
        x, gw, b = _inputs(w)
        got = _noalloc(capi, w, x, gw, b)
        ref = _reference(capi, w, x, gw, b)
        torch.cuda.synchronize()
        ids, gates, counts = (t.cpu().numpy() for t in got)
        rids, rgates, rcounts = (t.cpu().numpy() for t in ref)
        # against the oracle: the near-tie rule of every routing test, the
        # counts of the ids chosen, the gates from the unbiased affinities
        o_ids, _, s, score = O.route(I.bf16_bits_to_f32(I.make_x(w)), I.make_gate_w(w),
                                     I.make_bias(w), w.K)
        H.reconcile_ids(ids, o_ids, score, w.K)
        sel = np.take_along_axis(s, ids.astype(np.int64), axis=1)
        assert np.max(np.abs(gates - sel / sel.sum(axis=1, keepdims=True))) < 1e-5
        # the two entry points compute the fp32 logits differently (this one
        # with fp32 FMAs, moe_route on tensor cores), so ids may differ only on
        # tokens whose K-th and (K+1)-th scores are a near tie
        same = np.all(np.sort(ids, 1) == np.sort(rids, 1), axis=1)
        assert np.all(same | H.near_tie_tokens(score, w.K))
        assert counts.sum() == w.T * w.K
        assert np.array_equal(counts, O.expert_counts(ids, w.N))
        both = same & np.all(ids == rids, axis=1)
        assert np.max(np.abs(gates[both] - rgates[both])) <= 1e-5


def test_node_limited_routing_without_a_workspace(capi):
    """G = 4 groups of 4 experts, M = 2 per token, at the tiny shape: the ids
    lie in at most 2 groups and match the oracle's node-limited routing up to
    near ties of the group or expert scores."""
    from tests.test_gpu_routing_ext import _reconcile_grouped
    w = I.WORKLOADS["tiny"]
    x, gw, b = _inputs(w)
    got = _noalloc(capi, w, x, gw, b, groups=4, top=2)
    torch.cuda.synchronize()
    ids, gates, counts = (t.cpu().numpy() for t in got)
    assert np.all([len(set((ids[t] // 4).tolist())) <= 2 for t in range(w.T)])
    o_ids, _, s, score, gscore = O.route_grouped(I.bf16_bits_to_f32(I.make_x(w)),
                                                 I.make_gate_w(w), I.make_bias(w), w.K, 4, 2)
    _reconcile_grouped(ids, o_ids, score, gscore, w.K, 4, 2)
    assert np.array_equal(counts, O.expert_counts(ids, w.N))
    sel = np.take_along_axis(s, ids.astype(np.int64), axis=1)
    assert np.max(np.abs(gates - sel / sel.sum(axis=1, keepdims=True))) < 1e-5


def test_size_beyond_the_scratch_is_refused(capi):
    w = I.Workload("too_big", T=4097, H=256, N=256, K=8, I=128)
    sh = capi.shape_of(w.T, w.H, w.N, w.K, w.I)
    x = torch.zeros((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    gw = torch.zeros((w.N, w.H), dtype=torch.float32, device="cuda")
    b = torch.zeros((w.N,), dtype=torch.float32, device="cuda")
    ids, gates, counts = _outputs(w)
    rc = capi.LIB.moe_route_noalloc(sh, gw.data_ptr(), x.data_ptr(), b.data_ptr(), ids.data_ptr(),
                                    gates.data_ptr(), counts.data_ptr(), None)
    assert rc == -6  # MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert np.all(counts.cpu().numpy() == 12345)  # nothing was queued
