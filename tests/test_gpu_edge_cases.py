"""GPU edge cases of the layer forward against the oracle: an empty batch, an
all-zero input (every score ties, every tile has the zero-tile scale), every
expert selected (K = N), and the largest supported expert count and K
(N = 1024, K = 16; 1025 GEMM groups)."""
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


def _layer(w, case):
    return MoELayer(w.T, w.H, w.N, w.K, w.I, device_weights(w, case.pool, case.gate_w, "cuda"))


def test_empty_batch():
    w = I.Workload("empty", T=0, H=256, N=16, K=4, I=128, bias_range=0.1, seed=21)
    pool_w = I.Workload("pool", T=1, H=256, N=16, K=4, I=128, bias_range=0.1, seed=21)
    case = H.make_case(pool_w)
    layer = MoELayer(0, w.H, w.N, w.K, w.I, device_weights(pool_w, case.pool, case.gate_w, "cuda"))
    layer.counts.fill_(7)
    bd = torch.from_numpy(case.bias).cuda()
    y = layer.forward(torch.empty((0, w.H), dtype=torch.bfloat16, device="cuda"), bd)
    assert y.shape == (0, w.H)
    assert layer.status() == 0
    assert torch.count_nonzero(layer.counts).item() == 0
    layer.update_bias(bd, w.gamma)
    # no load, so sign(T*K - N*c) = 0 for every expert: the bias is unchanged
    nb = O.update_bias(case.bias, np.zeros(w.N, np.int32), 0, w.K, w.gamma)
    assert np.array_equal(bd.cpu().numpy(), nb) and np.array_equal(nb, case.bias)


def test_all_zero_input():
    w = I.Workload("zero", T=77, H=512, N=32, K=4, I=256, bias_range=0.0, seed=22)
    case = H.make_case(w)
    x_bits = np.zeros((w.T, w.H), np.uint16)
    bias = np.zeros(w.N, np.float32)
    layer = _layer(w, case)
    y = H.bf16_to_f32(layer.forward(H.x_to_device(x_bits), torch.from_numpy(bias).cuda()))
    assert layer.status() == 0
    # every affinity is sigmoid(0) = 0.5: all ties, so experts 0..K-1 win and
    # every gate is 1/K; every tile is all-zero (scale 1, codes 0), y = 0
    ids, gates, _, _ = O.route(np.zeros((w.T, w.H), np.float32), case.gate_w, bias, w.K)
    assert np.array_equal(layer.ids.cpu().numpy(), ids)
    assert np.array_equal(ids, np.tile(np.arange(w.K, dtype=np.int32), (w.T, 1)))
    assert np.all(layer.gates.cpu().numpy() == np.float32(1.0 / w.K))
    assert np.all(y == 0.0)
    a_s = layer.view("a_s", torch.float32, (layer.layout.rows_total, w.H // 128))
    assert torch.all(a_s[layer.layout.routed_cap:layer.layout.routed_cap + w.T] == 1.0)


def test_every_expert_selected():
    w = I.Workload("kn", T=50, H=256, N=16, K=16, I=128, bias_range=0.1, seed=23)
    case = H.make_case(w)
    layer = _layer(w, case)
    y = H.bf16_to_f32(layer.forward(H.x_to_device(case.x_bits), torch.from_numpy(case.bias).cuda()))
    assert layer.status() == 0
    gid = layer.ids.cpu().numpy()
    assert np.all(np.sort(gid, axis=1) == np.arange(16))
    assert np.array_equal(layer.counts.cpu().numpy(), np.full(16, w.T, np.int32))
    r_ids, _, _, score = O.route(case.x, case.gate_w, case.bias, w.K)
    use, _, _ = H.reconcile_ids(gid, r_ids, score, w.K)
    H.expert_path_parity(w, case, layer, y, use, np.arange(w.T))


def test_largest_expert_count_and_k():
    w = I.Workload("maxn", T=256, H=256, N=1024, K=16, I=128, bias_range=0.1, seed=24)
    case = H.make_case(w)
    layer = _layer(w, case)
    y = H.bf16_to_f32(layer.forward(H.x_to_device(case.x_bits), torch.from_numpy(case.bias).cuda()))
    assert layer.status() == 0
    gid = layer.ids.cpu().numpy()
    r_ids, _, _, score = O.route(case.x, case.gate_w, case.bias, w.K)
    use, _, _ = H.reconcile_ids(gid, r_ids, score, w.K)
    assert np.array_equal(layer.counts.cpu().numpy(), O.expert_counts(use, w.N))
    H.expert_path_parity(w, case, layer, y, use, np.arange(w.T))


_TWO_THREADS = r"""
import sys, threading
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from mixture_experts_layer_40_b200 import inputs as I
from mixture_experts_layer_40_b200.layer import MoELayer, device_weights
w = I.Workload("threads", T=200, H=512, N=32, K=4, I=256, bias_range=0.1, seed=77)
xb = I.make_x(w)
pool = I.make_weight_pool(w)
layers = [MoELayer(w.T, w.H, w.N, w.K, w.I, device_weights(w, pool, I.make_gate_w(w), "cuda"))
          for _ in range(2)]
x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
bias = torch.from_numpy(I.make_bias(w)).cuda()
torch.cuda.synchronize()
start = threading.Barrier(2)
out, errors = [None, None], []
def run(i):
    try:
        torch.cuda.set_device(0)
        s = torch.cuda.Stream()
        start.wait()
        with torch.cuda.stream(s):
            out[i] = layers[i].forward(x, bias, stream=s)
            out[i] = out[i].clone()
        s.synchronize()
        assert layers[i].status(s) == 0
    except Exception as e:
        errors.append(repr(e))
ts = [threading.Thread(target=run, args=(i,)) for i in range(2)]
[t.start() for t in ts]
[t.join() for t in ts]
assert not errors, errors
assert torch.equal(out[0], out[1])
assert torch.equal(out[0], layers[0].forward(x, bias))
print("ok")
"""


def test_first_calls_from_two_host_threads():
    """The once-per-device set-up of the kernels (shared-memory limits, the
    register-count check) is taken under a lock: in a fresh process, two host
    threads whose first library calls run at the same time on one device
    both get the layer's result, bit for bit."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _TWO_THREADS, root], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
