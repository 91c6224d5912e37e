"""A layer step captured as a CUDA graph (MoELayer.graphed_step) against the
same step called kernel by kernel: the graph launches the same kernels with
the same arguments, so outputs, routing and the controlled bias are
identical bit for bit, over several steps of forward + bias update and after
new inputs are written into the captured x in place."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_40_b200 import inputs as I
from mixture_experts_layer_40_b200.layer import MoELayer, device_weights
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from __graft_entry__ import build
    build()
    assert torch.cuda.is_available()


def _pair(w):
    case = H.make_case(w)
    dw = device_weights(w, case.pool, case.gate_w, "cuda")
    return case, MoELayer(w.T, w.H, w.N, w.K, w.I, dw), MoELayer(w.T, w.H, w.N, w.K, w.I, dw)


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_graphed_steps_match_eager_steps(name):
    w = I.WORKLOADS[name]
    case, eager, graphed = _pair(w)
    x = H.x_to_device(case.x_bits)
    b_eager = torch.from_numpy(case.bias).cuda()
    b_graph = b_eager.clone()
    step = graphed.graphed_step(x, b_graph, gamma=1e-3)
    # the capture ran one uncaptured forward and changed nothing
    assert torch.equal(b_graph, b_eager)
    rng = np.random.default_rng(5)
    for i in range(4):
        if i == 2:
            # new inputs go into the captured buffer in place
            x.copy_(H.x_to_device(I.f32_to_bf16_bits(
                rng.standard_normal((w.T, w.H)).astype(np.float32))))
        y_e = eager.forward(x, b_eager)
        eager.update_bias(b_eager, 1e-3)
        y_g = step.replay()
        torch.cuda.synchronize()
        assert torch.equal(y_e, y_g), i
        assert torch.equal(eager.ids, graphed.ids) and torch.equal(eager.gates, graphed.gates)
        assert torch.equal(eager.counts, graphed.counts)
        assert torch.equal(b_eager, b_graph), i
    assert eager.status() == 0 and graphed.status() == 0


def test_graphed_forward_v3_prefill():
    w = I.WORKLOADS["v3_prefill"]
    case, eager, graphed = _pair(w)
    x = H.x_to_device(case.x_bits)
    b = torch.from_numpy(case.bias).cuda()
    step = graphed.graphed_step(x, b)
    y_g = step.replay()
    y_e = eager.forward(x, b)
    torch.cuda.synchronize()
    assert torch.equal(y_e, y_g)
    assert graphed.status() == 0
