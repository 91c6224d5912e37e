"""Save and load of the routing bias, the layer's only changing state (the
aux-loss-free controller of "DeepSeek-V3: Auxiliary-Loss-Free MoE Load
Balancing...", section III): the float32 bits survive the round trip, so a
resumed controller run continues bit for bit; files of another format are
refused."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_40_b200.layer import load_bias, save_bias


def test_round_trip_keeps_every_bit(tmp_path):
    rng = np.random.default_rng(3)
    b = rng.uniform(-0.1, 0.1, 256).astype(np.float32)
    b[:4] = [0.0, -0.0, np.float32(1e-45), np.float32(-3.4e38)]
    p = tmp_path / "bias.bin"
    save_bias(str(p), torch.from_numpy(b), step=17, gamma=1e-3)
    got, step, gamma = load_bias(str(p))
    assert got.dtype == torch.float32
    assert np.array_equal(got.numpy().view(np.uint32), b.view(np.uint32))
    assert step == 17 and gamma == np.float32(1e-3)


def test_resumed_controller_matches_an_uninterrupted_run(tmp_path):
    """The oracle's controller on fixed loads: 10 steps in one go against 4
    steps, save, load, 6 more steps."""
    rng = np.random.default_rng(4)
    n, t, k = 64, 512, 4
    loads = [rng.multinomial(t * k, rng.dirichlet(np.ones(n))).astype(np.int32) for _ in range(10)]
    b = np.zeros(n, np.float32)
    for c in loads:
        b = O.update_bias(b, c, t, k, 1e-3)
    r = np.zeros(n, np.float32)
    for c in loads[:4]:
        r = O.update_bias(r, c, t, k, 1e-3)
    p = tmp_path / "ctl.bin"
    save_bias(str(p), torch.from_numpy(r), step=4, gamma=1e-3)
    rt, step, gamma = load_bias(str(p))
    r = rt.numpy()
    for c in loads[step:]:
        r = O.update_bias(r, c, t, k, gamma)
    assert np.array_equal(r.view(np.uint32), b.view(np.uint32))


def test_other_files_are_refused(tmp_path):
    p = tmp_path / "x.bin"
    p.write_bytes(b"NOTABIAS" + bytes(40))
    with pytest.raises(ValueError):
        load_bias(str(p))
    save_bias(str(p), torch.zeros(8), 0, 1e-3)
    p.write_bytes(p.read_bytes()[:-4])
    with pytest.raises(ValueError):
        load_bias(str(p))
