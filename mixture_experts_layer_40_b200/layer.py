"""A thin holder for one MoE layer on the GPU: shape, device weights and the
workspace, with methods that call the C ABI. All compute is in the CUDA
library; this module only owns memory and forwards pointers.

Also builds a workload's device weights from its block pool: the pool is
quantised on the GPU by moe_quantize_128x128 and the code/scale blocks are
placed into the ABI layout (w13 interleaves W_gate and W_up per 128 rows) by
indexing, which moves bytes and computes nothing.
"""
from __future__ import annotations

import dataclasses
import struct

import numpy as np
import torch

from . import capi
from .inputs import WeightPool, Workload


@dataclasses.dataclass
class DeviceWeights:
    gate_w: torch.Tensor  # [N, H] float32
    w13: torch.Tensor     # [E, 2I, H] uint8
    s13: torch.Tensor     # [E, 2I/128, H/128] float32
    w2: torch.Tensor      # [E, H, I] uint8
    s2: torch.Tensor      # [E, H/128, I/128] float32


def quantise_pool(pool: np.ndarray, device) -> tuple[torch.Tensor, torch.Tensor]:
    """[P,128,128] float32 blocks -> codes [P,128,128] uint8, scales [P]."""
    p = pool.shape[0]
    w = torch.from_numpy(np.ascontiguousarray(pool.reshape(p * 128, 128))).to(device)
    q = torch.empty((p * 128, 128), dtype=torch.uint8, device=device)
    s = torch.empty((p, 1), dtype=torch.float32, device=device)
    capi.moe_quantize_128x128(w, q, s)
    return q.view(p, 128, 128), s.view(p)


def _place(codes: torch.Tensor, scales: torch.Tensor, slots: np.ndarray, out_q: torch.Tensor,
           out_s: torch.Tensor, chunk: int = 16) -> None:
    """out_q[e] = block matrix of codes[slots[e]]; out_s[e] = scales[slots[e]]."""
    e_total, rb, cb = slots.shape
    idx_all = torch.from_numpy(np.ascontiguousarray(slots)).to(codes.device)
    for e0 in range(0, e_total, chunk):
        idx = idx_all[e0:e0 + chunk]
        blocks = codes[idx]  # [e, rb, cb, 128, 128]
        out_q[e0:e0 + chunk] = blocks.permute(0, 1, 3, 2, 4).reshape(idx.shape[0], rb * 128, cb * 128)
        out_s[e0:e0 + chunk] = scales[idx]


def device_weights(w: Workload, pool: WeightPool, gate_w: np.ndarray, device) -> DeviceWeights:
    q13, s13p = quantise_pool(pool.pool13, device)
    q2, s2p = quantise_pool(pool.pool2, device)
    e, ib, hb = w.E, w.I // 128, w.H // 128
    # row-block order of w13: gate block c, then up block c, for c = 0 .. I/128-1
    slots13 = np.stack([pool.slot_gate, pool.slot_up], axis=2).reshape(e, 2 * ib, hb)
    w13 = torch.empty((e, 2 * w.I, w.H), dtype=torch.uint8, device=device)
    s13 = torch.empty((e, 2 * ib, hb), dtype=torch.float32, device=device)
    _place(q13, s13p, slots13, w13, s13)
    w2 = torch.empty((e, w.H, w.I), dtype=torch.uint8, device=device)
    s2 = torch.empty((e, hb, ib), dtype=torch.float32, device=device)
    _place(q2, s2p, pool.slot_down, w2, s2)
    del q13, s13p, q2, s2p
    gw = torch.from_numpy(np.ascontiguousarray(gate_w, dtype=np.float32)).to(device)
    return DeviceWeights(gw, w13, s13, w2, s2)


class MoELayer:
    """One layer: forward(x, bias) -> y through moe_forward."""

    def __init__(self, T: int, H: int, N: int, K: int, I: int, weights: DeviceWeights,
                 device="cuda", groups: int = 0, topk_groups: int = 0, presplit_gate: bool = True):
        self.T, self.H, self.N, self.K, self.I = T, H, N, K, I
        self.shape = capi.shape_of(T, H, N, K, I, groups, topk_groups)
        nbytes = capi.moe_workspace_size(self.shape)
        if nbytes == 0:
            raise ValueError(f"unsupported shape T={T} H={H} N={N} K={K} I={I} "
                             f"G={groups} M={topk_groups}")
        self.device = torch.device(device)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.ws[:16].zero_()
        self.weights = weights
        # the centroids' three bf16 terms, made once here (resplit_gate after
        # changing weights.gate_w); without them every forward splits again
        self.gate_split = None
        if presplit_gate:
            self.gate_split = torch.empty((3, N, H), dtype=torch.bfloat16, device=self.device)
            capi.moe_split_gate(weights.gate_w, self.gate_split)
        self._cw = capi.make_weights(weights.gate_w, weights.w13, weights.s13, weights.w2,
                                     weights.s2, self.gate_split)
        self.layout = capi.moe_workspace_layout(self.shape)
        self.ids = torch.empty((T, K), dtype=torch.int32, device=self.device)
        self.gates = torch.empty((T, K), dtype=torch.float32, device=self.device)
        self.counts = torch.empty((N,), dtype=torch.int32, device=self.device)

    def forward(self, x: torch.Tensor, bias: torch.Tensor, y: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        if y is None:
            y = torch.empty((self.T, self.H), dtype=torch.bfloat16, device=self.device)
        capi.moe_forward(self.shape, self._cw, x, bias, y, self.ids, self.gates, self.counts,
                         self.ws, stream)
        return y

    def resplit_gate(self, stream=None) -> None:
        """Re-make the centroids' bf16 terms after weights.gate_w changed."""
        if self.gate_split is not None:
            capi.moe_split_gate(self.weights.gate_w, self.gate_split, stream)

    def weights_changed(self, stream=None) -> None:
        """After the weights were updated in place (gate_w, w13/s13, w2/s2):
        re-make the centroids' bf16 terms and, once a backward has made them,
        the transposed expert weights the backward reads."""
        self.resplit_gate(stream)
        if getattr(self, "_wt", None) is not None:
            capi.moe_transpose_weights(self.shape, self._cw, *self._wt_bufs, stream)

    def route(self, x: torch.Tensor, bias: torch.Tensor, stream=None):
        capi.moe_route(self.shape, self.weights.gate_w, x, bias, self.ids, self.gates,
                       self.counts, self.ws, stream)
        return self.ids, self.gates, self.counts

    def balance_stats(self, seq_len: int, alpha: float, stream=None):
        """f, P [S, N] and loss [S] of the last route/forward's routing."""
        n_seq = -(-self.T // seq_len)
        f = torch.empty((n_seq, self.N), dtype=torch.float32, device=self.device)
        p = torch.empty_like(f)
        loss = torch.empty((n_seq,), dtype=torch.float32, device=self.device)
        capi.moe_balance_stats(self.shape, seq_len, alpha, self.ws, self.ids, f, p, loss, stream)
        return f, p, loss

    def backward(self, dy: torch.Tensor, x: torch.Tensor | None = None, stream=None):
        """Input and gate gradients of the last forward for the upstream
        gradient dy (bf16 [T, H]), and with the forward's input x also the
        expert weight gradients; the transposed weights and the backward
        workspace are made on first use. Returns (dx bf16 [T, H], dgates
        [T, K]) or, with x, (dx, dgates, dw13 [E, 2I, H], dw2 [E, H, I])."""
        if getattr(self, "_wt", None) is None:
            E, H, I = self.N + 1, self.H, self.I
            dev = self.device
            self._wt_bufs = (torch.empty((E, H, 2 * I), dtype=torch.uint8, device=dev),
                             torch.empty((E, H // 128, 2 * I // 128), dtype=torch.float32,
                                         device=dev),
                             torch.empty((E, I, H), dtype=torch.uint8, device=dev),
                             torch.empty((E, I // 128, H // 128), dtype=torch.float32, device=dev))
            capi.moe_transpose_weights(self.shape, self._cw, *self._wt_bufs, stream)
            nb = capi.moe_backward_workspace_size(self.shape)
            if nb == 0:
                raise ValueError("the backward needs I to be a multiple of 256")
            self._bws = torch.empty(nb, dtype=torch.uint8, device=dev)
            w13t, s13t, w2t, s2t = self._wt_bufs
            self._wt = capi.make_weights(self.weights.gate_w, w13t, s13t, w2t, s2t)
        dx = torch.empty((self.T, self.H), dtype=torch.bfloat16, device=self.device)
        dgates = torch.empty((self.T, self.K), dtype=torch.float32, device=self.device)
        dw13 = dw2 = None
        if x is not None:
            E = self.N + 1
            dw13 = torch.empty((E, 2 * self.I, self.H), dtype=torch.float32, device=self.device)
            dw2 = torch.empty((E, self.H, self.I), dtype=torch.float32, device=self.device)
        capi.moe_backward(self.shape, self._cw, self._wt, self.ids, self.gates, x, dy, self.ws,
                          self._bws, dx, dgates, dw13, dw2, stream)
        return (dx, dgates) if x is None else (dx, dgates, dw13, dw2)

    def update_bias(self, bias: torch.Tensor, gamma: float, stream=None) -> None:
        capi.moe_update_bias(bias, self.counts, self.N, self.T, self.K, gamma, stream)

    def graphed_step(self, x: torch.Tensor, bias: torch.Tensor, y: torch.Tensor | None = None,
                     gamma: float | None = None) -> "GraphedStep":
        """The layer step on fixed buffers (x, bias, y) captured once as a CUDA
        graph: forward, and with gamma also the bias update. See GraphedStep."""
        return GraphedStep(self, x, bias, y, gamma)

    def status(self, stream=None) -> int:
        return capi.moe_get_status(self.ws, stream)

    def view(self, name: str, dtype: torch.dtype, shape) -> torch.Tensor:
        """A workspace intermediate (see moe_ws_layout) as a tensor view."""
        off = getattr(self.layout, name)
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        return self.ws[off:off + n].view(dtype).view(*shape)


class GraphedStep:
    """One layer step captured as a CUDA graph and replayed: the same kernels
    with the same arguments as layer.forward (and layer.update_bias when gamma
    is given), launched by one graph launch instead of one call per kernel.
    The library allocates nothing and launches everything on the stream it
    is given, so the capture holds the whole step; the tensor maps are
    encoded at capture time and hold the buffers' addresses, so x, bias and y
    must stay the same tensors (write new inputs into x in place). One
    uncaptured forward runs first, so that the one-time set-up per device
    (kernel attributes) happens outside the capture; it leaves the bias
    untouched."""

    def __init__(self, layer: MoELayer, x: torch.Tensor, bias: torch.Tensor,
                 y: torch.Tensor | None = None, gamma: float | None = None):
        self.layer, self.x, self.bias, self.gamma = layer, x, bias, gamma
        self.y = y if y is not None else torch.empty((layer.T, layer.H), dtype=torch.bfloat16,
                                                     device=layer.device)
        side = torch.cuda.Stream(layer.device)
        side.wait_stream(torch.cuda.current_stream(layer.device))
        with torch.cuda.stream(side):
            layer.forward(x, bias, self.y)
        torch.cuda.current_stream(layer.device).wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            layer.forward(x, bias, self.y)
            if gamma is not None:
                layer.update_bias(bias, gamma)

    def replay(self) -> torch.Tensor:
        """Runs the step on the current stream; returns y (the same tensor)."""
        self.graph.replay()
        return self.y


# ---------------------------------------------------------------- controller state
#
# The routing bias is the layer's only state that changes during training
# (the aux-loss-free controller, "DeepSeek-V3: Auxiliary-Loss-Free MoE Load
# Balancing...", section III). It is saved with its exact float32 bits, so a
# run resumed from the file takes the same routing decisions and bias steps
# as one that never stopped.
BIAS_MAGIC = b"MOEBIAS1"


def save_bias(path: str, bias: torch.Tensor, step: int, gamma: float) -> None:
    """Writes the bias (float32 [N], device or host) and the controller's step
    count and gamma: magic, then N and step (int64), gamma (float32), then
    the N float32 values, all little-endian."""
    b = bias.detach().to("cpu", torch.float32).contiguous().numpy()
    with open(path, "wb") as f:
        f.write(BIAS_MAGIC)
        f.write(struct.pack("<qqf", b.shape[0], int(step), float(gamma)))
        f.write(b.astype("<f4").tobytes())


def load_bias(path: str, device="cpu") -> tuple[torch.Tensor, int, float]:
    """Reads a file written by save_bias: (bias float32 [N] on `device`, step,
    gamma). Raises ValueError on a file of another format or a short file."""
    with open(path, "rb") as f:
        data = f.read()
    head = len(BIAS_MAGIC) + struct.calcsize("<qqf")
    if len(data) < head or data[:len(BIAS_MAGIC)] != BIAS_MAGIC:
        raise ValueError(f"{path}: not a routing-bias file")
    n, step, gamma = struct.unpack("<qqf", data[len(BIAS_MAGIC):head])
    if n < 0 or len(data) != head + 4 * n:
        raise ValueError(f"{path}: {len(data) - head} bytes of values for N = {n}")
    vals = np.frombuffer(data[head:], dtype="<f4").astype(np.float32)
    return torch.from_numpy(vals.copy()).to(device), int(step), float(gamma)
