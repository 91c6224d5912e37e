"""Expert-parallel MoE layer over torch.distributed ranks (one GPU each).

The layer of "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, Multi-Token
Prediction, and FP8 Training at 671B Scale" (section V, "Training at Scale"
and "Custom all-to-all kernels") with its routed experts sharded over W
ranks: rank d holds experts [d N/W, (d+1) N/W), every rank holds the gate and
the shared expert, and every rank routes its own tokens. One step:

    dispatch   (library)  route, plan and FP8-pack this rank's send rows
    counts     all-to-all of [W, 2] int32 (rows, pairs) per rank pair
    rows       all-to-all of the packed rows (sizes from the counts)
    shared     (library)  the shared expert, while the rows are in flight
    experts    (library)  local grouped FP8 GEMMs on the received rows and
                          the per-row gate-weighted sums over local experts
    return     all-to-all of the fp32 partial sums back to their sources
    combine    (library)  shared + partials, one bf16 rounding

All arithmetic runs in the library's CUDA kernels; this module only sizes
buffers and moves rows between ranks with torch.distributed (NCCL on GPUs).
The row counts are read on the host once per step, because they size the
exchanges.

With peer=True the rows are not exchanged by all-to-alls: the dispatch and
expert kernels store them straight into the other ranks' receive and return
buffers (mapped into every process with CUDA IPC), and two stream-ordered
all-reduces of one int act as the barriers. There is no host
synchronisation in a step.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import capi


def exchange_counts(send_counts: torch.Tensor, group=None) -> torch.Tensor:
    """send_counts [W, 2] (row d: what this rank sends to rank d) ->
    recv_counts [W, 2] (row s: what rank s sends to this rank)."""
    recv = torch.empty_like(send_counts)
    dist.all_to_all_single(recv, send_counts.contiguous(), group=group)
    return recv


def exchange_rows(send: torch.Tensor, send_rows: list[int], recv_rows: list[int], group=None,
                  async_op: bool = False):
    """Rows send[:sum(send_rows)] (destination-major: send_rows[d] rows for
    rank d) -> recv [sum(recv_rows), ...] (source-major: recv_rows[s] rows from
    rank s, in the order rank s sent them). Returns (recv, work); work is None
    unless async_op."""
    n_send = int(sum(send_rows))
    recv = torch.empty((int(sum(recv_rows)),) + tuple(send.shape[1:]), dtype=send.dtype,
                       device=send.device)
    work = dist.all_to_all_single(recv, send[:n_send].contiguous(),
                                  output_split_sizes=[int(r) for r in recv_rows],
                                  input_split_sizes=[int(r) for r in send_rows], group=group,
                                  async_op=async_op)
    return recv, work


def check_same_layout(sizes: tuple, W: int, peer: bool, group=None) -> None:
    """sizes = (T, H, N, K, I, G, M) of this rank. The packed row layout needs
    the same H, N, K, I and routing groups on every rank; peer mode also needs
    the same T, the stride of every rank's buffer segments. Raises ValueError
    on every rank otherwise (a collective: all ranks call it)."""
    gathered = [None] * W
    dist.all_gather_object(gathered, tuple(sizes), group=group)
    first = 0 if peer else 1
    if any(t[first:] != gathered[0][first:] for t in gathered):
        raise ValueError(f"ranks were built with different sizes (T, H, N, K, I, G, M): {gathered}")


def local_weights(w13: torch.Tensor, s13: torch.Tensor, w2: torch.Tensor, s2: torch.Tensor,
                  N: int, W: int, rank: int):
    """Rank `rank`'s weight sets out of the full [N+1, ...] tensors: its N/W
    routed experts in order, then the shared expert (set N). Copies."""
    El = N // W
    pick = lambda t: torch.cat([t[rank * El:(rank + 1) * El], t[N:N + 1]]).contiguous()
    return pick(w13), pick(s13), pick(w2), pick(s2)


class ExpertParallelMoE:
    """One rank of the expert-parallel layer.

    gate_w: float32 [N, H] (all experts); w13, s13, w2, s2: this rank's N/W + 1
    weight sets (see local_weights), on this rank's GPU. T is the number of
    tokens this rank routes per step (the batch may be smaller: forward takes
    any T' <= T). With presplit_gate the centroids' three bf16 terms are made
    once here (resplit_gate after changing gate_w); without them every
    dispatch splits again.
    """

    def __init__(self, T: int, H: int, N: int, K: int, I: int, W: int, rank: int,
                 gate_w: torch.Tensor, w13: torch.Tensor, s13: torch.Tensor, w2: torch.Tensor,
                 s2: torch.Tensor, groups: int = 0, topk_groups: int = 0, group=None,
                 peer: bool = False, presplit_gate: bool = True):
        self.T, self.H, self.N, self.K, self.I, self.W, self.rank = T, H, N, K, I, W, rank
        self.G, self.M = groups, topk_groups
        self.group = group
        dev = gate_w.device
        self.device = dev
        sh = capi.shape_of(T, H, N, K, I, groups, topk_groups)
        if capi.moe_ep_dispatch_workspace_size(sh, W) == 0:
            raise ValueError("shape or rank count not supported for expert parallelism")
        self.row_bytes = capi.moe_ep_row_bytes(sh)
        self._keep = (gate_w, w13, s13, w2, s2)
        self.gate_w = gate_w
        self.gate_split = None
        if presplit_gate:
            self.gate_split = torch.empty((3, N, H), dtype=torch.bfloat16, device=dev)
            capi.moe_split_gate(gate_w, self.gate_split)
        self.w_local = capi.make_weights(gate_w, w13, s13, w2, s2)
        self.send = torch.empty(max(T * min(W, K), 1), self.row_bytes, dtype=torch.uint8,
                                device=dev)
        self.send_counts = torch.zeros(W, 2, dtype=torch.int32, device=dev)
        self.ws = torch.empty(capi.moe_ep_dispatch_workspace_size(sh, W), dtype=torch.uint8,
                              device=dev)
        self.ids = torch.empty(T, K, dtype=torch.int32, device=dev)
        self.gates = torch.empty(T, K, dtype=torch.float32, device=dev)
        self.counts = torch.zeros(N, dtype=torch.int32, device=dev)
        self._ews = torch.empty(0, dtype=torch.uint8, device=dev)
        self.last = {}
        self.peer = peer
        if W > 1:
            check_same_layout((T, H, N, K, I, groups, topk_groups), W, peer, group)
        if peer:
            # every rank's receive buffer, its counts and its return buffer,
            # T rows per source; other ranks' copies mapped into this process
            self.recv = torch.zeros(W * T, self.row_bytes, dtype=torch.uint8, device=dev)
            self.recv_counts = torch.zeros(W, dtype=torch.int32, device=dev)
            self.ret = torch.zeros(W * T, H, dtype=torch.float32, device=dev)
            ptrs = lambda views: torch.tensor([v.data_ptr() for v in views], dtype=torch.int64,
                                              device=dev)
            self._views = [self._peer_views(t) for t in (self.recv, self.recv_counts, self.ret)]
            self.p_recv, self.p_counts, self.p_ret = (ptrs(v) for v in self._views)
            self._ews = torch.empty(capi.moe_ep_peer_expert_workspace_size(sh, W, T),
                                    dtype=torch.uint8, device=dev)
            self._flag = torch.zeros(1, dtype=torch.int32, device=dev)

    def _peer_views(self, t: torch.Tensor):
        """t on every rank, as tensors of this process (CUDA IPC handles
        gathered over the group; this rank's own entry is t itself)."""
        if self.W == 1:
            return [t]
        from torch.multiprocessing.reductions import reduce_tensor
        rebuild, args = reduce_tensor(t)
        gathered = [None] * self.W
        dist.all_gather_object(gathered, args, group=self.group)
        return [t if r == self.rank else rebuild(*gathered[r]) for r in range(self.W)]

    def _barrier(self):
        """Every rank's kernels enqueued so far finish before any rank's
        next kernel starts (a stream-ordered all-reduce of one int)."""
        dist.all_reduce(self._flag, group=self.group)

    def _shape(self, T: int):
        return capi.shape_of(T, self.H, self.N, self.K, self.I, self.G, self.M)

    def _expert_ws(self, R: int, pairs: int) -> torch.Tensor:
        need = capi.moe_ep_expert_workspace_size(self._shape(self.T), self.W, R, pairs)
        if need > self._ews.numel():
            self._ews = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self._ews

    def forward(self, x: torch.Tensor, bias: torch.Tensor) -> torch.Tensor:
        """y = shared(x) + sum_k g_k expert_k(x) for this rank's tokens x
        (bf16 [T', H]); the routed experts run on the ranks that hold them.
        Every rank of the group must call forward in the same step."""
        T = x.shape[0]
        if T > self.T:
            raise ValueError(f"batch of {T} tokens exceeds the {self.T} this layer was sized for")
        sh = self._shape(T)
        c = capi
        if self.peer:
            return self._forward_peer(sh, x, bias)
        c.moe_ep_dispatch(sh, self.W, self.gate_w, x, bias, self.send, self.send_counts, self.ws,
                          topk_ids=self.ids[:T], topk_gates=self.gates[:T], counts=self.counts,
                          gate_split=self.gate_split)
        recv_counts = exchange_counts(self.send_counts, self.group)
        sc = self.send_counts.cpu()
        rc = recv_counts.cpu()
        send_rows = sc[:, 0].tolist()
        recv_rows = rc[:, 0].tolist()
        pairs = int(rc[:, 1].sum())
        R, S = int(sum(recv_rows)), int(sum(send_rows))
        recv, work = exchange_rows(self.send, send_rows, recv_rows, self.group, async_op=True)
        c.moe_ep_shared(sh, self.W, self.w_local, self.ws)  # overlaps the exchange
        if work is not None:
            work.wait()
        out = torch.empty(R, self.H, dtype=torch.float32, device=self.device)
        c.moe_ep_experts(sh, self.W, self.w_local, recv, R, pairs, out,
                         self._expert_ws(R, pairs))
        ret, _ = exchange_rows(out, recv_rows, send_rows, self.group)
        y = torch.empty(T, self.H, dtype=torch.bfloat16, device=self.device)
        c.moe_ep_combine(sh, self.W, ret, S, self.ws, y)
        self.last = {"send_rows": send_rows, "recv_rows": recv_rows, "pairs": pairs}
        return y

    def _forward_peer(self, sh, x, bias):
        c = capi
        T = x.shape[0]
        c.moe_ep_dispatch_peer(sh, self.W, self.rank, self.T, self.gate_w, x, bias, self.p_recv,
                               self.p_counts, self.ws, topk_ids=self.ids[:T],
                               topk_gates=self.gates[:T], counts=self.counts,
                               send_counts=self.send_counts, gate_split=self.gate_split)
        self._barrier()          # every rank's rows are in place
        c.moe_ep_shared(sh, self.W, self.w_local, self.ws)
        c.moe_ep_experts_peer(sh, self.W, self.rank, self.T, self.w_local, self.recv,
                              self.recv_counts, self.p_ret, self._ews)
        self._barrier()          # every rank's partial sums are back
        y = torch.empty(T, self.H, dtype=torch.bfloat16, device=self.device)
        c.moe_ep_combine_peer(sh, self.W, self.T, self.ret, self.ws, y)
        return y

    def resplit_gate(self, stream=None) -> None:
        """Re-make the centroids' bf16 terms after gate_w changed."""
        if self.gate_split is not None:
            capi.moe_split_gate(self.gate_w, self.gate_split, stream)

    def batch_counts(self) -> torch.Tensor:
        """Per-expert counts of the last step summed over all ranks (the
        bias controller balances the whole batch)."""
        total = self.counts.clone()
        dist.all_reduce(total, group=self.group)
        return total

    def status(self) -> int:
        """Device status of the last step on this rank (both workspaces)."""
        s = capi.moe_get_status(self.ws)
        if self._ews.numel() >= 4:
            s2 = capi.moe_get_status(self._ews)
            s = s if s != capi.MOE_OK else s2
        return s
