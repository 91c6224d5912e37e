"""ctypes binding of the C ABI in include/moe_capi.h (libmoe_b200.so).

Argument marshalling only: every function takes torch tensors (device
memory), checks dtype / contiguity / device, and passes raw pointers, sizes
and the current CUDA stream to the library function of the same name. No
computation happens here, and there is no fallback: if the library is
missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_SHAPE", -2: "MOE_ERR_NULL", -3: "MOE_ERR_CUDA",
                -4: "MOE_ERR_TIMEOUT", -5: "MOE_ERR_BOUNDS", -6: "MOE_ERR_WORKSPACE",
                -7: "MOE_ERR_ALIGN"}


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("K", ctypes.c_int32), ("I", ctypes.c_int32), ("G", ctypes.c_int32),
                ("M", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [("gate_w", ctypes.c_void_p), ("w13", ctypes.c_void_p), ("s13", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("s2", ctypes.c_void_p), ("gate_split", ctypes.c_void_p)]


_LAYOUT_FIELDS = ["status", "counts", "offsets", "group_rows", "row_start", "row_token",
                  "token_row", "topk_ids", "topk_gates", "logits", "a_q", "a_s", "h_q", "h_s",
                  "y_rows", "gate_split", "bal_scratch", "perm_scratch", "total"]


class moe_ws_layout(ctypes.Structure):
    _fields_ = ([("routed_cap", ctypes.c_int64), ("rows_total", ctypes.c_int64)]
                + [(f, ctypes.c_size_t) for f in _LAYOUT_FIELDS])


# name -> (restype, argtypes) of every function declared in the header
_P = ctypes.c_void_p
_I32, _I64, _F32, _SZ = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "moe_quantize_1x128": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "moe_quantize_128x128": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P]),
    "moe_workspace_size": (_SZ, [moe_shape]),
    "moe_workspace_layout": (ctypes.c_int, [moe_shape, ctypes.POINTER(moe_ws_layout)]),
    "moe_split_gate": (ctypes.c_int, [_P, _I32, _I32, _P, _P]),
    "moe_route": (ctypes.c_int, [moe_shape, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_route_noalloc": (ctypes.c_int, [moe_shape, _P, _P, _P, _P, _P, _P, _P]),
    "moe_balance_stats": (ctypes.c_int, [moe_shape, ctypes.c_int32, ctypes.c_float, _P, _SZ, _P,
                                         _P, _P, _P, _P]),
    "moe_transpose_weights": (ctypes.c_int, [moe_shape, ctypes.POINTER(moe_weights), _P, _P, _P,
                                             _P, _P]),
    "moe_backward_workspace_size": (_SZ, [moe_shape]),
    "moe_backward": (ctypes.c_int, [moe_shape, ctypes.POINTER(moe_weights),
                                    ctypes.POINTER(moe_weights), _P, _P, _P, _P, _P, _SZ, _P, _SZ,
                                    _P, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [moe_shape, ctypes.POINTER(moe_weights), _P, _P, _P, _P, _P, _P,
                                   _P, _SZ, _P]),
    "moe_forward_traced": (ctypes.c_int, [moe_shape, ctypes.POINTER(moe_weights), _P, _P, _P, _P,
                                          _P, _P, _P, _SZ, _P, ctypes.POINTER(_P), _I32]),
    "moe_update_bias": (ctypes.c_int, [_P, _P, _I32, _I32, _I32, _F32, _P]),
    "moe_expert_up": (ctypes.c_int, [_I32, _I32, _I32, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_down": (ctypes.c_int, [_I32, _I32, _I32, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_down_bf16": (ctypes.c_int, [_I32, _I32, _I32, _P, _P, _I64, _P, _P, _P, _P, _P, _P,
                                            _P]),
    "moe_ep_row_bytes": (_I64, [moe_shape]),
    "moe_ep_dispatch_workspace_size": (_SZ, [moe_shape, _I32]),
    "moe_ep_dispatch": (ctypes.c_int, [moe_shape, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _I64, _P,
                                       _P, _SZ, _P]),
    "moe_ep_shared": (ctypes.c_int, [moe_shape, _I32, ctypes.POINTER(moe_weights), _P, _SZ, _P]),
    "moe_ep_expert_workspace_size": (_SZ, [moe_shape, _I32, _I64, _I64]),
    "moe_ep_experts": (ctypes.c_int, [moe_shape, _I32, ctypes.POINTER(moe_weights), _P, _I64,
                                      _I64, _P, _P, _SZ, _P]),
    "moe_ep_combine": (ctypes.c_int, [moe_shape, _I32, _P, _I64, _P, _SZ, _P, _P]),
    "moe_ep_peer_expert_workspace_size": (_SZ, [moe_shape, _I32, _I32]),
    "moe_ep_dispatch_peer": (ctypes.c_int, [moe_shape, _I32, _I32, _I32, _P, _P, _P, _P, _P, _P,
                                            _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_ep_experts_peer": (ctypes.c_int, [moe_shape, _I32, _I32, _I32,
                                           ctypes.POINTER(moe_weights), _P, _P, _P, _P, _SZ, _P]),
    "moe_ep_combine_peer": (ctypes.c_int, [moe_shape, _I32, _I32, _P, _P, _SZ, _P, _P]),
    "moe_get_status": (ctypes.c_int, [_P, _P]),
    "moe_device_sm_count": (ctypes.c_int, []),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_40_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def _check(name: str, code: int) -> None:
    if code != MOE_OK:
        raise MoeError(name, code)


def _ptr(t: torch.Tensor | None, dtype: torch.dtype | None = None, name: str = "tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def shape_of(T: int, H: int, N: int, K: int, I: int, G: int = 0, M: int = 0) -> moe_shape:
    """G, M: node-limited routing over G expert groups, M per token (G = 0: off)."""
    return moe_shape(T, H, N, K, I, G, M)


def moe_quantize_1x128(x: torch.Tensor, q: torch.Tensor, scales: torch.Tensor, stream=None):
    rows, cols = x.shape
    _check("moe_quantize_1x128", LIB.moe_quantize_1x128(
        _ptr(x, torch.bfloat16, "x"), rows, cols, _ptr(q, torch.uint8, "q"),
        _ptr(scales, torch.float32, "scales"), _stream(stream)))


def moe_quantize_128x128(w: torch.Tensor, q: torch.Tensor, scales: torch.Tensor, stream=None):
    rows, cols = w.shape
    _check("moe_quantize_128x128", LIB.moe_quantize_128x128(
        _ptr(w, torch.float32, "w"), rows, cols, _ptr(q, torch.uint8, "q"),
        _ptr(scales, torch.float32, "scales"), _stream(stream)))


def moe_workspace_size(sh: moe_shape) -> int:
    return int(LIB.moe_workspace_size(sh))


def moe_workspace_layout(sh: moe_shape) -> moe_ws_layout:
    out = moe_ws_layout()
    _check("moe_workspace_layout", LIB.moe_workspace_layout(sh, ctypes.byref(out)))
    return out


def moe_route(sh: moe_shape, gate_w, x, bias, topk_ids, topk_gates, counts, ws, stream=None):
    _check("moe_route", LIB.moe_route(
        sh, _ptr(gate_w, torch.float32, "gate_w"), _ptr(x, torch.bfloat16, "x"),
        _ptr(bias, torch.float32, "bias"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(counts, torch.int32, "counts"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_balance_stats(sh: moe_shape, seq_len: int, alpha: float, ws, topk_ids, f, P, loss,
                      stream=None):
    """Sequence-wise balance statistics of the routing the last moe_route /
    moe_forward on `ws` made: f, P float [S, N], loss float [S]."""
    _check("moe_balance_stats", LIB.moe_balance_stats(
        sh, seq_len, alpha, _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _ptr(topk_ids, torch.int32, "topk_ids"), _ptr(f, torch.float32, "f"),
        _ptr(P, torch.float32, "P"), _ptr(loss, torch.float32, "loss"), _stream(stream)))


def moe_transpose_weights(sh: moe_shape, w: moe_weights, w13t, s13t, w2t, s2t, stream=None):
    _check("moe_transpose_weights", LIB.moe_transpose_weights(
        sh, ctypes.byref(w), _ptr(w13t, torch.uint8, "w13t"), _ptr(s13t, torch.float32, "s13t"),
        _ptr(w2t, torch.uint8, "w2t"), _ptr(s2t, torch.float32, "s2t"), _stream(stream)))


def moe_backward_workspace_size(sh: moe_shape) -> int:
    return int(LIB.moe_backward_workspace_size(sh))


def moe_backward(sh: moe_shape, w: moe_weights, wt: moe_weights, topk_ids, topk_gates, x, dy, ws,
                 bws, dx, dgates, dw13=None, dw2=None, stream=None):
    _check("moe_backward", LIB.moe_backward(
        sh, ctypes.byref(w), ctypes.byref(wt), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(x, torch.bfloat16, "x"),
        _ptr(dy, torch.bfloat16, "dy"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _ptr(bws, torch.uint8, "bws"), bws.numel(), _ptr(dx, torch.bfloat16, "dx"),
        _ptr(dgates, torch.float32, "dgates"), _ptr(dw13, torch.float32, "dw13"),
        _ptr(dw2, torch.float32, "dw2"), _stream(stream)))


ROUTE_NOALLOC_MAX_LOGITS = 1048576


def moe_route_noalloc(sh: moe_shape, gate_w, x, bias, topk_ids, topk_gates, counts, stream=None):
    """moe_route without a workspace: the logits scratch is a fixed 4 MiB array
    inside the library (T * N <= ROUTE_NOALLOC_MAX_LOGITS). For callers that
    cannot give the library device memory; calls must not overlap on the GPU."""
    _check("moe_route_noalloc", LIB.moe_route_noalloc(
        sh, _ptr(gate_w, torch.float32, "gate_w"), _ptr(x, torch.bfloat16, "x"),
        _ptr(bias, torch.float32, "bias"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(counts, torch.int32, "counts"),
        _stream(stream)))


def make_weights(gate_w, w13, s13, w2, s2, gate_split=None) -> moe_weights:
    return moe_weights(_ptr(gate_w, torch.float32, "gate_w"), _ptr(w13, torch.uint8, "w13"),
                       _ptr(s13, torch.float32, "s13"), _ptr(w2, torch.uint8, "w2"),
                       _ptr(s2, torch.float32, "s2"),
                       None if gate_split is None else _ptr(gate_split, torch.bfloat16,
                                                            "gate_split"))


def _check_split_size(gate_split, N: int, H: int) -> None:
    # the three bf16 terms are written (moe_split_gate) or read whole
    if gate_split is not None and gate_split.numel() < 3 * N * H:
        raise ValueError(f"gate_split holds {gate_split.numel()} values; the three terms of "
                         f"[{N}, {H}] centroids need {3 * N * H}")


def moe_split_gate(gate_w, gate_split, stream=None):
    N, H = gate_w.shape
    _check_split_size(gate_split, N, H)
    _check("moe_split_gate", LIB.moe_split_gate(
        _ptr(gate_w, torch.float32, "gate_w"), N, H, _ptr(gate_split, torch.bfloat16, "gate_split"),
        _stream(stream)))


def moe_forward(sh: moe_shape, w: moe_weights, x, bias, y, topk_ids=None, topk_gates=None,
                counts=None, ws=None, stream=None):
    _check("moe_forward", LIB.moe_forward(
        sh, ctypes.byref(w), _ptr(x, torch.bfloat16, "x"), _ptr(bias, torch.float32, "bias"),
        _ptr(y, torch.bfloat16, "y"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(counts, torch.int32, "counts"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


TRACE_EVENTS = 7
TRACE_STAGES = ["route", "permute", "quantize", "expert_up", "expert_down", "combine"]


def moe_forward_traced(sh: moe_shape, w: moe_weights, x, bias, y, events, topk_ids=None,
                       topk_gates=None, counts=None, ws=None, stream=None):
    """moe_forward that also records `events` (TRACE_EVENTS torch.cuda.Event
    objects created with enable_timing=True) around its six stages."""
    arr = (_P * len(events))(*[ev.cuda_event for ev in events])
    _check("moe_forward_traced", LIB.moe_forward_traced(
        sh, ctypes.byref(w), _ptr(x, torch.bfloat16, "x"), _ptr(bias, torch.float32, "bias"),
        _ptr(y, torch.bfloat16, "y"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(counts, torch.int32, "counts"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream), arr, len(events)))


def moe_update_bias(bias, counts, N: int, T: int, K: int, gamma: float, stream=None):
    _check("moe_update_bias", LIB.moe_update_bias(
        _ptr(bias, torch.float32, "bias"), _ptr(counts, torch.int32, "counts"), N, T, K,
        float(gamma), _stream(stream)))


def moe_expert_up(H, I, n_groups, group_rows, group_start, rows, a_q, a_s, w13, s13, h_q, h_s,
                  status, stream=None):
    _check("moe_expert_up", LIB.moe_expert_up(
        H, I, n_groups, _ptr(group_rows, torch.int32), _ptr(group_start, torch.int32), rows,
        _ptr(a_q, torch.uint8), _ptr(a_s, torch.float32), _ptr(w13, torch.uint8),
        _ptr(s13, torch.float32), _ptr(h_q, torch.uint8), _ptr(h_s, torch.float32),
        _ptr(status), _stream(stream)))


def moe_expert_down(H, I, n_groups, group_rows, group_start, rows, h_q, h_s, w2, s2, y_rows,
                    status, stream=None):
    _check("moe_expert_down", LIB.moe_expert_down(
        H, I, n_groups, _ptr(group_rows, torch.int32), _ptr(group_start, torch.int32), rows,
        _ptr(h_q, torch.uint8), _ptr(h_s, torch.float32), _ptr(w2, torch.uint8),
        _ptr(s2, torch.float32), _ptr(y_rows, torch.float32), _ptr(status), _stream(stream)))


def moe_expert_down_bf16(H, I, n_groups, group_rows, group_start, rows, h_q, h_s, w2, s2, y_rows,
                         status, stream=None):
    _check("moe_expert_down_bf16", LIB.moe_expert_down_bf16(
        H, I, n_groups, _ptr(group_rows, torch.int32), _ptr(group_start, torch.int32), rows,
        _ptr(h_q, torch.uint8), _ptr(h_s, torch.float32), _ptr(w2, torch.uint8),
        _ptr(s2, torch.float32), _ptr(y_rows, torch.bfloat16), _ptr(status), _stream(stream)))


def moe_ep_row_bytes(sh: moe_shape) -> int:
    return int(LIB.moe_ep_row_bytes(sh))


def moe_ep_dispatch_workspace_size(sh: moe_shape, W: int) -> int:
    return int(LIB.moe_ep_dispatch_workspace_size(sh, W))


def moe_ep_expert_workspace_size(sh: moe_shape, W: int, R: int, pairs: int) -> int:
    return int(LIB.moe_ep_expert_workspace_size(sh, W, R, pairs))


def moe_ep_dispatch(sh: moe_shape, W: int, gate_w, x, bias, send, send_counts, ws,
                    topk_ids=None, topk_gates=None, counts=None, stream=None, gate_split=None):
    """send: uint8 [send_cap, moe_ep_row_bytes(sh)]; send_counts: int32 [W, 2];
    gate_split: None, or bf16 [3, N, H] from moe_split_gate."""
    _check_split_size(gate_split, sh.N, sh.H)
    _check("moe_ep_dispatch", LIB.moe_ep_dispatch(
        sh, W, _ptr(gate_w, torch.float32, "gate_w"),
        _ptr(gate_split, torch.bfloat16, "gate_split"), _ptr(x, torch.bfloat16, "x"),
        _ptr(bias, torch.float32, "bias"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(counts, torch.int32, "counts"),
        _ptr(send, torch.uint8, "send"), send.shape[0] if send is not None else 0,
        _ptr(send_counts, torch.int32, "send_counts"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def moe_ep_shared(sh: moe_shape, W: int, w_local: moe_weights, ws, stream=None):
    _check("moe_ep_shared", LIB.moe_ep_shared(
        sh, W, ctypes.byref(w_local), _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_ep_experts(sh: moe_shape, W: int, w_local: moe_weights, recv, R: int, pairs: int, out, ws,
                   stream=None):
    """recv: uint8 [>= R, row_bytes]; out: float32 [>= R, H]."""
    _check("moe_ep_experts", LIB.moe_ep_experts(
        sh, W, ctypes.byref(w_local), _ptr(recv, torch.uint8, "recv"), R, pairs,
        _ptr(out, torch.float32, "out"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def moe_ep_combine(sh: moe_shape, W: int, ret, ret_rows: int, ws, y, stream=None):
    _check("moe_ep_combine", LIB.moe_ep_combine(
        sh, W, _ptr(ret, torch.float32, "ret"), ret_rows, _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _ptr(y, torch.bfloat16, "y"), _stream(stream)))


def moe_ep_peer_expert_workspace_size(sh: moe_shape, W: int, T_cap: int) -> int:
    return int(LIB.moe_ep_peer_expert_workspace_size(sh, W, T_cap))


def moe_ep_dispatch_peer(sh: moe_shape, W: int, rank: int, T_cap: int, gate_w, x, bias,
                         peer_recv, peer_counts, ws, topk_ids=None, topk_gates=None, counts=None,
                         send_counts=None, stream=None, gate_split=None):
    """peer_recv, peer_counts: int64 device tensors [W] of device pointers;
    gate_split as in moe_ep_dispatch."""
    _check_split_size(gate_split, sh.N, sh.H)
    _check("moe_ep_dispatch_peer", LIB.moe_ep_dispatch_peer(
        sh, W, rank, T_cap, _ptr(gate_w, torch.float32, "gate_w"),
        _ptr(gate_split, torch.bfloat16, "gate_split"), _ptr(x, torch.bfloat16, "x"),
        _ptr(bias, torch.float32, "bias"), _ptr(topk_ids, torch.int32, "topk_ids"),
        _ptr(topk_gates, torch.float32, "topk_gates"), _ptr(counts, torch.int32, "counts"),
        _ptr(peer_recv, torch.int64, "peer_recv"), _ptr(peer_counts, torch.int64, "peer_counts"),
        _ptr(send_counts, torch.int32, "send_counts"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)))


def moe_ep_experts_peer(sh: moe_shape, W: int, rank: int, T_cap: int, w_local: moe_weights, recv,
                        recv_counts, peer_ret, ws, stream=None):
    """peer_ret: int64 device tensor [W] of device pointers."""
    _check("moe_ep_experts_peer", LIB.moe_ep_experts_peer(
        sh, W, rank, T_cap, ctypes.byref(w_local), _ptr(recv, torch.uint8, "recv"),
        _ptr(recv_counts, torch.int32, "recv_counts"), _ptr(peer_ret, torch.int64, "peer_ret"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)))


def moe_ep_combine_peer(sh: moe_shape, W: int, T_cap: int, ret, ws, y, stream=None):
    _check("moe_ep_combine_peer", LIB.moe_ep_combine_peer(
        sh, W, T_cap, _ptr(ret, torch.float32, "ret"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _ptr(y, torch.bfloat16, "y"), _stream(stream)))


def moe_get_status(ws, stream=None) -> int:
    return int(LIB.moe_get_status(_ptr(ws), _stream(stream)))


def moe_device_sm_count() -> int:
    return int(LIB.moe_device_sm_count())
