"""Benchmark of the MoE layer forward (plus the per-step bias update) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3_prefill]
                    [--impl ours|reference] [--no-cpu-baseline] [--backward]
                    [--groups G --topk-groups M] [--ep [--peer]]

`--backward` also times the FP8 backward of the expert path after the step;
`--groups/--topk-groups` route node-limited; `--ep` runs the expert-parallel
step instead (routed experts sharded over the ranks), `--peer` with the
kernels storing rows into the other ranks' buffers.

With --gpus N > 1 and no rank environment (RANK / WORLD_SIZE), bench.py
starts the N ranks itself under torchrun on 127.0.0.1.

One step = one pass of the whole hot path on one batch of synthetic input:
quantise x, route, permute, up/gate GEMM + SwiGLU + re-quantisation, down
GEMM, combine, and the aux-loss-free bias update. With N > 1 ranks (torchrun,
one GPU each) every rank runs its own batch (weak scaling) and the per-expert
counts are summed across ranks (NCCL all-reduce of N int32) before the bias
update, since the controller balances the whole batch.

Rank 0 prints one JSON line. `value` is tokens per second of the whole job
with inputs resident in HBM; `e2e` is the same through the public API with
the input copied from pinned host memory and the output copied back inside
the timed region. `--impl reference` times the CPU oracle instead (a bounded
sample of the same workload per step, scaled to the whole layer).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s and grouped-GEMM FP8 TFLOP/s (% of B200 dense FP8 peak)"
FP8_SPEC_TFLOPS = 4500.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="v3_prefill")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-fp8-peak", action="store_true")
    p.add_argument("--groups", type=int, default=0,
                   help="node-limited routing: G expert groups (0: top-K over all N)")
    p.add_argument("--topk-groups", type=int, default=0, help="node-limited routing: M groups")
    p.add_argument("--ep", action="store_true",
                   help="expert parallelism: the routed experts sharded over the ranks "
                        "(ep.ExpertParallelMoE), every rank routing its own batch")
    p.add_argument("--peer", action="store_true",
                   help="with --ep: the kernels store rows straight into the other ranks' "
                        "buffers (CUDA IPC), no all-to-alls and no host synchronisation")
    p.add_argument("--backward", action="store_true",
                   help="also time the FP8 expert backward (Dgrad + Wgrad) after the forward")
    p.add_argument("--launch-check", action="store_true",
                   help="start the ranks, exchange one value, print n_gpus; no kernels")
    p.add_argument("--seq-len", type=int, default=0,
                   help="sequence length for the balance statistics (0: the whole batch)")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples (every 50 ms) while the timed regions run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- workload

def algorithmic_work(w, counts: np.ndarray):
    """Bytes and FLOPs each expert GEMM launch must move / compute."""
    rows = w.T * w.K + w.T
    touched = int(np.count_nonzero(counts)) + 1  # + the shared expert
    hb, ib = w.H // 128, w.I // 128
    w13_bytes = touched * (2 * w.I * w.H + 2 * ib * hb * 4)
    w2_bytes = touched * (w.H * w.I + hb * ib * 4)
    a_bytes = rows * (w.H + hb * 4)
    h_bytes = rows * (w.I + ib * 4)
    y_bytes = rows * w.H * 2
    return {
        "expert_up": {"bytes": w13_bytes + a_bytes + h_bytes, "flops": 2.0 * rows * w.H * 2 * w.I},
        "expert_down": {"bytes": w2_bytes + h_bytes + y_bytes, "flops": 2.0 * rows * w.I * w.H},
        # x read once, codes + scales written to the shared row and K routed rows
        "quantize": {"bytes": w.T * w.H * 2 + (w.K + 1) * w.T * (w.H + hb * 4), "flops": 0.0},
        "combine": {"bytes": (w.T * w.K + w.T) * w.H * 2 + w.T * w.H * 2, "flops": 0.0},
        # ids read, row_token and token_row written
        "permute": {"bytes": 3 * w.T * w.K * 4, "flops": 0.0},
        "route": {"bytes": w.T * w.H * 2 + w.N * w.H * 4, "flops": 2.0 * w.T * w.N * w.H},
    }


GEMM_SOURCES = ["mixture_experts_layer_40_b200/csrc/gemm.cu",
                "mixture_experts_layer_40_b200/csrc/common.cuh"]
# one line per recorded capture: "traffic <kernel> bytes=<B> workload=<name>
# fingerprint=<gemm sources> [key=value ...]"; the summary beside it says how
# each figure was taken
TRAFFIC_FILE = "profiles/grouped_gemm_traffic.txt"


def gemm_fingerprint() -> str:
    """Hash of the grouped-GEMM sources: a recorded DRAM capture is only
    reported while the kernel it measured is unchanged."""
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def roofline_of(work: dict, ms: float, hbm_gbs: float, fp8_tflops: float) -> dict:
    """The kernel's bound from its arithmetic intensity against the ridge
    point of the two peaks (FLOPs per byte at which both take equal time),
    and the achieved rate as a fraction of that peak."""
    intensity = work["flops"] / work["bytes"] if work["bytes"] else 0.0
    ridge = fp8_tflops * 1e12 / (hbm_gbs * 1e9)
    if work["flops"] > 0 and intensity > ridge:
        achieved = work["flops"] / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": achieved, "peak": fp8_tflops, "unit": "TFLOP/s",
                "frac": achieved / fp8_tflops, "intensity_flop_per_byte": intensity,
                "ridge_flop_per_byte": ridge}
    achieved = work["bytes"] / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
            "frac": achieved / hbm_gbs, "intensity_flop_per_byte": intensity,
            "ridge_flop_per_byte": ridge}


def recorded_traffic(kernel: str, workload: str):
    """dram__bytes_read.sum + dram__bytes_write.sum of one launch of `kernel`
    from the committed ncu summary, or None when there is none for this
    workload or the GEMM sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, TRAFFIC_FILE)) as fh:
            lines = fh.read().splitlines()
        fp = gemm_fingerprint()
    except OSError:
        return None
    for ln in lines:
        f = ln.split()
        if len(f) >= 5 and f[0] == "traffic" and f[1] == kernel:
            kv = dict(x.split("=", 1) for x in f[2:] if "=" in x)
            if kv.get("workload") == workload and kv.get("fingerprint") == fp:
                return int(kv["bytes"])
    return None


def measure_fp8_peak(torch, device):
    """Dense FP8 E4M3 GEMM throughput of the vendor library (torch._scaled_mm,
    8192^3, per-tensor scales): the measured denominator for the FP8 fraction."""
    n = 8192
    a = torch.randn(n, n, device=device).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=device).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=device)
    for _ in range(3):
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(10):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e.record()
        e.synchronize()
        best = min(best, s.elapsed_time(e))
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


# ---------------------------------------------------------------- CPU oracle

def router_launches(T: int, N: int, K: int, G: int, M: int, H: int, sms: int = 148) -> int:
    """Kernels the router launches per forward (the centroids are split once
    at set-up), following launch_router_tc in csrc/router.cu: wide tiles
    (`use_wide_logits`) make the selection in their epilogue at N = 256,
    K <= 8 (plain, or node-limited with 8 groups), else logits + top-K;
    smaller batches split the reduction (`splitk_slices`: logits, slice sum,
    top-K) or run 128 x 64 tiles (logits, top-K)."""
    small = -(-T // 128) * -(-N // 64)
    wide = -(-T // 256) * -(-N // 256)
    if N % 256 == 0 and 10 * -(-small // sms) > 32 * -(-wide // sms):
        grouped = G > 1 and M < G
        return 1 if N == 256 and K <= 8 and (not grouped or G == 8) else 2
    if N % 256 == 0 and T > 0 and min(148 // wide, (H // 32) // 8) >= 2:
        return 3
    return 2


def step_launches(T: int, N: int, K: int, G: int, M: int, H: int) -> int:
    """The library's kernels in one timed step: the router's, rank + scan +
    place (the permutation), quantise-and-scatter, up GEMM, down GEMM,
    combine, bias update."""
    return router_launches(T, N, K, G, M, H) + 3 + 5


def ep_step_launches(T: int, N: int, K: int, G: int, M: int, H: int) -> int:
    """The library's kernels in one expert-parallel step on a rank that
    receives rows (csrc/ep.cu; the centroids are split once at set-up): the
    router's, then count, slot and pack (the send plan); the shared expert's
    two GEMMs; on the receiver the index kernel, rank + scan + place, the row
    gather, two GEMMs and the per-row reduction; the combine; the bias
    update."""
    return router_launches(T, N, K, G, M, H) + 3 + 2 + 1 + 3 + 1 + 2 + 1 + 1 + 1


def oracle_sample_step(w, x, gate_w, bias, ew, step: int, sample_tokens: int = 512,
                       groups: int = 1, shared_rows: int = 64, node_limit: tuple = (0, 0)):
    """One bounded sample of the layer on the CPU oracle; returns its time
    scaled to the whole layer. The sample (a window of `sample_tokens`
    tokens moving with the step): their quantisation, routing, permutation
    and combine (scaled by T / sample); `groups` routed experts, each with
    the sampled tokens that chose it (assembly of the expert's weights timed
    once per expert, its FFN scaled by T / sample, then both by N / groups);
    the shared expert on `shared_rows` of the sampled tokens (its FFN scaled
    to all T tokens)."""
    from oracle import moe_oracle as O
    n = min(w.T, sample_tokens)
    t0s = (step * n) % max(1, w.T - n + 1)
    xs_ = x[t0s:t0s + n]
    scale = w.T / n
    t0 = time.perf_counter()
    xq, xsc = O.quantize_1x128(xs_)
    if node_limit[0] > 1 and node_limit[1] < node_limit[0]:
        ids, gates, *_ = O.route_grouped(xs_, gate_w, bias, w.K, node_limit[0], node_limit[1])
    else:
        ids, gates, _, _ = O.route(xs_, gate_w, bias, w.K)
    O.permutation(ids, w.N)
    t_tokens = time.perf_counter() - t0
    y_routed = np.zeros((n, w.K, w.H))
    t_assemble = t_ffn = 0.0
    for j in range(groups):
        e = (step * groups + j) % w.N
        t0 = time.perf_counter()
        wts = ew.dequantised(e)
        t_assemble += time.perf_counter() - t0
        rr, kk = np.nonzero(ids == e)
        t0 = time.perf_counter()
        if len(rr):
            y_routed[rr, kk] = O.expert_ffn_q(xq[rr], xsc[rr], *wts)[0]
        t_ffn += time.perf_counter() - t0
    m = min(shared_rows, n)
    t0 = time.perf_counter()
    wts = ew.dequantised(w.N)
    t_shared_assemble = time.perf_counter() - t0
    t0 = time.perf_counter()
    y_shared = np.zeros((n, w.H))
    y_shared[:m] = O.expert_ffn_q(xq[:m], xsc[:m], *wts)[0]
    t_shared = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.combine(y_shared, y_routed, ids, gates)
    t_combine = time.perf_counter() - t0
    return ((t_tokens + t_combine) * scale + (t_assemble + t_ffn * scale) * w.N / groups
            + t_shared_assemble + t_shared * w.T / m)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_setup(w, x_bits):
    from mixture_experts_layer_40_b200 import inputs as I
    from oracle import moe_oracle as O
    pool = I.make_weight_pool(w)
    ew = O.ExpertWeights(pool.pool13, pool.pool2, pool.slot_gate, pool.slot_up, pool.slot_down)
    # the quantised and dequantised block pools are built once, untimed (the
    # first dequantised() call builds the pool every expert is assembled from)
    ew.quantised_pools()
    ew.dequantised(0)
    return I.bf16_bits_to_f32(x_bits), I.make_gate_w(w), I.make_bias(w), ew


def oracle_sample_text(w, steps: int) -> str:
    return (f"{steps} steps, each extrapolated from a sample: quantisation, routing, "
            f"permutation and combine of 512 of the {w.T} tokens (scaled by T/512), 1 of the "
            f"{w.N} routed experts on its sampled tokens (weight assembly + FFN, scaled by "
            f"T/512 and N) and the shared expert on 64 tokens (scaled to T); block pools "
            f"built before timing")


# ---------------------------------------------------------------- ranks

def rank_batch(w, rank: int):
    """Weak scaling: every rank routes its own batch of T tokens (its own
    seed); the weights, centroids and starting bias are the same on all."""
    return dataclasses.replace(w, seed=w.seed + rank)


def batch_counts(counts, world: int):
    """The bias controller balances the whole batch: per-expert counts are
    summed over the ranks (one all-reduce of N int32) before the update,
    which then uses T_total = world * T."""
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(counts)
    return counts


def max_over_ranks(v: float, world: int, device) -> float:
    """A multi-rank time is the slowest rank's."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_config(args, w, world: int) -> dict:
    """The `config` object of both arms' lines."""
    weight_gb = (w.N + 1) * 3 * w.H * w.I / 1e9
    return {"workload": f"{w.name}: T={w.T} per GPU, H={w.H}, N={w.N} routed top-{w.K} "
                        f"+ 1 shared, I={w.I}, SwiGLU, FP8 E4M3 1x128/128x128",
            "tokens_per_gpu": w.T, "parallelism": f"dp{world} (weak: own batch per GPU)",
            "routing": (f"node-limited: {args.topk_groups} of {args.groups} expert groups"
                        if args.groups > 1 and args.topk_groups < args.groups
                        else f"top-{w.K} of all {w.N}"),
            "l2": f"no flush: each step streams {weight_gb:.2f} GB of expert weights, "
                  f"{weight_gb * 1e3 / 126:.0f}x the 126 MB L2"}


def run_reference(args, w, rank):
    if rank != 0:
        return
    from mixture_experts_layer_40_b200 import inputs as I
    x, gate_w, bias, ew = oracle_setup(w, I.make_x(w))
    for s in range(args.warmup):
        oracle_sample_step(w, x, gate_w, bias, ew, s, node_limit=(args.groups, args.topk_groups))
    times = [oracle_sample_step(w, x, gate_w, bias, ew, args.warmup + s,
                                node_limit=(args.groups, args.topk_groups))
             for s in range(args.steps)]
    ms = 1e3 * float(np.mean(times))
    value = w.T / (ms * 1e-3)
    sample = oracle_sample_text(w, args.steps)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": run_config(args, w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm

def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from __graft_entry__ import build
    build()
    from mixture_experts_layer_40_b200 import capi
    from mixture_experts_layer_40_b200 import inputs as I
    from mixture_experts_layer_40_b200.layer import MoELayer, device_weights

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wr = rank_batch(w, rank)
    x_bits = I.make_x(wr)
    pool = I.make_weight_pool(w)   # same weights on every rank
    gate_w = I.make_gate_w(w)
    bias0 = I.make_bias(w)
    layer = MoELayer(w.T, w.H, w.N, w.K, w.I, device_weights(w, pool, gate_w, dev), dev,
                     groups=args.groups, topk_groups=args.topk_groups)
    del pool
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    x = x_host.to(dev)
    y = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
    y_host = torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory()
    bias = torch.from_numpy(bias0).to(dev)
    stream = torch.cuda.current_stream()
    t_total = w.T * world

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(capi.TRACE_EVENTS)]
              for _ in range(args.steps)]
    for evs in events:
        for ev in evs:
            ev.record(stream)
    launches_per_step = step_launches(w.T, w.N, w.K, args.groups, args.topk_groups, w.H)

    def step(traced_events=None, x_in=x, y_out=y):
        if traced_events is None:
            capi.moe_forward(layer.shape, layer._cw, x_in, bias, y_out, layer.ids, layer.gates,
                             layer.counts, layer.ws)
        else:
            capi.moe_forward_traced(layer.shape, layer._cw, x_in, bias, y_out, traced_events,
                                    layer.ids, layer.gates, layer.counts, layer.ws)
        batch_counts(layer.counts, world)
        capi.moe_update_bias(bias, layer.counts, w.N, t_total, w.K, w.gamma)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    if layer.status() != 0:
        raise RuntimeError("device status error during warm-up")

    # ------------------------------------------------ timed region (HBM-resident inputs)
    clocks = ClockSampler(local_rank) if rank == 0 else None
    if clocks:
        clocks.start()
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        step(events[k])
    t_end.record(stream)
    barrier()
    ms_total = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    ms_step = ms_total / args.steps
    stage_ms = {name: float(np.mean([evs[i].elapsed_time(evs[i + 1]) for evs in events]))
                for i, name in enumerate(capi.TRACE_STAGES)}
    if layer.status() != 0:
        raise RuntimeError("device status error in the timed region")
    counts = layer.counts.cpu().numpy()

    # ------------------------------------------------ end to end (host buffers)
    # Every step copies its input from pinned host memory and its output back.
    # The copies run on their own streams with two device buffers each way, so
    # step i+1's upload and step i-1's download overlap step i's kernels; the
    # layer's steps themselves stay in order on the compute stream (each
    # step's routing uses the bias the previous step updated).
    up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()
    xs = [x, torch.empty_like(x)]
    ys = [y, torch.empty_like(y)]
    y_hosts = [y_host, torch.empty_like(y_host).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        b = i % 2
        up_s.wait_event(ev_done[b])          # step i-2 no longer reads xs[b]
        with torch.cuda.stream(up_s):
            xs[b].copy_(x_host, non_blocking=True)
        ev_in[b].record(up_s)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])         # ys[b] of step i-2 is downloaded
        step(x_in=xs[b], y_out=ys[b])
        ev_done[b].record(stream)
        down_s.wait_event(ev_done[b])
        with torch.cuda.stream(down_s):
            y_hosts[b].copy_(ys[b], non_blocking=True)
        ev_out[b].record(down_s)

    for i in range(2):
        e2e_step(i)
    barrier()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    up_s.wait_event(e_start)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(ev_out[0])
    stream.wait_event(ev_out[1])
    e_end.record(stream)
    barrier()
    # ------------------------------------------------ the same step as a CUDA graph
    # captured once and replayed (one graph launch per step instead of one
    # call per kernel); one GPU only (the count all-reduce is not captured)
    graph = None
    if world == 1 and args.steps > 0:
        gstep = layer.graphed_step(x, bias, y, gamma=w.gamma)
        for _ in range(3):
            gstep.replay()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            gstep.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        if layer.status() != 0:
            raise RuntimeError("device status error in the graph replays")
        g_ms = g0.elapsed_time(g1) / args.steps
        graph = {"value": w.T / (g_ms * 1e-3), "unit": "tokens/s", "ms_per_step": g_ms,
                 "note": "the timed step (forward + bias update, no stage events) captured "
                         "once as a CUDA graph and replayed; measured after the end-to-end "
                         "run, on a warmer GPU under the power cap than the timed region"}
        del gstep
    # ------------------------------------------------ controller trace (untimed)
    # workloads with several steps (the skewed one: 50) replay forward + bias
    # update from the starting bias and record each step's max/mean load
    trace = None
    if w.steps > 1:
        bias.copy_(torch.from_numpy(bias0).to(dev))
        ratios = []
        for _ in range(w.steps):
            step()
            c = layer.counts.cpu().numpy().astype(np.float64)
            ratios.append(float(c.max() / c.mean()))
        trace = {"steps": w.steps, "gamma": w.gamma, "load_max_over_mean": ratios,
                 "bias_abs_max": float(bias.abs().max().item())}
    barrier()
    # ------------------------------------------------ balance statistics (not part of the step)
    seq_len = args.seq_len or w.T
    bal_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    layer.balance_stats(seq_len, 1e-4)
    bal_ev[0].record(stream)
    for _ in range(20):
        layer.balance_stats(seq_len, 1e-4)
    bal_ev[1].record(stream)
    barrier()
    clk = clocks.stop() if clocks else None
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world, dev) / args.steps
    bal_ms = bal_ev[0].elapsed_time(bal_ev[1]) / 20
    # ------------------------------------------------ backward (not part of the step)
    bwd = None
    if args.backward and world == 1:
        gdy = torch.randn((w.T, w.H), device=dev).mul_(0.05).to(torch.bfloat16)
        step()
        layer.backward(gdy)             # set-up: transposed weights, workspace
        layer.backward(gdy, x=x)
        out = {}
        for name, kw in [("dgrad", {}), ("dgrad_wgrad", {"x": x})]:
            b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            ms = 0.0
            for _ in range(reps):
                step()                  # the backward needs its own forward's state
                b0.record(stream)
                layer.backward(gdy, **kw)
                b1.record(stream)
                b1.synchronize()
                ms += b0.elapsed_time(b1)
            out[name] = ms / reps
        if layer.status() != 0:
            raise RuntimeError("device status error in the backward")
        rows = w.T * (w.K + 1)
        flops_d = 2.0 * rows * w.H * w.I * 2 + 2.0 * rows * w.H * w.I + 2.0 * rows * w.H * 2 * w.I
        flops_w = 2.0 * rows * w.H * w.I + 2.0 * rows * 2 * w.I * w.H
        bwd = {"dgrad_ms": out["dgrad"], "dgrad_wgrad_ms": out["dgrad_wgrad"],
               "dgrad_tflops": flops_d / (out["dgrad"] * 1e-3) / 1e12,
               "wgrad_ms": out["dgrad_wgrad"] - out["dgrad"],
               "wgrad_out_gb": (w.N + 1) * 3 * w.H * w.I * 4 / 1e9,
               "note": "moe_backward after a forward; Dgrad = recompute [G|U], dh, dX rows (3 FP8 "
                       "grouped GEMMs); Wgrad adds dW2 and dW13 in fp32 for all N+1 experts"}

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    fp8_meas = None
    if not args.no_fp8_peak:
        try:
            fp8_meas = measure_fp8_peak(torch, dev)
        except Exception:
            fp8_meas = None
    work = algorithmic_work(w, counts)
    dom = max(stage_ms, key=stage_ms.get)
    gemm_ms = stage_ms["expert_up"] + stage_ms["expert_down"]
    gemm_tflops = (work["expert_up"]["flops"] + work["expert_down"]["flops"]) / (gemm_ms * 1e-3) / 1e12
    hbm_peak = float(peaks["hbm_gbs"])
    # FP8 dense peak: the library FP8 GEMM measured here, else twice the
    # measured (or fallback) bf16 burst (the nominal FP8 : BF16 ratio)
    fp8_peak = fp8_meas if fp8_meas else 2.0 * float(peaks["bf16_tflops"])
    fp8_peak_source = ("measured: library FP8 GEMM 8192^3 (torch._scaled_mm)" if fp8_meas else
                       f"2 x {peak_kind} bf16_tflops (nominal FP8:BF16 ratio)")
    roofline = roofline_of(work[dom], stage_ms[dom], hbm_peak, fp8_peak)
    roofline.update({"kernel": dom, "traffic": recorded_traffic(dom, w.name),
                     "traffic_source": TRAFFIC_FILE,
                     "peak_source": (f"{peak_kind} hbm_gbs (copy)" if roofline["bound"] == "hbm"
                                     else fp8_peak_source),
                     "algorithmic_bytes": work[dom]["bytes"], "algorithmic_flops": work[dom]["flops"]})
    value = w.T * world / (ms_step * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
        "data": "synthetic",
        "config": run_config(args, w, world),
        "gemm": {"tflops": gemm_tflops, "fp8_spec_tflops": FP8_SPEC_TFLOPS,
                 "frac_of_fp8_spec": gemm_tflops / FP8_SPEC_TFLOPS,
                 "fp8_library_tflops_measured": fp8_meas,
                 "frac_of_fp8_measured": (gemm_tflops / fp8_meas) if fp8_meas else None},
        "stages_ms": stage_ms,
        "roofline": roofline,
        "gpu_launches": launches_per_step * args.steps,
        "e2e": {"value": w.T * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 2,
                "copies": "pinned host buffers; upload and download on side streams, "
                          "double-buffered, overlapping the neighbouring steps' kernels"},
        "clocks": clk,
        "controller": trace,
        "backward": bwd,
        "graph": graph,
        "balance_stats": {"ms": bal_ms, "seq_len": seq_len,
                          "note": "moe_balance_stats after the step, not part of it"},
    }
    if world == 1 and not args.no_cpu_baseline:
        x32, gw, b0, ew = oracle_setup(w, x_bits)
        nl = (args.groups, args.topk_groups)
        oracle_sample_step(w, x32, gw, b0, ew, 0, node_limit=nl)      # warm-up, untimed
        t = [oracle_sample_step(w, x32, gw, b0, ew, 1 + s, node_limit=nl) for s in range(3)]
        v = w.T / float(np.mean(t))
        line["cpu_baseline"] = {
            "value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": "after 1 untimed step, " + oracle_sample_text(w, 3)}
    print(json.dumps(line), flush=True)


def run_ep(args, w, rank, world, local_rank):
    """One expert-parallel step per iteration: every rank routes its own T
    tokens, holds N/world routed experts and the shared expert, and exchanges
    rows with the others over NCCL (ep.ExpertParallelMoE); then the
    batch-level bias update. Weak scaling over ranks."""
    import socket

    import torch
    import torch.distributed as dist

    from __graft_entry__ import build
    build()
    from mixture_experts_layer_40_b200 import capi, ep
    from mixture_experts_layer_40_b200 import inputs as I
    from mixture_experts_layer_40_b200.layer import device_weights

    own_group = False
    if not dist.is_initialized():   # one rank without torchrun: a one-rank NCCL group
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, device_id=torch.device("cuda", local_rank))
        own_group = True
    try:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        pool = I.make_weight_pool(w)
        gate_w = I.make_gate_w(w)
        full = device_weights(w, pool, gate_w, dev)
        del pool
        local = ep.local_weights(full.w13, full.s13, full.w2, full.s2, w.N, world, rank)
        gw = full.gate_w
        del full
        torch.cuda.empty_cache()
        layer = ep.ExpertParallelMoE(w.T, w.H, w.N, w.K, w.I, world, rank, gw, *local,
                                     groups=args.groups, topk_groups=args.topk_groups,
                                     peer=args.peer)
        x_bits = I.make_x(rank_batch(w, rank))
        x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        x = x_host.to(dev)
        y_host = torch.empty((w.T, w.H), dtype=torch.bfloat16).pin_memory()
        bias = torch.from_numpy(I.make_bias(w)).to(dev)
        stream = torch.cuda.current_stream()

        def step(x_in):
            y = layer.forward(x_in, bias)
            total = layer.batch_counts()
            capi.moe_update_bias(bias, total, w.N, w.T * world, w.K, w.gamma)
            return y

        def barrier():
            dist.barrier()
            torch.cuda.synchronize()

        for _ in range(args.warmup):
            step(x)
        barrier()
        if layer.status() != 0:
            raise RuntimeError("device status error during warm-up")
        clocks = ClockSampler(local_rank) if rank == 0 else None
        if clocks:
            clocks.start()
        barrier()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(x)
        t1.record(stream)
        barrier()
        ms_step = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps
        if layer.status() != 0:
            raise RuntimeError("device status error in the timed region")
        # end to end: each step uploads x from pinned memory and downloads y,
        # on their own streams with two buffers each way, so step i+1's upload
        # and step i-1's download overlap step i's kernels (as in run_layer)
        up_s, down_s = torch.cuda.Stream(), torch.cuda.Stream()
        xs = [x, torch.empty_like(x)]
        y_hosts = [y_host, torch.empty_like(y_host).pin_memory()]
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i % 2
            up_s.wait_event(ev_done[b])          # step i-2 no longer reads xs[b]
            with torch.cuda.stream(up_s):
                xs[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(up_s)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])         # y_hosts[b] of step i-2 is written
            y = step(xs[b])
            ev_done[b].record(stream)
            down_s.wait_event(ev_done[b])
            y.record_stream(down_s)
            with torch.cuda.stream(down_s):
                y_hosts[b].copy_(y, non_blocking=True)
            ev_out[b].record(down_s)

        for i in range(2):
            e2e_step(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        e0.record(stream)
        up_s.wait_event(e0)
        for i in range(args.steps):
            e2e_step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        e1.record(stream)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
        clk = clocks.stop() if clocks else None
        rb = layer.row_bytes
        sc = layer.send_counts.cpu()
        send = int(sc[:, 0].sum())
        if rank == 0:
            line = {
                "metric": METRIC, "value": w.T * world / (ms_step * 1e-3), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
                "config": dict(run_config(args, w, world),
                               parallelism=f"ep{world} (routed experts sharded over ranks; own "
                                           f"batch per GPU)"),
                "gpu_launches": ep_step_launches(w.T, w.N, w.K, args.groups, args.topk_groups,
                                                 w.H) * args.steps,
                "e2e": {"value": w.T * world / (e2e_ms * 1e-3), "unit": "tokens/s",
                        "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 2,
                        "copies": "pinned host buffers, on two copy streams overlapping the "
                                  "neighbouring steps' kernels"},
                "clocks": clk,
                "ep": {"ranks": world, "experts_per_rank": w.N // world,
                       "mode": "peer" if args.peer else "all-to-all",
                       "send_rows_rank0": sc[:, 0].tolist(),
                       "dispatch_bytes_rank0": send * rb, "return_bytes_rank0": send * w.H * 4,
                       "host_syncs_per_step": 0 if args.peer else 1,
                       "note": ("library kernels: dispatch (router, plan, pack) storing rows "
                                "into the ranks' receive buffers, shared expert, local experts "
                                "storing partial sums into the sources' return buffers, "
                                "combine, bias update; two all-reduce barriers and the count "
                                "all-reduce" if args.peer else
                                "library kernels: dispatch (router, plan, pack), shared expert, "
                                "local experts, combine, bias update; exchanges: NCCL "
                                "all-to-all of counts, rows and partial sums, all-reduce of "
                                "counts")},
            }
            print(json.dumps(line), flush=True)
    finally:
        if own_group:
            dist.destroy_process_group()


def launch_ranks(n: int) -> None:
    """Re-runs this command as n ranks under torchrun (one process per GPU,
    rendezvous on 127.0.0.1), bounded by an outer timeout well above the
    process group's own; called when --gpus n > 1 and no rank environment
    is set. Does not return."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    sys.stdout.flush()
    os.execvp(cmd[0], cmd)


def launch_check(world: int, rank: int) -> None:
    """--launch-check: the rank plumbing alone (no kernels): every rank joins
    the process group (gloo without a GPU), the ranks sum one int and take
    the max of their times as the bench does, and rank 0 prints n_gpus."""
    import datetime

    import torch
    import torch.distributed as dist
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if world > 1:
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        one = torch.ones(1, dtype=torch.int64)
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
            one = one.cuda()
        ranks = int(batch_counts(one, world).item())
        t = torch.tensor([float(rank)], dtype=torch.float64, device=one.device)
        if world > 1:
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
        if rank == 0:
            print(json.dumps({"launch_check": True, "n_gpus": world, "ranks_counted": ranks,
                              "max_rank": float(t.item()), "backend": backend}), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


def main():
    args = parse()
    from mixture_experts_layer_40_b200 import inputs as I
    w = I.WORKLOADS[args.workload]
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "ours":
        launch_ranks(args.gpus)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if args.launch_check:
        launch_check(world, rank)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.ep:
            run_ep(args, w, rank, world, local_rank)
        else:
            run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
