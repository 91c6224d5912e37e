"""Host-side checks of bench.py (no GPU): the reference arm's JSON line on the
tiny workload, the algorithmic byte counts the roofline divides by, and the
rule that a recorded DRAM capture is reported only for the GEMM sources it
measured."""
import json
import os
import subprocess
import sys

import numpy as np

import bench
from mixture_experts_layer_40_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3", *extra],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_reference_arm_line():
    d = _run()
    for key in ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"]:
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_node_limited():
    d = _run("--groups", "4", "--topk-groups", "2")
    assert d["value"] > 0


def test_algorithmic_bytes_by_hand():
    w = I.WORKLOADS["v3_prefill"]
    work = bench.algorithmic_work(w, np.ones(256))
    # up: 257 experts x (2 I H codes + 2 (I/128)(H/128) fp32 scales), plus
    # 36864 rows x (H codes + H/128 scales) in and x (I codes + I/128 scales) out
    up = 257 * (2 * 2048 * 7168 + 2 * 16 * 56 * 4) + 36864 * (7168 + 56 * 4) + 36864 * (2048 + 16 * 4)
    assert work["expert_up"]["bytes"] == up
    assert work["expert_up"]["flops"] == 2.0 * 36864 * 7168 * 4096
    # down: weights, h rows in, bf16 rows out (2 bytes x H)
    down = 257 * (7168 * 2048 + 56 * 16 * 4) + 36864 * (2048 + 16 * 4) + 36864 * 7168 * 2
    assert work["expert_down"]["bytes"] == down


def test_recorded_traffic_follows_the_sources(tmp_path, monkeypatch):
    fp = bench.gemm_fingerprint()
    assert len(fp) == 16
    note = tmp_path / "t.md"
    note.write_text(f"traffic expert_up bytes=123 workload=v3_prefill fingerprint={fp}\n"
                    f"traffic expert_down bytes=456 workload=v3_prefill fingerprint=0000000000000000\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(note))
    assert bench.recorded_traffic("expert_up", "v3_prefill") == 123
    assert bench.recorded_traffic("expert_up", "decode") is None
    assert bench.recorded_traffic("expert_down", "v3_prefill") is None   # stale capture


def test_gpus_flag_starts_the_ranks():
    """bench.py --gpus 2 without a rank environment starts two ranks itself
    (torchrun on 127.0.0.1); they meet in a process group (gloo here, no GPU)
    and rank 0 reports n_gpus = 2."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--launch-check"], capture_output=True, text=True, timeout=300,
                         cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["ranks_counted"] == 2 and d["max_rank"] == 1.0


def test_cpu_baseline_builds_the_pools_before_timing():
    """The oracle's dequantised block pool is built in the set-up, so no
    timed sample step pays for it."""
    w = I.WORKLOADS["tiny"]
    _, _, _, ew = bench.oracle_setup(w, I.make_x(w))
    assert getattr(ew, "_deq", None) is not None


def test_roofline_bound_follows_the_ridge():
    """An HBM-bound launch (V3 prefill's up GEMM: about 300 FLOP per byte,
    below the ridge of 3160 TFLOP/s over 6650 GB/s) is reported in GB/s; a
    compute-bound one (the same GEMM at T = 32768, about 1900 FLOP per byte)
    in TFLOP/s against the FP8 peak."""
    up = bench.algorithmic_work(I.WORKLOADS["v3_prefill"], np.ones(256))["expert_up"]
    r = bench.roofline_of(up, 1.0, 6650.0, 3160.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["achieved"] - up["bytes"] / 1e-3 / 1e9) < 1e-6 * r["achieved"]
    big = bench.algorithmic_work(I.WORKLOADS["large_prefill"], np.ones(256))["expert_up"]
    r = bench.roofline_of(big, 10.0, 6650.0, 3160.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - big["flops"] / 1e-2 / 1e12 / 3160.0) < 1e-9


def test_launch_count_follows_the_router_path():
    """The `gpu_launches` claim: per step the router's kernels (1 with the
    selection in the wide tiles' epilogue, 3 with a split reduction, 2
    otherwise), the permutation's 3, and quantise, up, down, combine, bias
    update. The counts match the launch lists of V3 prefill (11 kernels) and
    large prefill (9) in profiles/."""
    assert bench.step_launches(4096, 256, 8, 0, 0, 7168) == 11   # split logits
    assert bench.step_launches(32768, 256, 8, 0, 0, 7168) == 9   # fused selection
    assert bench.step_launches(32768, 256, 8, 8, 4, 7168) == 9   # node-limited, 8 groups
    assert bench.step_launches(32768, 256, 16, 0, 0, 7168) == 10  # K > 8: logits + top-K
    assert bench.step_launches(512, 32, 8, 0, 0, 7168) == 10     # N = 32: 128 x 64 tiles
    assert bench.step_launches(128, 256, 8, 0, 0, 7168) == 11
    # an expert-parallel step at V3 prefill: 18 kernels, as in its launch list
    assert bench.ep_step_launches(4096, 256, 8, 0, 0, 7168) == 18
