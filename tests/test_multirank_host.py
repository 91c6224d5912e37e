"""The multi-rank host logic of bench.py on CPU (gloo, world size 2): every
rank routes its own batch, the per-expert counts are summed across ranks
before the bias update (the controller balances the whole batch, "DeepSeek-V3:
Auxiliary-Loss-Free MoE Load Balancing...", section III), and a multi-rank
time is the slowest rank's. Routing here is the oracle's; the GPU arm runs
the same helpers over NCCL."""
import json
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from oracle import moe_oracle as O
    from mixture_experts_layer_40_b200 import inputs as I
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        w = I.WORKLOADS["tiny"]
        wr = bench.rank_batch(w, rank)
        x = I.bf16_bits_to_f32(I.make_x(wr))
        ids, *_ = O.route(x, I.make_gate_w(w), I.make_bias(w), w.K)
        counts = torch.from_numpy(O.expert_counts(ids, w.N))
        summed = bench.batch_counts(counts.clone(), world)
        new_bias = O.update_bias(I.make_bias(w), summed.numpy(), w.T * world, w.K, w.gamma)
        slowest = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as fh:
            json.dump({"summed": summed.tolist(), "bias": new_bias.tolist(), "slowest": slowest},
                      fh)
    finally:
        dist.destroy_process_group()


def test_two_ranks_balance_the_whole_batch(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    from oracle import moe_oracle as O
    from mixture_experts_layer_40_b200 import inputs as I
    import bench
    w = I.WORKLOADS["tiny"]
    # the oracle on the two ranks' batches concatenated
    x = np.concatenate([I.bf16_bits_to_f32(I.make_x(bench.rank_batch(w, r))) for r in range(world)])
    ids, *_ = O.route(x, I.make_gate_w(w), I.make_bias(w), w.K)
    counts = O.expert_counts(ids, w.N)
    bias = O.update_bias(I.make_bias(w), counts, w.T * world, w.K, w.gamma)
    for r in range(world):
        assert res[r]["summed"] == counts.tolist()
        assert np.array_equal(np.array(res[r]["bias"], np.float32), bias)
        assert res[r]["slowest"] == 2.5
    assert counts.sum() == world * w.T * w.K
