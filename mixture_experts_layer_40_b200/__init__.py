"""B200 (sm_100a) DeepSeekMoE layer forward: FP8 E4M3 grouped expert GEMMs on
tcgen05 tensor cores with aux-loss-free bias routing.

    from mixture_experts_layer_40_b200 import capi        # C ABI binding
    from mixture_experts_layer_40_b200.layer import MoELayer

The compute lives in libmoe_b200.so (hand-written CUDA for sm_100a, C ABI in
include/moe_capi.h); `capi` marshals torch tensors to it. Build the library
with `python -m mixture_experts_layer_40_b200.build`.
"""
