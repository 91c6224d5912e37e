// moe_route_noalloc: the routing entry point for callers that cannot give the
// library a workspace.
//
// moe_route needs caller-provided scratch (the T x N gate logits live in the
// workspace). Some callers have no way to provide it: a host application that
// owns every device allocation through its own pool and does not let plug-in
// libraries allocate, or a latency-critical loop in which a cudaMalloc (which
// may synchronise the whole device) is not acceptable. This variant keeps its
// scratch in a fixed array in the library's own device memory instead, so the
// caller passes only the inputs and outputs and nothing is allocated.
//
// The logits come from the fp32 SIMT kernel (launch_router), not from the
// split-bf16 tensor-core kernel of moe_route: the top-K, gates and counts are
// moe_route's up to near ties of the K-th score and fp32 logit rounding.
//
// The array exists once per GPU that loads the library and stays resident
// until the process exits. Every call shares it: two calls whose kernels
// overlap on the GPU (different streams, or different host threads on one
// device) race on it and must be serialised by the caller. The logits are
// fully rewritten by each call, so no part of the array needs clearing; the
// counts output is zeroed by the call itself.
#include "kernels.cuh"

namespace moe {
namespace {

// Scratch for the gate logits: T * N floats at most (4 MiB).
__device__ __align__(256) float g_route_scratch[MOE_ROUTE_NOALLOC_MAX_LOGITS];

// Device address of g_route_scratch on the current device. Host code cannot
// use the array's name as a device pointer (it names a host-side stand-in),
// so the address is looked up, with the device current, on every call: the
// lookup is cheap, and an address cached across calls would go stale if the
// device's context were reset.
float* scratch_on_current_device() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
  return static_cast<float*>(p);
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_noalloc(moe_shape sh, const float* gate_w, const void* x,
                                 const float* bias, int32_t* topk_ids, float* topk_gates,
                                 int32_t* counts, void* stream) {
  using namespace moe;
  if (!shape_ok(sh)) return MOE_ERR_SHAPE;
  if ((int64_t)sh.T * sh.N > (int64_t)MOE_ROUTE_NOALLOC_MAX_LOGITS) return MOE_ERR_WORKSPACE;
  if (sh.T == 0) {  // an empty batch: only the counts are cleared
    if (!counts) return MOE_ERR_NULL;
    return cudaMemsetAsync(counts, 0, (size_t)sh.N * sizeof(int32_t),
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  }
  if (!gate_w || !x || !bias || !topk_ids || !topk_gates || !counts) return MOE_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(x) % 16) != 0 || (reinterpret_cast<uintptr_t>(gate_w) % 16) != 0)
    return MOE_ERR_ALIGN;
  float* scratch = scratch_on_current_device();
  if (scratch == nullptr) return MOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)sh.N * sizeof(int32_t), s);
  if (e == cudaSuccess)
    e = launch_router(x, gate_w, bias, sh.T, sh.H, sh.N, sh.K, sh.G, sh.M, scratch, topk_ids,
                      topk_gates, counts, nullptr, s, moe_device_sm_count());
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
