// Router: s = sigmoid(x . e_i), top-K of s + b, unbiased normalised gates,
// per-expert counts. "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
// Multi-Token Prediction, and FP8 Training at 671B Scale" (trishampatil.com),
// section III, "The mechanism": the bias enters only the TopK comparison and
// the gate is the unbiased affinity normalised over the K chosen. Gating stays
// in fp32 ("DeepSeek-V3, explained", recipe step 7), so the logits come from an
// fp32 FMA GEMM of the bf16 input and the fp32 centroids.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kLT = 64;    // tokens per CTA tile
constexpr int kLE = 64;    // experts per CTA tile
constexpr int kLK = 32;    // reduction chunk
constexpr int kLPad = kLT + 4;

// z[t, e] = sum_h x[t, h] * g[e, h], fp32 accumulation. 256 threads, each a
// 4x4 block of (token, expert) outputs; both operands staged k-major in
// shared memory.
__global__ void __launch_bounds__(256) logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                     const float* __restrict__ gw, int T, int H,
                                                     int N, float* __restrict__ z) {
  __shared__ __align__(16) float xs[kLK][kLPad];
  __shared__ __align__(16) float ws[kLK][kLPad];
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * kLT, e0 = blockIdx.y * kLE;
  const int ty = tid >> 4, tx = tid & 15;
  float acc[4][4] = {};
  // loader coordinates: x -> one token, 8 consecutive k; w -> one expert, 4 k
  const int xl_t = tid >> 2, xl_k = (tid & 3) * 8;
  for (int k0 = 0; k0 < H; k0 += kLK) {
    {
      const int t = t0 + xl_t;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (t < T) v = __ldg(reinterpret_cast<const uint4*>(x + (int64_t)t * H + k0 + xl_k));
      const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                          bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
      for (int j = 0; j < 8; ++j) xs[xl_k + j][xl_t] = f[j];
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int f = tid + 256 * i;
      const int e = f >> 3, k4 = (f & 7) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e0 + e < N) v = __ldg(reinterpret_cast<const float4*>(gw + (int64_t)(e0 + e) * H + k0 + k4));
      ws[k4 + 0][e] = v.x;
      ws[k4 + 1][e] = v.y;
      ws[k4 + 2][e] = v.z;
      ws[k4 + 3][e] = v.w;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < kLK; ++k) {
      const float4 a = *reinterpret_cast<const float4*>(&xs[k][ty * 4]);
      const float4 b = *reinterpret_cast<const float4*>(&ws[k][tx * 4]);
      const float av[4] = {a.x, a.y, a.z, a.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < N) z[(int64_t)t * N + e] = acc[i][j];
    }
  }
}

constexpr int kMaxPerLane = 32;  // N <= 1024

// One warp per token: sigmoid, biased scores, K rounds of a warp arg-max
// (highest score, lower id on ties), gates from the unbiased affinities,
// counts by integer atomics (exact, order-independent).
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ z,
                                                   const float* __restrict__ bias, int T, int N,
                                                   int K, int32_t* __restrict__ ids,
                                                   float* __restrict__ gates,
                                                   int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int per_lane = (N + 31) >> 5;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    float sc[kMaxPerLane], sv[kMaxPerLane];
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
      sc[j] = -INFINITY;
      sv[j] = 0.0f;
      const int e = lane + 32 * j;
      if (j < per_lane && e < N) {
        const float s = 1.0f / (1.0f + expf(-z[(int64_t)t * N + e]));
        const float v = s + bias[e];
        sv[j] = s;
        sc[j] = (v == v) ? v : -INFINITY;
      }
    }
    uint32_t taken = 0;
    int my_id = 0;
    float my_s = 0.0f, sum = 0.0f;
    for (int k = 0; k < K; ++k) {
      float best = -INFINITY, best_s = 0.0f;
      int bid = N, bj = -1;
#pragma unroll
      for (int j = 0; j < kMaxPerLane; ++j) {
        const int e = lane + 32 * j;
        if (j < per_lane && e < N && !((taken >> j) & 1u) && (sc[j] > best || (sc[j] == best && e < bid))) {
          best = sc[j];
          bid = e;
          best_s = sv[j];
          bj = j;
        }
      }
      const int owner_bid = bid;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bid, o);
        const float os = __shfl_xor_sync(0xffffffffu, best_s, o);
        if (ob > best || (ob == best && oi < bid)) {
          best = ob;
          bid = oi;
          best_s = os;
        }
      }
      if (bid == owner_bid && bj >= 0) taken |= 1u << bj;
      sum += best_s;
      if (lane == k) {
        my_id = bid;
        my_s = best_s;
      }
    }
    if (lane < K) {
      ids[(int64_t)t * K + lane] = my_id;
      gates[(int64_t)t * K + lane] = my_s / sum;
      atomicAdd(&counts[my_id], 1);
    }
  }
}

}  // namespace

cudaError_t launch_router(const void* x, const float* gate_w, const float* bias, int T, int H,
                          int N, int K, float* logits, int32_t* ids, float* gates, int32_t* counts,
                          uint32_t* status, cudaStream_t stream, int sm_count) {
  (void)status;
  if (T == 0) return cudaSuccess;
  dim3 g1((T + kLT - 1) / kLT, (N + kLE - 1) / kLE);
  logits_kernel<<<g1, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(x), gate_w, T, H, N,
                                        logits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int blocks = (T + 7) / 8;
  if (blocks > sm_count * 8) blocks = sm_count * 8;
  topk_kernel<<<blocks, 256, 0, stream>>>(logits, bias, T, N, K, ids, gates, counts);
  return cudaGetLastError();
}

}  // namespace moe
