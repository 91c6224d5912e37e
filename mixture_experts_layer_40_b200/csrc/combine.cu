// Weighted combine with the shared expert, and the bias controller.
//
// Combine: y_t = FFN_shared(x_t) + sum_k g[t,k] FFN_{ids_k}(x_t) ("DeepSeek-V3,
// explained", the K_r note: normalised gates, shared expert at full weight).
// fp32 accumulation in a fixed order (shared first, then slots by ascending
// expert id) and one rounding to bf16, so the result does not depend on
// scheduling. A gather per token: no atomics.
//
// Bias update: "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing, ..."
// (trishampatil.com), section III "How the bias is set".
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kMaxK = 16;

__global__ void __launch_bounds__(128) combine_kernel(const float* __restrict__ y_rows,
                                                      const int32_t* __restrict__ ids,
                                                      const float* __restrict__ gates,
                                                      const int32_t* __restrict__ token_row,
                                                      int T, int H, int K, int64_t routed_cap,
                                                      int64_t rows_total,
                                                      __nv_bfloat16* __restrict__ y,
                                                      uint32_t* __restrict__ status) {
  __shared__ int64_t s_row[kMaxK];
  __shared__ float s_gate[kMaxK];
  __shared__ int s_n;
  const int t = blockIdx.x;
  if (threadIdx.x == 0) {
    int id[kMaxK];
    int n = 0;
    for (int k = 0; k < K; ++k) {
      const int e = ids[(int64_t)t * K + k];
      const int64_t r = token_row[(int64_t)t * K + k];
      const float g = gates != nullptr ? gates[(int64_t)t * K + k] : 1.0f;
      if (r < 0 || r >= routed_cap) {
        flag_status(status, kStatusBounds);
        continue;
      }
      // insertion by ascending expert id
      int j = n;
      while (j > 0 && id[j - 1] > e) {
        id[j] = id[j - 1];
        s_row[j] = s_row[j - 1];
        s_gate[j] = s_gate[j - 1];
        --j;
      }
      id[j] = e;
      s_row[j] = r;
      s_gate[j] = g;
      ++n;
    }
    s_n = n;
  }
  __syncthreads();
  const int n = s_n;
  const int64_t shared_row = routed_cap + t;
  if (shared_row >= rows_total) return;
  const float4* ys = reinterpret_cast<const float4*>(y_rows + shared_row * H);
  uint4* out = reinterpret_cast<uint4*>(y + (int64_t)t * H);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const float4 v0 = __ldcs(ys + 2 * c), v1 = __ldcs(ys + 2 * c + 1);
    float acc[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    for (int k = 0; k < n; ++k) {
      const float4* yk = reinterpret_cast<const float4*>(y_rows + s_row[k] * H);
      const float4 u0 = __ldcs(yk + 2 * c), u1 = __ldcs(yk + 2 * c + 1);
      const float g = s_gate[k];
      const float f[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, f[i], acc[i]);
    }
    uint4 o;
    o.x = pack_bf16x2(acc[0], acc[1]);
    o.y = pack_bf16x2(acc[2], acc[3]);
    o.z = pack_bf16x2(acc[4], acc[5]);
    o.w = pack_bf16x2(acc[6], acc[7]);
    out[c] = o;
  }
}

__global__ void update_bias_kernel(float* __restrict__ bias, const int32_t* __restrict__ counts,
                                   int N, int64_t TK, float gamma) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int64_t d = TK - (int64_t)N * counts[i];
  const float step = d > 0 ? gamma : (d < 0 ? -gamma : 0.0f);
  bias[i] = __fadd_rn(bias[i], step);
}

}  // namespace

cudaError_t launch_combine(const float* y_rows, const int32_t* ids, const float* gates,
                           const int32_t* token_row, int T, int H, int K, int64_t routed_cap,
                           int64_t rows_total, __nv_bfloat16* y, uint32_t* status,
                           cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  combine_kernel<<<T, 128, 0, stream>>>(y_rows, ids, gates, token_row, T, H, K, routed_cap,
                                        rows_total, y, status);
  return cudaGetLastError();
}

cudaError_t launch_update_bias(float* bias, const int32_t* counts, int N, int T, int K,
                               float gamma, cudaStream_t stream) {
  update_bias_kernel<<<(N + 255) / 256, 256, 0, stream>>>(bias, counts, N, (int64_t)T * K, gamma);
  return cudaGetLastError();
}

}  // namespace moe
