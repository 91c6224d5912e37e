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

// 8 consecutive row elements as fp32
MOE_DEV void load8(const __nv_bfloat16* p, int64_t c, float (&v)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p) + c);
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
MOE_DEV void load8(const float* p, int64_t c, float (&v)[8]) {
  const float4 a = __ldcs(reinterpret_cast<const float4*>(p) + 2 * c);
  const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 2 * c + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename Row>
__global__ void __launch_bounds__(128) combine_kernel(const Row* __restrict__ y_rows,
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
  // slot k (thread k) goes to position = the number of its token's slots with
  // a lower expert id (the K experts of a token are distinct); slots whose
  // row is out of range are dropped and flagged
  if (threadIdx.x < K) {
    const int k = threadIdx.x;
    const int e = ids[(int64_t)t * K + k];
    const int64_t r = token_row[(int64_t)t * K + k];
    const float g = gates != nullptr ? gates[(int64_t)t * K + k] : 1.0f;
    const bool ok = r >= 0 && r < routed_cap;
    if (!ok) flag_status(status, kStatusBounds);
    const unsigned mask = (1u << K) - 1u;
    int pos = 0;
    for (int j = 0; j < K; ++j) {
      const int ej = __shfl_sync(mask, e, j);
      const bool okj = __shfl_sync(mask, ok, j);
      pos += (okj && ej < e) ? 1 : 0;
    }
    const int n_ok = __popc(__ballot_sync(mask, ok));
    if (ok) {
      s_row[pos] = r;
      s_gate[pos] = g;
    }
    if (k == 0) s_n = n_ok;
  }
  __syncthreads();
  const int n = s_n;
  const int64_t shared_row = routed_cap + t;
  if (shared_row >= rows_total) return;
  const Row* ys = y_rows + shared_row * H;
  uint4* out = reinterpret_cast<uint4*>(y + (int64_t)t * H);
  int64_t rows[kMaxK];
  float gk[kMaxK];
#pragma unroll
  for (int k = 0; k < kMaxK; ++k) {
    rows[k] = k < n ? s_row[k] * H : 0;
    gk[k] = k < n ? s_gate[k] : 0.0f;
  }
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float acc[8];
    load8(ys, c, acc);
    if (n == 8) {
      // the common case: all eight rows' loads in flight before the adds
      float f[8][8];
#pragma unroll
      for (int k = 0; k < 8; ++k) load8(y_rows + rows[k], c, f[k]);
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(gk[k], f[k][i], acc[i]);
    } else {
      for (int k = 0; k < n; ++k) {
        float f[8];
        load8(y_rows + s_row[k] * H, c, f);
        const float g = s_gate[k];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(g, f[i], acc[i]);
      }
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

template <typename Row>
cudaError_t combine(const Row* y_rows, const int32_t* ids, const float* gates,
                    const int32_t* token_row, int T, int H, int K, int64_t routed_cap,
                    int64_t rows_total, __nv_bfloat16* y, uint32_t* status, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  combine_kernel<Row><<<T, 128, 0, stream>>>(y_rows, ids, gates, token_row, T, H, K, routed_cap,
                                             rows_total, y, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y_rows, const int32_t* ids, const float* gates,
                           const int32_t* token_row, int T, int H, int K, int64_t routed_cap,
                           int64_t rows_total, __nv_bfloat16* y, uint32_t* status,
                           cudaStream_t stream) {
  return combine(y_rows, ids, gates, token_row, T, H, K, routed_cap, rows_total, y, status, stream);
}

cudaError_t launch_combine(const float* y_rows, const int32_t* ids, const float* gates,
                           const int32_t* token_row, int T, int H, int K, int64_t routed_cap,
                           int64_t rows_total, __nv_bfloat16* y, uint32_t* status,
                           cudaStream_t stream) {
  return combine(y_rows, ids, gates, token_row, T, H, K, routed_cap, rows_total, y, status, stream);
}

cudaError_t launch_update_bias(float* bias, const int32_t* counts, int N, int T, int K,
                               float gamma, cudaStream_t stream) {
  update_bias_kernel<<<(N + 255) / 256, 256, 0, stream>>>(bias, counts, N, (int64_t)T * K, gamma);
  return cudaGetLastError();
}

}  // namespace moe
