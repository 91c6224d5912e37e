// Token permutation by expert. Every (token, slot) pair is kept ("no tokens
// are dropped in training or at inference": "DeepSeek-V3, explained", recipe
// step 5) and placed expert-major, tokens ascending inside each expert, so the
// order is unique and the scatter needs no atomics on output positions.
//   scan    : counts -> offsets, GEMM group rows and 128-aligned row starts
//   scatter : one CTA per expert compacts the tokens that chose it, in token
//             order, with a block-wide prefix sum over ballots, and records
//             each (token, slot)'s GEMM row; the activation quantiser then
//             writes every token's codes straight into its rows
#include "block_scan.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

// One CTA of 1024 threads; N <= 1024. `pairs` is the number of (token, slot)
// pairs the counts must add up to (negative: not checked).
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ counts, int N,
                                                    int T, int64_t pairs, int64_t routed_cap,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ group_rows,
                                                    int32_t* __restrict__ row_start,
                                                    uint32_t* __restrict__ status) {
  __shared__ int sums[33];
  const int e = threadIdx.x;
  const int c = e < N ? counts[e] : 0;
  const int padded = (c + kTile - 1) / kTile * kTile;
  int total_c, total_p;
  const int off = block_scan_int(c, sums, &total_c);
  const int start = block_scan_int(padded, sums, &total_p);
  if (e < N) {
    offsets[e] = off;
    group_rows[e] = c;
    row_start[e] = start;
  }
  if (e == 0) {
    offsets[N] = total_c;
    group_rows[N] = T;
    row_start[N] = (int32_t)routed_cap;
    if ((pairs >= 0 && (int64_t)total_c != pairs) || (int64_t)total_p > routed_cap) {
      flag_status(status, kStatusBounds);
    }
  }
}

// One CTA (1024 threads) per routed expert e: walks the tokens in order and
// writes the GEMM rows of the pairs (t, k) with ids[t, k] == e.
__global__ void __launch_bounds__(1024) scatter_kernel(const int32_t* __restrict__ ids, int T, int K,
                                                       const int32_t* __restrict__ group_rows,
                                                       const int32_t* __restrict__ row_start,
                                                       int64_t routed_cap,
                                                       int32_t* __restrict__ row_token,
                                                       int32_t* __restrict__ token_row,
                                                       uint32_t* __restrict__ status) {
  __shared__ int sums[33];
  const int e = blockIdx.x;
  const int base = row_start[e];
  const int count = group_rows[e];
  int running = 0;
  for (int t0 = 0; t0 < T; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    int slot = -1;
    if (t < T) {
      for (int k = 0; k < K; ++k)
        if (__ldg(ids + (int64_t)t * K + k) == e) slot = k;
    }
    int total;
    const int pos = block_scan_flag(slot >= 0, sums, &total);
    if (slot >= 0) {
      const int64_t r = (int64_t)base + running + pos;
      if (running + pos < count && r < routed_cap) {
        row_token[r] = t;
        token_row[(int64_t)t * K + slot] = (int32_t)r;
      } else {
        flag_status(status, kStatusBounds);
      }
    }
    running += total;
  }
  if (threadIdx.x == 0 && running != count) flag_status(status, kStatusBounds);
}

}  // namespace

cudaError_t launch_permute(const int32_t* ids, const int32_t* counts, int T, int N, int K,
                           int64_t pairs, int64_t routed_cap, int32_t* offsets, int32_t* group_rows,
                           int32_t* row_start, int32_t* row_token, int32_t* token_row,
                           uint32_t* status, cudaStream_t stream) {
  scan_kernel<<<1, 1024, 0, stream>>>(counts, N, T, pairs, routed_cap, offsets, group_rows,
                                      row_start, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(row_token, 0xFF, (size_t)routed_cap * sizeof(int32_t), stream);
  if (e != cudaSuccess) return e;
  scatter_kernel<<<N, 1024, 0, stream>>>(ids, T, K, group_rows, row_start, routed_cap, row_token,
                                         token_row, status);
  return cudaGetLastError();
}

}  // namespace moe
