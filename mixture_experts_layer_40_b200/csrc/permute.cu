// Token permutation by expert. Every (token, slot) pair is kept ("no tokens
// are dropped in training or at inference": "DeepSeek-V3, explained", recipe
// step 5) and placed expert-major, tokens ascending inside each expert, so the
// order is unique and the placement needs no atomics on output positions.
//   rank  : per chunk of 128 tokens, the rank of each (token, slot) among the
//           chunk's earlier pairs with the same expert (per-warp lane masks of
//           each expert, then a scan over the chunk's four warps), and the
//           chunk's count of each expert
//   scan  : the per-chunk counts summed into each expert's count (written, or
//           checked against the router's), offsets, GEMM group rows and
//           128-aligned row starts, and for every (chunk, expert) the first
//           GEMM row of that chunk's pairs
//   place : row = chunk base + rank for every pair; records row_token and
//           token_row (the activation quantiser then writes every token's
//           codes straight into its rows)
// The work is linear in T*K, spread over T/128 CTAs.
#include "block_scan.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kChunk = 128;          // tokens per rank CTA, one per thread
constexpr int kChunkWarps = kChunk / 32;
constexpr int kMaxK = 16;

// One CTA per chunk of kChunk tokens. ranks[t, k] (in token_row) = the
// number of pairs (t', k') of this chunk with t' < t and ids[t', k'] ==
// ids[t, k]; hist[chunk, e] = the chunk's pairs with expert e. Slots with a
// negative id are skipped; an id >= N is a bounds error. Shared memory:
// 2 * kChunkWarps * N ints.
__global__ void __launch_bounds__(kChunk) rank_kernel(const int32_t* __restrict__ ids, int T,
                                                      int N, int K, int32_t* __restrict__ ranks,
                                                      int32_t* __restrict__ hist,
                                                      uint32_t* __restrict__ status) {
  extern __shared__ uint32_t perm_smem[];
  uint32_t* mask = perm_smem;                                          // [warps][N]
  int* base = reinterpret_cast<int*>(perm_smem + kChunkWarps * N);     // [warps][N]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kChunkWarps * N; i += blockDim.x) mask[i] = 0u;
  __syncthreads();
  const int64_t t = (int64_t)blockIdx.x * kChunk + threadIdx.x;
  int e[kMaxK];
#pragma unroll
  for (int k = 0; k < kMaxK; ++k) {
    e[k] = -1;
    if (k < K && t < T) {
      const int v = ids[t * K + k];
      if (v >= N) flag_status(status, kStatusBounds);
      e[k] = v < N ? v : -1;
    }
  }
  // lanes that chose each expert (a token's K experts are distinct)
#pragma unroll
  for (int k = 0; k < kMaxK; ++k)
    if (e[k] >= 0) atomicOr(&mask[warp * N + e[k]], 1u << lane);
  __syncthreads();
  // per expert: the pairs of earlier warps, and the chunk total
  for (int x = threadIdx.x; x < N; x += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kChunkWarps; ++w) {
      base[w * N + x] = run;
      run += __popc(mask[w * N + x]);
    }
    hist[(int64_t)blockIdx.x * N + x] = run;
  }
  __syncthreads();
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < kMaxK; ++k)
    if (e[k] >= 0)
      ranks[t * K + k] = base[warp * N + e[k]] + __popc(mask[warp * N + e[k]] & below);
}

// One CTA of 1024 threads; N <= 1024. Each expert's count is the sum of its
// per-chunk counts; with count_out the counts are written from them, else
// they are read from `counts` and checked against them. Then the group
// tables, and for every chunk c: hist[c, e] <- row_start[e] + the pairs of e
// in chunks before c. `pairs` is the number of (token, slot) pairs the counts
// must add up to (negative: not checked). Eight chunks' counts are fetched
// before any is used, so the loads overlap.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ counts, bool count_out,
                                                    int N, int T, int64_t pairs,
                                                    int64_t routed_cap, int n_chunks,
                                                    int32_t* __restrict__ hist,
                                                    int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ group_rows,
                                                    int32_t* __restrict__ row_start,
                                                    uint32_t* __restrict__ status) {
  __shared__ int sums[33];
  const int e = threadIdx.x;
  int c = 0;
  if (e < N) {
    for (int ch0 = 0; ch0 < n_chunks; ch0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = ch0 + j < n_chunks ? hist[(int64_t)(ch0 + j) * N + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) c += v[j];
    }
    if (count_out) {
      counts[e] = c;
    } else if (counts[e] != c) {
      flag_status(status, kStatusBounds);
    }
  }
  const int padded = (c + kTile - 1) / kTile * kTile;
  int total_c, total_p;
  const int off = block_scan_int(c, sums, &total_c);
  const int start = block_scan_int(padded, sums, &total_p);
  if (e < N) {
    offsets[e] = off;
    group_rows[e] = c;
    row_start[e] = start;
    int run = start;
    for (int ch0 = 0; ch0 < n_chunks; ch0 += 8) {
      int v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = ch0 + j < n_chunks ? hist[(int64_t)(ch0 + j) * N + e] : 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (ch0 + j < n_chunks) hist[(int64_t)(ch0 + j) * N + e] = run;
        run += v[j];
      }
    }
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

// One thread per (token, slot): its GEMM row is the chunk's base row for its
// expert plus its rank; rows outside the expert's segment are bounds errors.
__global__ void __launch_bounds__(256) place_kernel(const int32_t* __restrict__ ids, int64_t T,
                                                    int N, int K,
                                                    const int32_t* __restrict__ hist,
                                                    const int32_t* __restrict__ group_rows,
                                                    const int32_t* __restrict__ row_start,
                                                    int64_t routed_cap,
                                                    int32_t* __restrict__ row_token,
                                                    int32_t* __restrict__ token_row,
                                                    uint32_t* __restrict__ status) {
  const int64_t n = T * K;
  for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < n;
       p += (int64_t)gridDim.x * blockDim.x) {
    const int e = ids[p];
    if (e < 0 || e >= N) continue;
    const int64_t t = p / K;
    const int64_t r = (int64_t)hist[(t / kChunk) * N + e] + token_row[p];
    if (r < row_start[e] + (int64_t)group_rows[e] && r < routed_cap) {
      row_token[r] = (int32_t)t;
      token_row[p] = (int32_t)r;
    } else {
      flag_status(status, kStatusBounds);
    }
  }
}

}  // namespace

size_t permute_scratch_bytes(int64_t T, int N) {
  return (size_t)((T + kChunk - 1) / kChunk) * (size_t)N * 4;
}

cudaError_t launch_permute(const int32_t* ids, int32_t* counts, bool count_out, int T, int N,
                           int K, int64_t pairs, int64_t routed_cap, int32_t* hist,
                           int32_t* offsets, int32_t* group_rows, int32_t* row_start,
                           int32_t* row_token, int32_t* token_row, uint32_t* status,
                           cudaStream_t stream, int sm_count) {
  const int n_chunks = (T + kChunk - 1) / kChunk;
  // at most 2 * 4 * 1024 ints = 32 KB (N <= 1024): under the default limit
  const size_t smem = (size_t)2 * kChunkWarps * N * sizeof(int);
  cudaError_t e = cudaSuccess;
  if (n_chunks > 0) {
    rank_kernel<<<n_chunks, kChunk, smem, stream>>>(ids, T, N, K, token_row, hist, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  scan_kernel<<<1, 1024, 0, stream>>>(counts, count_out, N, T, pairs, routed_cap, n_chunks, hist,
                                      offsets, group_rows, row_start, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(row_token, 0xFF, (size_t)routed_cap * sizeof(int32_t), stream);
  if (e != cudaSuccess || n_chunks == 0) return e;
  const int64_t n = (int64_t)T * K;
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)sm_count * 16) blocks = (int64_t)sm_count * 16;
  place_kernel<<<(unsigned)blocks, 256, 0, stream>>>(ids, T, N, K, hist, group_rows, row_start,
                                                     routed_cap, row_token, token_row, status);
  return cudaGetLastError();
}

}  // namespace moe
