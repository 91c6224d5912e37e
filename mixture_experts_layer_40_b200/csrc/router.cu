// Router: s = sigmoid(x . e_i), top-K of s + b, unbiased normalised gates,
// per-expert counts. "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
// Multi-Token Prediction, and FP8 Training at 671B Scale" (trishampatil.com),
// section III, "The mechanism": the bias enters only the TopK comparison and
// the gate is the unbiased affinity normalised over the K chosen. Gating stays
// in fp32 ("DeepSeek-V3, explained", recipe step 7), so the logits are fp32
// sums of the bf16 input times the fp32 centroids: either an fp32 FMA GEMM
// (logits_kernel, the no-allocation route) or BF16 tensor-core MMAs against
// the centroids split exactly into three bf16 terms with fp32 accumulation
// (logits_tc_kernel, and logits_tc_wide_kernel whose 256 x 256 tiles either
// cover the whole depth, then at N = 256 also make the selection in their
// epilogue, or a slice of it that splitk_reduce_kernel sums).
#include <algorithm>

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

// The affinity s = sigmoid(z) and the biased selection score s + b (a NaN
// score ranks below every number). Every top-K path uses these two, so that
// equal logits give equal choices whichever kernel made them.
// The reciprocal is the hardware one (__fdividef: within 2 ulp, no branch,
// and 0 once exp(-z) overflows), so that the 32 affinities of a chunk can be
// scheduled together; the exact quotient's slow-path branch serialised them.
MOE_DEV float affinity(float z) { return __fdividef(1.0f, 1.0f + expf(-z)); }
MOE_DEV float biased_score(float s, float b) {
  const float v = s + b;
  return v == v ? v : -INFINITY;
}

// Warp arg-max of (score, id) pairs: the highest score, the lower id on ties.
MOE_DEV void warp_argmax(float& best, int& bid) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bid, o);
    if (ob > best || (ob == best && oi < bid)) {
      best = ob;
      bid = oi;
    }
  }
}

// One warp per token: sigmoid, biased scores, K rounds of a warp arg-max
// (highest score, lower id on ties), gates from the unbiased affinities,
// counts by integer atomics (exact, order-independent) unless counts is null
// (the layer forward takes them from the permutation's histograms instead:
// at T = 32768 the atomics on N counters cost about 0.1 ms).
// Node-limited routing (G > 1, "DeepSeek-V3, explained", recipe step 5):
// before the K rounds, each of the G contiguous expert groups is scored by
// the sum of its K/M highest biased scores (taken in descending order), the
// M best groups are kept (lower group id on ties) and every expert outside
// them is masked out of the selection.
// kPerLane: a compile-time bound on the scores each lane holds (N <= 32 *
// kPerLane), so that the per-lane arrays stay in registers.
template <int kPerLane>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ z,
                                                   const float* __restrict__ bias, int T, int N,
                                                   int K, int G, int M,
                                                   int32_t* __restrict__ ids,
                                                   float* __restrict__ gates,
                                                   int32_t* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int per_lane = (N + 31) >> 5;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    float sc[kPerLane], sv[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
      sc[j] = -INFINITY;
      sv[j] = 0.0f;
      const int e = lane + 32 * j;
      if (j < per_lane && e < N) {
        const float s = affinity(z[(int64_t)t * N + e]);
        sv[j] = s;
        sc[j] = biased_score(s, bias[e]);
      }
    }
    if (G > 1 && M < G) {
      const int size = N / G, per_group = K / M;
      float my_group_score = -INFINITY;  // lane g holds group g's score
      for (int g = 0; g < G; ++g) {
        uint32_t used = 0;
        float gsum = 0.0f;
        for (int r = 0; r < per_group; ++r) {
          float best = -INFINITY;
          int bid = N, bj = -1;
#pragma unroll
          for (int j = 0; j < kPerLane; ++j) {
            const int e = lane + 32 * j;
            if (j < per_lane && e < N && e / size == g && !((used >> j) & 1u) &&
                (sc[j] > best || (sc[j] == best && e < bid))) {
              best = sc[j];
              bid = e;
              bj = j;
            }
          }
          const int own = bid;
          warp_argmax(best, bid);
          if (bid == own && bj >= 0) used |= 1u << bj;
          gsum += best;
        }
        if (lane == g) my_group_score = gsum;
      }
      uint32_t keep = 0;  // warp-uniform mask of the eligible groups
      for (int r = 0; r < M; ++r) {
        float best = (lane < G && !((keep >> lane) & 1u)) ? my_group_score : -INFINITY;
        int bid = lane < G ? lane : 32;
        if ((keep >> lane) & 1u) bid = 32;
        warp_argmax(best, bid);
        keep |= 1u << bid;
      }
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) {
        const int e = lane + 32 * j;
        if (j < per_lane && e < N && !((keep >> (e / size)) & 1u)) sc[j] = -INFINITY;
      }
    }
    uint32_t taken = 0;
    int my_id = 0;
    float my_s = 0.0f, sum = 0.0f;
    for (int k = 0; k < K; ++k) {
      float best = -INFINITY, best_s = 0.0f;
      int bid = N, bj = -1;
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) {
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
      if (counts != nullptr) atomicAdd(&counts[my_id], 1);
    }
  }
}

// Top-K over the logits with the smallest per-lane bound that holds N.
cudaError_t launch_topk(const float* logits, const float* bias, int T, int N, int K, int G, int M,
                        int32_t* ids, float* gates, int32_t* counts, cudaStream_t stream,
                        int sm_count) {
  int blocks = (T + 7) / 8;
  if (blocks > sm_count * 8) blocks = sm_count * 8;
  const int per_lane = (N + 31) / 32;
  if (per_lane <= 4)
    topk_kernel<4><<<blocks, 256, 0, stream>>>(logits, bias, T, N, K, G, M, ids, gates, counts);
  else if (per_lane <= 8)
    topk_kernel<8><<<blocks, 256, 0, stream>>>(logits, bias, T, N, K, G, M, ids, gates, counts);
  else if (per_lane <= 16)
    topk_kernel<16><<<blocks, 256, 0, stream>>>(logits, bias, T, N, K, G, M, ids, gates, counts);
  else
    topk_kernel<kMaxPerLane><<<blocks, 256, 0, stream>>>(logits, bias, T, N, K, G, M, ids, gates,
                                                        counts);
  return cudaGetLastError();
}

// Sequence-wise balance statistics in three passes, every sum in a fixed
// order so the results do not depend on scheduling:
//   1. one warp per token: D_t = sum_j s_tj over all N affinities, recomputed
//      from the logits exactly as topk_kernel computes them;
//   2. one CTA per chunk of <= kBalChunk tokens of one sequence, one thread
//      per expert: the chunk's sum of s_ti / D_t (token order) and its
//      selection counts (integer atomics);
//   3. one CTA per sequence: chunk partials added in chunk order, then f, P
//      and alpha * sum_i f_i P_i (expert order).
constexpr int kBalChunk = 128;

__global__ void __launch_bounds__(256) token_sum_kernel(const float* __restrict__ z, int T, int N,
                                                        float* __restrict__ denom) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int per_lane = (N + 31) >> 5;
  for (int t = blockIdx.x * warps + (threadIdx.x >> 5); t < T; t += gridDim.x * warps) {
    float part = 0.0f;
    for (int j = 0; j < per_lane; ++j) {
      const int e = lane + 32 * j;
      if (e < N) part += affinity(z[(int64_t)t * N + e]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) denom[t] = part;
  }
}

__global__ void __launch_bounds__(1024) chunk_partial_kernel(
    const float* __restrict__ z, const int32_t* __restrict__ ids, const float* __restrict__ denom,
    int T, int N, int K, int seq_len, int chunks_per_seq, float* __restrict__ part_p,
    int32_t* __restrict__ part_c) {
  __shared__ int cnt[1024];
  const int seq = blockIdx.x / chunks_per_seq, chunk = blockIdx.x % chunks_per_seq;
  const int seq_end = min(T, (seq + 1) * seq_len);
  const int lo = seq * seq_len + chunk * kBalChunk;
  const int hi = min(seq_end, lo + kBalChunk);
  for (int i = threadIdx.x; i < N; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  for (int i = lo * K + threadIdx.x; i < hi * K; i += blockDim.x) {
    const int e = ids[i];
    if (e >= 0 && e < N) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    float acc = 0.0f;
    for (int t = lo; t < hi; ++t) acc += affinity(z[(int64_t)t * N + e]) / denom[t];
    part_p[(int64_t)blockIdx.x * N + e] = acc;
    part_c[(int64_t)blockIdx.x * N + e] = cnt[e];
  }
}

__global__ void __launch_bounds__(1024) seq_reduce_kernel(const float* __restrict__ part_p,
                                                          const int32_t* __restrict__ part_c,
                                                          int T, int N, int K, int seq_len,
                                                          int chunks_per_seq, float alpha,
                                                          float* __restrict__ f,
                                                          float* __restrict__ P,
                                                          float* __restrict__ loss) {
  __shared__ float fp[1024];
  const int q = blockIdx.x;
  const int t_seq = min(T, (q + 1) * seq_len) - q * seq_len;
  for (int e = threadIdx.x; e < N; e += blockDim.x) {
    float ps = 0.0f;
    int c = 0;
    for (int k = 0; k < chunks_per_seq; ++k) {
      const int64_t at = ((int64_t)q * chunks_per_seq + k) * N + e;
      ps += part_p[at];
      c += part_c[at];
    }
    const float pi = ps / (float)t_seq;
    const float fi = (float)N * (float)c / ((float)K * (float)t_seq);
    P[(int64_t)q * N + e] = pi;
    f[(int64_t)q * N + e] = fi;
    fp[e] = fi * pi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float sum = 0.0f;
    for (int e = 0; e < N; ++e) sum += fp[e];
    loss[q] = alpha * sum;
  }
}

}  // namespace

size_t balance_scratch_bytes(int64_t T, int64_t N) {
  const int64_t parts = T + (T + kBalChunk - 1) / kBalChunk;
  return (size_t)((T * 4 + 255) / 256 * 256 + 2 * parts * N * 4);
}

cudaError_t launch_balance_stats(const float* logits, const int32_t* ids, int T, int N, int K,
                                 int seq_len, float alpha, uint8_t* scratch, float* f, float* P,
                                 float* loss, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int n_seq = (T + seq_len - 1) / seq_len;
  const int per_seq = (std::min(seq_len, T) + kBalChunk - 1) / kBalChunk;
  // n_seq * per_seq <= T + ceil(T / kBalChunk): the scratch bound
  float* denom = reinterpret_cast<float*>(scratch);
  const int64_t parts = (int64_t)n_seq * per_seq;
  if (parts > (int64_t)T + (T + kBalChunk - 1) / kBalChunk) return cudaErrorInvalidValue;
  float* part_p = reinterpret_cast<float*>(scratch + ((int64_t)T * 4 + 255) / 256 * 256);
  int32_t* part_c = reinterpret_cast<int32_t*>(part_p + parts * N);
  int blocks = (T + 7) / 8;
  if (blocks > 148 * 8) blocks = 148 * 8;
  token_sum_kernel<<<blocks, 256, 0, stream>>>(logits, T, N, denom);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int threads = std::min(1024, (N + 31) / 32 * 32);
  chunk_partial_kernel<<<(unsigned)parts, threads, 0, stream>>>(logits, ids, denom, T, N, K,
                                                                seq_len, per_seq, part_p, part_c);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  seq_reduce_kernel<<<n_seq, threads, 0, stream>>>(part_p, part_c, T, N, K, seq_len, per_seq,
                                                   alpha, f, P, loss);
  return cudaGetLastError();
}

cudaError_t launch_router(const void* x, const float* gate_w, const float* bias, int T, int H,
                          int N, int K, int G, int M, float* logits, int32_t* ids, float* gates,
                          int32_t* counts, uint32_t* status, cudaStream_t stream, int sm_count) {
  (void)status;
  if (T == 0) return cudaSuccess;
  dim3 g1((T + kLT - 1) / kLT, (N + kLE - 1) / kLE);
  logits_kernel<<<g1, 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16*>(x), gate_w, T, H, N,
                                        logits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_topk(logits, bias, T, N, K, G, M, ids, gates, counts, stream, sm_count);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Gate logits on tcgen05 tensor cores. The fp32 centroids are split exactly
// into three bf16 terms (hi + mid + lo carries all 24 significand bits), so
// x . e_i = sum over the terms of bf16 x bf16 products, each exact in fp32,
// accumulated in fp32 in TMEM: fp32-accurate logits from BF16 MMAs.
// One CTA computes a 128-token x 64-expert tile over the whole hidden size.
// ---------------------------------------------------------------------------
namespace moe {

namespace {

constexpr int kRM = 128;                  // tokens per tile
constexpr int kRN = 64;                   // experts per tile
constexpr int kRK = 64;                   // bf16 elements per k-block (128 bytes)
constexpr int kRStages = 5;
constexpr int kRABytes = kRM * kRK * 2;   // 16 KB
constexpr int kRBBytes = kRN * kRK * 2;   // 8 KB per split term
constexpr int kRStageBytes = kRABytes + 3 * kRBBytes;
constexpr int kRThreads = 256;
constexpr uint32_t kRIdesc = make_idesc(kRM, kRN, 1u, 1u);  // BF16 x BF16 -> fp32
constexpr size_t kRDynSmem = (size_t)kRStages * kRStageBytes + 1024;

__global__ void __launch_bounds__(256) split_gate_kernel(const float* __restrict__ w, int64_t n,
                                                         __nv_bfloat16* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = w[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);   // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);  // exact
    out[i] = hi;
    out[n + i] = mid;
    out[2 * n + i] = __float2bfloat16_rn(r2);
  }
}

struct alignas(8) RouterShared {
  uint64_t full[kRStages];
  uint64_t empty[kRStages];
  uint64_t tfull;
  uint32_t tmem_base;
  int abort;
};

__global__ void __launch_bounds__(kRThreads, 1)
    logits_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const __grid_constant__ CUtensorMap tm_w, int T, int H, int N,
                     float* __restrict__ z, uint32_t* __restrict__ status) {
  __shared__ RouterShared sh;
  extern __shared__ uint8_t dyn_smem[];
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kRM;
  const int n0 = blockIdx.y * kRN;
  const int kb_n = H / kRK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      mbar_init(smem_u32(&sh.empty[s]), 1);
    }
    mbar_init(smem_u32(&sh.tfull), 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), kRN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  volatile int* abort = &sh.abort;

  if (warp == 0) {
    if (lane == 0) {
      // producer: x tile and the three centroid terms of every k-block
      int kb = 0;
      for (; kb < kb_n; ++kb) {
        const int s = kb % kRStages;
        const uint32_t ph = (uint32_t)(kb / kRStages) & 1u;
        if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort, status)) break;
        const uint32_t full = smem_u32(&sh.full[s]);
        mbar_arrive_expect_tx(full, kRStageBytes);
        const uint32_t sa = ring + s * kRStageBytes;
        tma_load_2d(sa, &tm_x, kb * kRK, m0, full);
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(sa + kRABytes + t * kRBBytes),
              "l"(reinterpret_cast<uint64_t>(&tm_w)), "r"(kb * kRK), "r"(n0), "r"(t), "r"(full)
              : "memory");
        }
      }
      if (kb < kb_n) {
        for (int s = 0; s < kRStages && s < kb; ++s) {
          const int last = s + ((kb - 1 - s) / kRStages) * kRStages;
          mbar_wait(smem_u32(&sh.full[s]), (uint32_t)(last / kRStages) & 1u, nullptr, status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer: one fp32 accumulator over all of H and the three terms
      bool ok = true;
      bool issued = false;
      for (int kb = 0; kb < kb_n; ++kb) {
        const int s = kb % kRStages;
        const uint32_t ph = (uint32_t)(kb / kRStages) & 1u;
        if (!mbar_wait(smem_u32(&sh.full[s]), ph, abort, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = ring + s * kRStageBytes;
#pragma unroll
        for (int t = 0; t < 3; ++t) {
#pragma unroll
          for (int k = 0; k < kRK / 16; ++k) {
            mma_bf16(tmem_base, smem_desc_sw128(sa + k * 32),
                     smem_desc_sw128(sa + kRABytes + t * kRBBytes + k * 32), kRIdesc,
                     (kb | t | k) != 0 ? 1u : 0u);
          }
        }
        issued = true;
        mma_commit(smem_u32(&sh.empty[s]));
      }
      if (issued) mma_commit(smem_u32(&sh.tfull));
      if (!ok && issued) mbar_wait(smem_u32(&sh.tfull), 0u, nullptr, status);
    }
  } else if (warp >= 4) {
    // epilogue: 128 rows x 64 columns of fp32 logits -> z
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.tfull), 0u, abort, status));
    if (ok) {
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16);
      float v0[32], v1[32];
      tmem_ld32(t0, v0);
      tmem_ld32(t0 + 32, v1);
      tmem_wait_ld();
      const int t = m0 + row;
      if (t < T) {
        float* dst = z + (int64_t)t * N + n0;
        const int cols = min(kRN, N - n0);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (4 * j < cols) reinterpret_cast<float4*>(dst)[j] = make_float4(v0[4 * j], v0[4 * j + 1], v0[4 * j + 2], v0[4 * j + 3]);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (32 + 4 * j < cols) reinterpret_cast<float4*>(dst + 32)[j] = make_float4(v1[4 * j], v1[4 * j + 1], v1[4 * j + 2], v1[4 * j + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kRN);
}

// Wide tiles for large batches: one CTA computes 256 tokens x 256 experts
// (two 128-row fp32 accumulators in TMEM, 512 columns, sharing each k-block's
// centroid tile), so the split centroids are streamed once per 256 tokens
// instead of once per 128 tokens and 64 experts. k-blocks are 32 bf16 wide
// (64-byte rows, 64-byte swizzle) to fit three stages of x (16 KB) and the
// three centroid terms (48 KB).
constexpr int kWM = 256;                  // tokens per tile (two accumulators)
constexpr int kWN = 256;                  // experts per tile
constexpr int kWK = 32;                   // bf16 elements per k-block (64 bytes)
constexpr int kWStages = 3;
constexpr int kWABytes = kWM * kWK * 2;   // 16 KB
constexpr int kWBBytes = kWN * kWK * 2;   // 16 KB per split term
constexpr int kWStageBytes = kWABytes + 3 * kWBBytes;
constexpr int kWThreads = 384;
constexpr uint32_t kWIdesc = make_idesc(128, kWN, 1u, 1u);  // BF16 x BF16 -> fp32
constexpr size_t kWDynSmem = (size_t)kWStages * kWStageBytes + 1024;

struct alignas(8) WideShared {
  uint64_t full[kWStages];
  uint64_t empty[kWStages];
  uint64_t tfull;
  uint32_t tmem_base;
  int abort;
  float bias[kWN];
};

// Selection fused into the wide tiles' epilogue when one tile holds all of a
// token's scores (N = 256) and K <= kFuseL: each epilogue thread owns one
// token (one TMEM lane) and keeps its best kFuseL (score, id, affinity)
// triples in registers, sorted, while the 256 columns stream past in chunks
// of 32. Candidates arrive in ascending id, so a candidate ties with a kept
// entry only to lose (the lower id wins), exactly as in topk_kernel; the
// first K entries of the sorted list are topk_kernel's K choices in its
// order. Node-limited routing is fused for G = 8 groups of 32 experts (one
// chunk each): a first pass sums each group's K/M highest scores (highest
// first), the M best groups are kept (lower group on ties) and the other
// groups' experts enter the second pass with score -inf.
constexpr int kFuseL = 8;
constexpr int kStashStride = 256;  // one float per epilogue thread per row
static_assert(64 * kStashStride * 4 <= kWStages * kWStageBytes, "stash fits in the ring");

MOE_DEV bool ranks_above(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

struct FuseArgs {
  const float* bias;
  int K, G, M;
  int32_t* ids;
  float* gates;
  int32_t* counts;  // null: not counted
};

// Warps: 0 TMA producer, 1 TMEM allocator and MMA issuer, 2-3 idle, 4-11
// epilogue (warpgroup h reads accumulator h: tokens 128h .. 128h + 127).
// kMode: kWideLogits writes the logits; kWideSelect also makes the selection
// (above); kWideSplit covers the slice blockIdx.z of gridDim.z equal slices
// of the reduction and writes its fp32 partial sums to z + blockIdx.z * T * N
// (summed in slice order by splitk_reduce_kernel).
enum WideMode : int { kWideLogits = 0, kWideSelect = 1, kWideSplit = 2 };

template <int kMode>
__global__ void __launch_bounds__(kWThreads, 1)
    logits_tc_wide_kernel(const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_w, int T, int H, int N,
                          float* __restrict__ z, uint32_t* __restrict__ status, FuseArgs fa) {
  __shared__ WideShared sh;
  extern __shared__ uint8_t dyn_smem[];
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool kFuse = kMode == kWideSelect;
  constexpr bool kSplit = kMode == kWideSplit;
  const int m0 = blockIdx.x * kWM;
  const int n0 = blockIdx.y * kWN;
  const int kb_all = H / kWK;
  const int kb_lo = kSplit ? (int)((int64_t)kb_all * blockIdx.z / gridDim.z) : 0;
  const int kb_n = (kSplit ? (int)((int64_t)kb_all * (blockIdx.z + 1) / gridDim.z) : kb_all) - kb_lo;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      mbar_init(smem_u32(&sh.empty[s]), 1);
    }
    mbar_init(smem_u32(&sh.tfull), 1);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_w);
  }
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), 512);
  if (kFuse && warp >= 4) {
    const int i = threadIdx.x - 128;
    sh.bias[i] = fa.bias[n0 + i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  volatile int* abort = &sh.abort;

  if (warp == 0) {
    if (lane == 0) {
      // producer: 256 rows of x and the three centroid terms of every k-block
      int kb = 0;
      for (; kb < kb_n; ++kb) {
        const int s = kb % kWStages;
        const uint32_t ph = (uint32_t)(kb / kWStages) & 1u;
        if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort, status)) break;
        const uint32_t full = smem_u32(&sh.full[s]);
        mbar_arrive_expect_tx(full, kWStageBytes);
        const uint32_t sa = ring + s * kWStageBytes;
        tma_load_2d(sa, &tm_x, (kb_lo + kb) * kWK, m0, full);
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(sa + kWABytes),
            "l"(reinterpret_cast<uint64_t>(&tm_w)), "r"((kb_lo + kb) * kWK), "r"(n0), "r"(0),
            "r"(full)
            : "memory");
      }
      if (kb < kb_n) {
        for (int s = 0; s < kWStages && s < kb; ++s) {
          const int last = s + ((kb - 1 - s) / kWStages) * kWStages;
          mbar_wait(smem_u32(&sh.full[s]), (uint32_t)(last / kWStages) & 1u, nullptr, status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer: per k-block, each 128-token half against the three terms,
      // two K=16 steps each, all into that half's fp32 accumulator
      bool ok = true;
      bool issued = false;
      for (int kb = 0; kb < kb_n; ++kb) {
        const int s = kb % kWStages;
        const uint32_t ph = (uint32_t)(kb / kWStages) & 1u;
        if (!mbar_wait(smem_u32(&sh.full[s]), ph, abort, status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sa = ring + s * kWStageBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int t = 0; t < 3; ++t) {
#pragma unroll
            for (int k = 0; k < kWK / 16; ++k) {
              mma_bf16(tmem_base + (uint32_t)(h * kWN),
                       smem_desc_sw64(sa + h * (kWABytes / 2) + k * 32),
                       smem_desc_sw64(sa + kWABytes + t * kWBBytes + k * 32), kWIdesc,
                       (kb | t | k) != 0 ? 1u : 0u);
            }
          }
        }
        issued = true;
        mma_commit(smem_u32(&sh.empty[s]));
      }
      if (issued) mma_commit(smem_u32(&sh.tfull));
      if (!ok && issued) mbar_wait(smem_u32(&sh.tfull), 0u, nullptr, status);
    }
  } else if (warp >= 4) {
    // epilogue: each thread one token's 256 fp32 logits -> z
    const int h = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int t = m0 + h * 128 + quarter * 32 + lane;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.tfull), 0u, abort, status));
    if (ok) {
      tc_fence_after();
      const uint32_t t0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(h * kWN);
      const int cols = min(kWN, N - n0);
      float* dst = z + (kSplit ? (int64_t)blockIdx.z * T * N : 0) + (int64_t)t * N + n0;
      // this thread's column of the stash: 32 (affinity, score) pairs
      float* stash = reinterpret_cast<float*>(dyn_smem + (ring - smem_u32(dyn_smem))) +
                     (threadIdx.x - 128);
      // node-limited routing: which of the 8 groups this token keeps
      uint32_t keep = 0xffffffffu;
      if (kFuse && fa.G > 1 && fa.M < fa.G) {
        const int per_group = fa.K / fa.M;
        float gs[8];
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float v[32];
          tmem_ld32(t0 + (uint32_t)(32 * c), v);
          tmem_wait_ld();
          if (per_group <= 2) {
            // the two highest, branch-free: t0 >= t1 throughout
            float h0 = -INFINITY, h1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float sc = biased_score(affinity(v[j]), sh.bias[32 * c + j]);
              h1 = fmaxf(h1, fminf(h0, sc));
              h0 = fmaxf(h0, sc);
            }
            const float gsum = per_group == 1 ? 0.0f + h0 : (0.0f + h0) + h1;
#pragma unroll
            for (int g = 0; g < 8; ++g)
              if (g == c) gs[g] = gsum;
            continue;
          }
          float top[kFuseL];
#pragma unroll
          for (int i = 0; i < kFuseL; ++i) top[i] = -INFINITY;
          // the chunk's scores first (independent: no branch between them)
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = biased_score(affinity(v[j]), sh.bias[32 * c + j]);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float sc = v[j];
            if (sc > top[kFuseL - 1]) {
              bool b[kFuseL];
#pragma unroll
              for (int i = 0; i < kFuseL; ++i) b[i] = sc > top[i];
#pragma unroll
              for (int i = kFuseL - 1; i > 0; --i) top[i] = b[i - 1] ? top[i - 1] : (b[i] ? sc : top[i]);
              top[0] = b[0] ? sc : top[0];
            }
          }
          float gsum = 0.0f;
#pragma unroll
          for (int i = 0; i < kFuseL; ++i)
            if (i < per_group) gsum += top[i];
#pragma unroll
          for (int g = 0; g < 8; ++g)
            if (g == c) gs[g] = gsum;
        }
        keep = 0;
        for (int r = 0; r < fa.M; ++r) {
          float best = -INFINITY;
          int bid = 32;
#pragma unroll
          for (int g = 0; g < 8; ++g)
            if (!((keep >> g) & 1u) && ranks_above(gs[g], g, best, bid)) {
              best = gs[g];
              bid = g;
            }
          keep |= 1u << bid;
        }
      }
      float lv[kFuseL], ls[kFuseL];
      int li[kFuseL];
#pragma unroll
      for (int i = 0; i < kFuseL; ++i) {
        lv[i] = -INFINITY;
        li[i] = kWN;  // beaten by every real expert
        ls[i] = 0.0f;
      }
#pragma unroll 1
      for (int c = 0; c < kWN; c += 32) {
        float v[32];
        tmem_ld32(t0 + (uint32_t)c, v);
        tmem_wait_ld();
        if (t < T) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (c + 4 * j < cols)
              reinterpret_cast<float4*>(dst + c)[j] =
                  make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
        if (kFuse) {
          // a masked group's experts score -inf: they matter only while the
          // list still holds a -inf entry
          const bool masked = !((keep >> (c / 32)) & 1u);
          if (!masked || lv[kFuseL - 1] == -INFINITY) {
            // the chunk's affinities and scores (independent, no branches),
            // stashed in the idle operand ring; the candidates that beat the
            // list's last entry as it stood before the chunk are marked, and
            // only those are inserted, in ascending id: a warp then runs as
            // many insertions as its busiest lane, not one per column that
            // any lane wants
            uint32_t pass = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float a = affinity(v[j]);
              const float sc = masked ? -INFINITY : biased_score(a, sh.bias[c + j]);
              stash[(2 * j) * kStashStride] = a;
              stash[(2 * j + 1) * kStashStride] = sc;
              pass |= (uint32_t)ranks_above(sc, c + j, lv[kFuseL - 1], li[kFuseL - 1]) << j;
            }
            while (pass != 0u) {
              const int j = __ffs(pass) - 1;
              pass &= pass - 1u;
              const int e = c + j;
              const float s = stash[(2 * j) * kStashStride];
              const float sc = stash[(2 * j + 1) * kStashStride];
              if (ranks_above(sc, e, lv[kFuseL - 1], li[kFuseL - 1])) {
                bool b[kFuseL];
#pragma unroll
                for (int i = 0; i < kFuseL; ++i) b[i] = ranks_above(sc, e, lv[i], li[i]);
#pragma unroll
                for (int i = kFuseL - 1; i > 0; --i) {
                  lv[i] = b[i - 1] ? lv[i - 1] : (b[i] ? sc : lv[i]);
                  li[i] = b[i - 1] ? li[i - 1] : (b[i] ? e : li[i]);
                  ls[i] = b[i - 1] ? ls[i - 1] : (b[i] ? s : ls[i]);
                }
                lv[0] = b[0] ? sc : lv[0];
                li[0] = b[0] ? e : li[0];
                ls[0] = b[0] ? s : ls[0];
              }
            }
          }
        }
      }
      if (kFuse && t < T) {
        // gates from the unbiased affinities, normalised in selection order
        float sum = 0.0f;
#pragma unroll
        for (int i = 0; i < kFuseL; ++i)
          if (i < fa.K) sum += ls[i];
#pragma unroll
        for (int i = 0; i < kFuseL; ++i) {
          if (i < fa.K) {
            fa.ids[(int64_t)t * fa.K + i] = li[i];
            fa.gates[(int64_t)t * fa.K + i] = ls[i] / sum;
            if (fa.counts != nullptr) atomicAdd(&fa.counts[li[i]], 1);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

// z = the sum of the S slices' partial logits, added in slice order.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4* __restrict__ part,
                                                           int64_t n4, int S,
                                                           float4* __restrict__ z) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 a = part[i];
    for (int s = 1; s < S; ++s) {
      const float4 b = part[(int64_t)s * n4 + i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    z[i] = a;
  }
}

// Slices of the reduction for wide tiles when neither tile shape alone fills
// the GPU (batches below the wide tiles' threshold): as many as keep the 148
// SMs of a B200 busy, each at least 8 k-blocks (256 channels) deep; 0 = none.
// The count depends on the shape only (not on the device or on the scratch
// given), so every path that routes the same tokens sums the same slices.
int splitk_slices(int64_t T, int64_t N, int64_t H) {
  constexpr int64_t kSms = 148;
  if (N % kWN != 0 || T <= 0) return 0;
  const int64_t tiles = ((T + kWM - 1) / kWM) * (N / kWN);
  const int64_t s = std::min<int64_t>(kSms / tiles, (H / kWK) / 8);
  return s >= 2 ? (int)s : 0;
}

}  // namespace

size_t router_splitk_bytes(int64_t T, int N, int H) {
  return (size_t)splitk_slices(T, N, H) * (size_t)T * (size_t)N * sizeof(float);
}

size_t router_split_bytes(int N, int H) { return (size_t)3 * N * H * sizeof(__nv_bfloat16); }

// Wide tiles move about 3.2x the bytes of a 128 x 64 tile through L2 for 8x
// its logits; they pay off once the small tiles would need more than 3.2
// times as many waves as the wide ones (T = 32768 at N = 256: 7 against 1).
static bool use_wide_logits(int64_t T, int64_t N, int sm_count) {
  if (N % kWN != 0) return false;  // whole 256-expert tiles only
  const int64_t sms = sm_count > 0 ? sm_count : 148;
  const int64_t small = ((T + kRM - 1) / kRM) * ((N + kRN - 1) / kRN);
  const int64_t wide = ((T + kWM - 1) / kWM) * ((N + kWN - 1) / kWN);
  const int64_t small_waves = (small + sms - 1) / sms;
  const int64_t wide_waves = (wide + sms - 1) / sms;
  return 10 * small_waves > 32 * wide_waves;
}

cudaError_t launch_split_gate(const float* gate_w, int N, int H, __nv_bfloat16* wsplit,
                              cudaStream_t stream, int sm_count) {
  const int64_t nw = (int64_t)N * H;
  if (nw == 0) return cudaSuccess;
  split_gate_kernel<<<(unsigned)std::min<int64_t>((nw + 255) / 256, (int64_t)sm_count * 8), 256, 0,
                      stream>>>(gate_w, nw, wsplit);
  return cudaGetLastError();
}

cudaError_t launch_router_tc(const void* x, const float* gate_w, const float* bias, int T, int H,
                             int N, int K, int G, int M, __nv_bfloat16* wsplit, float* logits,
                             int32_t* ids, float* gates, int32_t* counts, uint32_t* status,
                             cudaStream_t stream, int sm_count, const __nv_bfloat16* presplit,
                             float* splitk_scratch, size_t splitk_bytes) {
  if (T == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  if (presplit == nullptr) {
    e = launch_split_gate(gate_w, N, H, wsplit, stream, sm_count);
    if (e != cudaSuccess) return e;
  }
  const __nv_bfloat16* terms = presplit != nullptr ? presplit : wsplit;
  static DeviceOnce once;  // the shared-memory limits are raised once per device
  e = once.run([] {
    cudaError_t r = cudaFuncSetAttribute(logits_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kRDynSmem);
    if (r != cudaSuccess) return r;
    r = cudaFuncSetAttribute(logits_tc_wide_kernel<kWideLogits>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWDynSmem);
    if (r != cudaSuccess) return r;
    r = cudaFuncSetAttribute(logits_tc_wide_kernel<kWideSplit>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWDynSmem);
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(logits_tc_wide_kernel<kWideSelect>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWDynSmem);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap mx, mw;
  if (use_wide_logits(T, N, sm_count)) {
    e = make_tmap_bf16(&mx, x, H, T, 1, kWK, kWM);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&mw, terms, H, N, 3, kWK, kWN, 3);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((T + kWM - 1) / kWM), (unsigned)((N + kWN - 1) / kWN));
    const bool grouped = G > 1 && M < G;
    FuseArgs fa{bias, K, G, M, ids, gates, counts};
    if (N == kWN && K <= kFuseL && (!grouped || G == 8)) {
      // the selection runs in the tiles' epilogue
      logits_tc_wide_kernel<kWideSelect><<<grid, kWThreads, kWDynSmem, stream>>>(
          mx, mw, T, H, N, logits, status, fa);
      return cudaGetLastError();
    }
    logits_tc_wide_kernel<kWideLogits><<<grid, kWThreads, kWDynSmem, stream>>>(
        mx, mw, T, H, N, logits, status, fa);
  } else if (const int S = splitk_slices(T, N, H);
             S >= 2 && splitk_scratch != nullptr &&
             (size_t)S * (size_t)T * (size_t)N * sizeof(float) <= splitk_bytes) {
    // wide tiles over S slices of the reduction, then the slices' sum
    e = make_tmap_bf16(&mx, x, H, T, 1, kWK, kWM);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&mw, terms, H, N, 3, kWK, kWN, 3);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((T + kWM - 1) / kWM), (unsigned)(N / kWN), (unsigned)S);
    FuseArgs fa{};
    logits_tc_wide_kernel<kWideSplit><<<grid, kWThreads, kWDynSmem, stream>>>(
        mx, mw, T, H, N, splitk_scratch, status, fa);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n4 = (int64_t)T * N / 4;
    const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, (int64_t)sm_count * 8);
    splitk_reduce_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        reinterpret_cast<const float4*>(splitk_scratch), n4, S, reinterpret_cast<float4*>(logits));
  } else {
    e = make_tmap_bf16(&mx, x, H, T, 1, kRK, kRM);
    if (e != cudaSuccess) return e;
    e = make_tmap_bf16(&mw, terms, H, N, 3, kRK, kRN);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((T + kRM - 1) / kRM), (unsigned)((N + kRN - 1) / kRN));
    logits_tc_kernel<<<grid, kRThreads, kRDynSmem, stream>>>(mx, mw, T, H, N, logits, status);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_topk(logits, bias, T, N, K, G, M, ids, gates, counts, stream, sm_count);
}

}  // namespace moe
