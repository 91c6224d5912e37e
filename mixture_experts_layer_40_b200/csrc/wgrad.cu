// Weight-gradient GEMMs of the expert backward in FP8 ("DeepSeek-V3:
// Auxiliary-Loss-Free MoE Load Balancing, Multi-Token Prediction, and FP8
// Training at 671B Scale", section V, Figure 6: Wgrad in E4M3, fp32
// accumulation). For every expert g,
//   C_g [M, N] = A_g [M, K_g] . B_g [N, K_g]^T,   K_g = the expert's GEMM rows
// with both operands stored transposed ([channel, GEMM row], K-major) and
// quantised in tiles of 1 channel x 128 GEMM rows, so the reduction runs
// over the tokens and every 128 of them is promoted to fp32 with its own
// per-row (A) and per-column (B) scale: C += P_kb * (1/s_a[m]) * (1/s_b[n]).
// The expert segments start 128-aligned and their padding rows hold zeros.
//
// Same machinery as the forward's grouped GEMM: one persistent CTA per SM,
// warp 0 TMA producer (3-stage ring of 128x128 A and 256x128 B k-blocks and
// B's 256 inverse column scales of the k-block; a stage is free again once
// the MMA and the promotion warps have both used it),
// warp 1 TMEM allocator and single-thread tcgen05 MMA issuer (two 256-column
// TMEM buffers), warps 4-11 promotion and fp32 output through shared memory
// and TMA stores. Every wait is bounded.
#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

// Plain bulk copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned) from global to shared memory, completing on `bar`.
MOE_DEV void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}


constexpr int kBM = 128, kBN = 256, kBK = 128;
constexpr int kStages = 3;  // two stages' worth of smem goes to output staging
constexpr int kABytes = kBM * kBK, kBBytes = kBN * kBK;
constexpr int kSBytes = kBN * 4;  // the k-block's inverse column scales of B
// a stage: A tile, B tile, then B's 256 inverse column scales (so that the
// promotion reads them from shared memory, not with L2 latency per k-block)
constexpr int kStageBytes = kABytes + kBBytes + 1024;
constexpr int kThreads = 384;
constexpr int kYCols = 32;                       // fp32 columns per TMA store
constexpr int kYBufBytes = 32 * kYCols * 4;      // 32 rows x 128 bytes
constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + 8 * 2 * kYBufBytes + 1024;
constexpr uint32_t kIdesc = make_idesc(kBM, kBN, 0u, 0u);  // E4M3 x E4M3 -> fp32
constexpr int kLaunchRegs = 168, kRegsCtl = 40, kRegsEpi = 232;
static_assert(128 * kRegsCtl + 256 * kRegsEpi <= kThreads * kLaunchRegs, "register split");
static_assert(kDynSmem + 1024 <= 232448, "shared memory");

struct WgradArgs {
  const int32_t* group_rows;   // [G] rows of each expert (without padding)
  const int32_t* group_start;  // [G] first GEMM row (multiple of 128)
  int32_t n_groups;
  int32_t m_tiles;             // M / 128
  int32_t n_tiles;             // N / 256
  int32_t kb_total;            // GEMM rows / 128
  int32_t M, N;
  const float* a_s;            // [M, kb_total] scales of A's tiles
  const float* b_inv;          // [kb_total, N] inverse scales of B's tiles
  uint32_t* status;
};

struct alignas(8) WgradShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem_base;
  int abort;
};

MOE_DEV void decode(int tile, const WgradArgs& p, int& g, int& m, int& n, int& kb0, int& kbn) {
  const int per_group = p.m_tiles * p.n_tiles;
  g = tile / per_group;
  const int local = tile - g * per_group;
  m = local / p.n_tiles;
  n = local - m * p.n_tiles;
  const int rows = p.group_rows[g], start = p.group_start[g];
  const bool ok = rows >= 0 && start >= 0 && start % kBM == 0 &&
                  (int64_t)start + rows <= (int64_t)p.kb_total * kBM;
  kb0 = ok ? start / kBM : 0;
  kbn = ok ? (rows + kBM - 1) / kBM : 0;
}

__global__ void __launch_bounds__(kThreads, 1)
    wgrad_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_b,
                      const __grid_constant__ CUtensorMap tm_c, const WgradArgs p) {
  __shared__ WgradShared sh;
  extern __shared__ uint8_t dyn_smem[];
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      // released by the MMA's commit and by the 8 promotion warps once they
      // have read the stage's column scales
      mbar_init(smem_u32(&sh.empty[s]), 1 + 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sh.tfull[b]), 1);
      mbar_init(smem_u32(&sh.tempty[b]), 8);
    }
    sh.abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_c);
  }
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sh.tmem_base;
  const int total_tiles = p.n_groups * p.m_tiles * p.n_tiles;
  volatile int* abort = &sh.abort;
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, m, n, kb0, kbn;
        decode(tile, p, g, m, n, kb0, kbn);
        for (int kb = 0; kb < kbn; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort, p.status)) { ok = false; break; }
          const uint32_t full = smem_u32(&sh.full[s]);
          mbar_arrive_expect_tx(full, kABytes + kBBytes + kSBytes);
          const uint32_t sa = ring + s * kStageBytes;
          tma_load_2d(sa, &tm_a, (kb0 + kb) * kBK, m * kBM, full);
          tma_load_2d(sa + kABytes, &tm_b, (kb0 + kb) * kBK, n * kBN, full);
          bulk_load(sa + kABytes + kBBytes, p.b_inv + (int64_t)(kb0 + kb) * p.N + n * kBN,
                    kSBytes, full);
        }
      }
      if (!ok) {
        for (int s = 0; s < kStages && s < it; ++s) {
          const int last = s + ((it - 1 - s) / kStages) * kStages;
          mbar_wait(smem_u32(&sh.full[s]), (uint32_t)(last / kStages) & 1u, nullptr, p.status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // -------------------------------------------------------- MMA issuer
      int it = 0, kbi = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, m, n, kb0, kbn;
        decode(tile, p, g, m, n, kb0, kbn);
        for (int kb = 0; kb < kbn; ++kb, ++it, ++kbi) {
          const int buf = kbi & 1;
          const uint32_t use = (uint32_t)(kbi >> 1);
          if (!mbar_wait(smem_u32(&sh.tempty[buf]), (use & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
          tc_fence_after();
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&sh.full[s]), ph, abort, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = ring + s * kStageBytes;
          const uint32_t d = tmem_base + (uint32_t)(buf * kBN);
#pragma unroll
          for (int k4 = 0; k4 < kBK / 32; ++k4)
            mma_f8(d, smem_desc_sw128(sa + k4 * 32), smem_desc_sw128(sa + kABytes + k4 * 32), kIdesc,
                   k4 > 0 ? 1u : 0u);
          mma_commit(smem_u32(&sh.empty[s]));
          mma_commit(smem_u32(&sh.tfull[buf]));
        }
      }
      if (!ok && kbi > 0) {
        const int last = kbi - 1;
        mbar_wait(smem_u32(&sh.tfull[last & 1]), (uint32_t)(last >> 1) & 1u, nullptr, p.status);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------- promotion + output
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    const int ew = warp - 4, eg = ew >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const uint32_t ybuf = ring + (uint32_t)(kStages * kStageBytes + ew * 2 * kYBufBytes);
    constexpr int kChunks = kYCols / 4;
    const uint32_t swz = (uint32_t)(lane & (kChunks - 1));  // 128-byte rows: c ^ (r % 8)
    int kbi = 0;
    float acc[128];
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      int g, m, n, kb0, kbn;
      decode(tile, p, g, m, n, kb0, kbn);
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      const int x0 = n * kBN + 128 * eg;
      const float* sa_row = p.a_s + (int64_t)(m * kBM + row) * p.kb_total + kb0;
      bool ok = true;
      for (int kb = 0; kb < kbn; ++kb, ++kbi) {
        const float inv_a = __fdividef(1.0f, ldg_early(sa_row + kb));
        const int buf = kbi & 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&sh.tfull[buf]), (uint32_t)(kbi >> 1) & 1u, abort, p.status));
        if (!ok) break;
        tc_fence_after();
        // the MMA of this k-block has completed, so its stage is still held
        // (the producer refills it only after these warps release it); the
        // wait on its full barrier, long complete, makes the column scales'
        // bulk copy visible to these threads
        const int stage = kbi % kStages;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.full[stage]),
                                               (uint32_t)(kbi / kStages) & 1u, abort, p.status));
        if (!ok) break;
        const float4* binv = reinterpret_cast<const float4*>(
            dyn_smem + (ring - smem_u32(dyn_smem)) + stage * kStageBytes + kABytes + kBBytes) +
            (128 * eg) / 4;
        const uint32_t t0 = lane_addr + (uint32_t)(buf * kBN + 128 * eg);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float4 b[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) b[q] = binv[8 * j + q];
          float v[32];
          tmem_ld32(t0 + 32 * j, v);
          tmem_wait_ld();
          if (j == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(smem_u32(&sh.tempty[buf]));
              mbar_arrive(smem_u32(&sh.empty[stage]));  // its column scales are read
            }
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            acc[32 * j + 4 * q + 0] = fmaf(v[4 * q + 0], inv_a * b[q].x, acc[32 * j + 4 * q + 0]);
            acc[32 * j + 4 * q + 1] = fmaf(v[4 * q + 1], inv_a * b[q].y, acc[32 * j + 4 * q + 1]);
            acc[32 * j + 4 * q + 2] = fmaf(v[4 * q + 2], inv_a * b[q].z, acc[32 * j + 4 * q + 2]);
            acc[32 * j + 4 * q + 3] = fmaf(v[4 * q + 3], inv_a * b[q].w, acc[32 * j + 4 * q + 3]);
          }
        }
      }
      if (!ok) break;
      // C rows g*M + m*128 + 32*quarter.., columns x0.. through shared memory
      const int y0 = g * p.M + m * kBM + quarter * 32;
#pragma unroll
      for (int j = 0; j < 128 / kYCols; ++j) {
        const uint32_t buf_j = ybuf + (uint32_t)((j & 1) * kYBufBytes);
        if (lane == 0) bulk_wait_read_1();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          const uint32_t dst = buf_j + (uint32_t)lane * (kYCols * 4) + (((uint32_t)c ^ swz) << 4);
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                       "f"(acc[kYCols * j + 4 * c]), "f"(acc[kYCols * j + 4 * c + 1]),
                       "f"(acc[kYCols * j + 4 * c + 2]), "f"(acc[kYCols * j + 4 * c + 3])
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tm_c, buf_j, x0 + kYCols * j, y0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

}  // namespace

cudaError_t launch_wgrad(const int32_t* group_rows, const int32_t* group_start, int n_groups,
                         int M, int N, int64_t gemm_rows, const uint8_t* a_t, const float* a_s,
                         const uint8_t* b_t, const float* b_inv, float* c, uint32_t* status,
                         cudaStream_t stream, int sm_count) {
  if (M % kBM != 0 || N % kBN != 0 || gemm_rows % kBM != 0) return cudaErrorInvalidValue;
  // once per device: the register split needs the launch register count it
  // was written for, and the large dynamic shared memory must be allowed
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, wgrad_gemm_kernel);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(wgrad_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kDynSmem);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap ma, mb, mc;
  e = make_tmap_u8(&ma, a_t, gemm_rows, M, kBK, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, b_t, gemm_rows, N, kBK, kBN);
  if (e != cudaSuccess) return e;
  e = make_tmap_f32(&mc, c, N, (int64_t)n_groups * M, kYCols, 32);
  if (e != cudaSuccess) return e;
  WgradArgs a{};
  a.group_rows = group_rows;
  a.group_start = group_start;
  a.n_groups = n_groups;
  a.m_tiles = M / kBM;
  a.n_tiles = N / kBN;
  a.kb_total = (int32_t)(gemm_rows / kBM);
  a.M = M;
  a.N = N;
  a.a_s = a_s;
  a.b_inv = b_inv;
  a.status = status;
  const int64_t tiles = (int64_t)n_groups * a.m_tiles * a.n_tiles;
  const int grid = (int)std::min<int64_t>(sm_count, tiles > 0 ? tiles : 1);
  wgrad_gemm_kernel<<<grid, kThreads, kDynSmem, stream>>>(ma, mb, mc, a);
  return cudaGetLastError();
}

}  // namespace moe
