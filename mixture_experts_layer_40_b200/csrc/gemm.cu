// Grouped FP8 E4M3 expert GEMMs on tcgen05 tensor cores (sm_100a).
//
// Numerics follow "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
// Multi-Token Prediction, and FP8 Training at 671B Scale" (trishampatil.com),
// section V "Four details", items 1-2: E4M3 operands with one scale per 1x128
// activation tile and per 128x128 weight block, and partial sums promoted to
// fp32 every N_C = 128 products. The pages' H800 design promotes on CUDA cores
// while a second WGMMA group computes. Here every 128-deep k-block is summed
// by the tensor core into its own 128-column TMEM buffer (four buffers in a
// ring, so the tensor core can run three k-blocks ahead) and eight promotion
// warps read each buffer back with tcgen05.ld and add partial * 1/(s_a s_b)
// into fp32 register totals.
//
// One persistent CTA per SM, 384 threads (three warpgroups):
//   warp 0     TMA producer: A (128 rows x 128 B) and B (128 rows x 128 B)
//              k-block tiles into a shared-memory ring
//   warp 1     TMEM allocator and MMA issuer (one thread): 4 MMAs of
//              M=128, N=128, K=32 per k-block into TMEM buffer (k-block & 3)
//   warps 2-3  idle (they only complete the first warpgroup)
//   warps 4-11 promotion + epilogue; warp w reads TMEM lanes 32*(w%4)..+31,
//              so each warpgroup covers the 128 rows of a tile and owns half
//              of its 128 columns (64 fp32 totals per thread)
// Work units are (group, n, m) with m fastest, so the m-tiles of one expert's
// weight tile run back to back and the weight tile is read from HBM about
// once.
//   down: a unit is a 128-row x 128-column output tile of Y (fp32).
//   up:   a unit is the 128-channel block n of h for 128 rows, computed as two
//         sub-tiles; sub-tile s multiplies by the 128 rows of w13 that hold
//         W_gate and W_up rows 128n+64s .. 128n+64s+63 (gate first), so the
//         SwiGLU pairs sit in the same tile. h of sub-tile 0 waits in shared
//         memory until sub-tile 1 is done; the 1x128 re-quantisation then
//         sees the whole 128-channel tile.
// Every wait is bounded; a time-out raises the status word and the CTA drains
// its in-flight copies and MMAs before releasing TMEM.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 128;
constexpr int kTmemBufs = 4;
constexpr int kABytes = kBM * kBK;
constexpr int kBBytes = kBN * kBK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;
constexpr int kMaxGroups = 1025;
constexpr uint32_t kIdesc = make_idesc(kBM, kBN, 0u, 0u);  // E4M3 x E4M3 -> fp32
constexpr int kHoldStride = 36;                            // floats per held row (padded)

template <bool kUp>
struct Cfg {
  static constexpr int kStages = kUp ? 5 : 6;
  static constexpr int kSub = kUp ? 2 : 1;  // sub-tiles per work unit
  static constexpr size_t kHoldBytes = kUp ? (size_t)2 * kBM * kHoldStride * 4 : 0;
  static constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + kHoldBytes + 1024;
};

struct GemmArgs {
  const int32_t* group_rows;
  const int32_t* group_start;
  int32_t n_groups;
  int32_t kblocks;        // reduction depth / 128
  int32_t n_units;        // work units per (group, m-tile)
  int32_t b_rows;         // rows of B per group
  int64_t rows;           // rows of A / outputs
  const float* a_s;       // [rows, kblocks]
  const float* b_s;       // [n_groups, b_rows / 128, kblocks]
  uint8_t* h_q;           // up: [rows, I]
  float* h_s;             // up: [rows, I / 128]
  int32_t I;
  float* y;               // down: [rows, H] fp32
  int32_t H;
  uint32_t* status;
};

template <int kStages>
struct alignas(8) GemmShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[kTmemBufs];
  uint64_t tempty[kTmemBufs];
  uint64_t xchg;           // amax exchange between the two epilogue groups
  uint32_t tmem_base;
  int abort;
  int prefix[kMaxGroups + 1];
  float amax[2][2][kBM];   // [unit parity][epilogue group][row]
};

MOE_DEV void decode_unit(int u, const int* prefix, int n_groups, int n_units, int& g, int& n,
                         int& m) {
  int lo = 0, hi = n_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] * n_units <= u) lo = mid; else hi = mid;
  }
  g = lo;
  const int mt = prefix[g + 1] - prefix[g];
  const int local = u - prefix[g] * n_units;
  n = local / mt;
  m = local - n * mt;
}

MOE_DEV float silu(float a) { return a / (1.0f + expf(-a)); }

MOE_DEV uint4 quant16(const float* v, float s) {
  uint4 o;
  o.x = e4m3x4(__fmul_rn(v[0], s), __fmul_rn(v[1], s), __fmul_rn(v[2], s), __fmul_rn(v[3], s));
  o.y = e4m3x4(__fmul_rn(v[4], s), __fmul_rn(v[5], s), __fmul_rn(v[6], s), __fmul_rn(v[7], s));
  o.z = e4m3x4(__fmul_rn(v[8], s), __fmul_rn(v[9], s), __fmul_rn(v[10], s), __fmul_rn(v[11], s));
  o.w = e4m3x4(__fmul_rn(v[12], s), __fmul_rn(v[13], s), __fmul_rn(v[14], s), __fmul_rn(v[15], s));
  return o;
}

template <bool kUp>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, const GemmArgs p) {
  using C = Cfg<kUp>;
  constexpr int kStages = C::kStages;
  constexpr int kSub = C::kSub;
  __shared__ GemmShared<kStages> sh;
  extern __shared__ uint8_t dyn_smem[];
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  // held h of sub-tile 0 (up only): [epilogue group][row][kHoldStride] floats
  float* hold = reinterpret_cast<float*>(dyn_smem + (ring - smem_u32(dyn_smem)) +
                                         (size_t)kStages * kStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      mbar_init(smem_u32(&sh.empty[s]), 1);
    }
    for (int b = 0; b < kTmemBufs; ++b) {
      mbar_init(smem_u32(&sh.tfull[b]), 1);
      mbar_init(smem_u32(&sh.tempty[b]), kEpiThreads / 32);
    }
    mbar_init(smem_u32(&sh.xchg), kEpiThreads);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), kTmemBufs * kBN);
  if (warp == 2) {
    // m-tile prefix over the groups; a group whose rows fall outside the
    // buffers or whose start is not 128-aligned is flagged and skipped
    int carry = 0;
    if (lane == 0) sh.prefix[0] = 0;
    for (int base = 0; base < p.n_groups; base += 32) {
      const int g = base + lane;
      int mt = 0;
      if (g < p.n_groups) {
        const int r = p.group_rows[g];
        const int st = p.group_start[g];
        const bool ok = r >= 0 && st >= 0 && (st % kBM) == 0 && (int64_t)st + r <= p.rows;
        if (!ok) flag_status(p.status, kStatusBounds);
        mt = ok ? (r + kBM - 1) / kBM : 0;
      }
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (g < p.n_groups) sh.prefix[g + 1] = carry + incl;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = sh.tmem_base;
  const int total_units = sh.prefix[p.n_groups] * p.n_units;
  const int kb_n = p.kblocks;
  volatile int* abort = &sh.abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
        int g, n, m;
        decode_unit(u, sh.prefix, p.n_groups, p.n_units, g, n, m);
        const int a_row = p.group_start[g] + m * kBM;
        for (int sub = 0; ok && sub < kSub; ++sub) {
          const int b_row = g * p.b_rows + (n * kSub + sub) * kBN;
          for (int kb = 0; kb < kb_n; ++kb, ++it) {
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)(it / kStages) & 1u;
            if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort, p.status)) { ok = false; break; }
            const uint32_t full = smem_u32(&sh.full[s]);
            mbar_arrive_expect_tx(full, kStageBytes);
            const uint32_t sa = ring + s * kStageBytes;
            tma_load_2d_hint(sa, &tm_a, kb * kBK, a_row, full, pol_a);
            tma_load_2d_hint(sa + kABytes, &tm_b, kb * kBK, b_row, full, pol_b);
          }
        }
      }
      if (!ok) {
        // drain: every armed stage must land before the CTA may exit
        for (int s = 0; s < kStages && s < it; ++s) {
          const int last = s + ((it - 1 - s) / kStages) * kStages;
          mbar_wait(smem_u32(&sh.full[s]), (uint32_t)(last / kStages) & 1u, nullptr, p.status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int it = 0, kbi = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x) {
        for (int sub = 0; ok && sub < kSub; ++sub) {
          for (int kb = 0; kb < kb_n; ++kb, ++it, ++kbi) {
            const int buf = kbi & (kTmemBufs - 1);
            const uint32_t use = (uint32_t)(kbi / kTmemBufs);
            if (!mbar_wait(smem_u32(&sh.tempty[buf]), (use & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
            tc_fence_after();
            const int s = it % kStages;
            const uint32_t ph = (uint32_t)(it / kStages) & 1u;
            if (!mbar_wait(smem_u32(&sh.full[s]), ph, abort, p.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sa = ring + s * kStageBytes;
            const uint32_t d = tmem_base + (uint32_t)(buf * kBN);
#pragma unroll
            for (int k4 = 0; k4 < kBK / 32; ++k4) {
              mma_f8(d, smem_desc_sw128(sa + k4 * 32), smem_desc_sw128(sa + kABytes + k4 * 32),
                     kIdesc, k4 > 0 ? 1u : 0u);
            }
            mma_commit(smem_u32(&sh.empty[s]));
            mma_commit(smem_u32(&sh.tfull[buf]));
          }
        }
      }
      if (!ok && kbi > 0) {
        const int last = kbi - 1;
        mbar_wait(smem_u32(&sh.tfull[last & (kTmemBufs - 1)]),
                  (uint32_t)(last / kTmemBufs) & 1u, nullptr, p.status);
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- epilogue
    const int ew = warp - 4;
    const int eg = ew >> 2;            // epilogue group 0 / 1
    const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const int b_blocks = p.b_rows / kBM;
    // TMEM columns of this thread inside a buffer: up -> gate [32eg, 32eg+32)
    // and up [64+32eg, 64+32eg+32); down -> [64eg, 64eg+64)
    const uint32_t col_a = kUp ? (uint32_t)(32 * eg) : (uint32_t)(64 * eg);
    const uint32_t col_b = kUp ? (uint32_t)(64 + 32 * eg) : (uint32_t)(64 * eg + 32);
    float* my_hold = hold + ((size_t)eg * kBM + row) * kHoldStride;
    int kbi = 0;
    uint32_t xchg_phase = 0;
    int unit_count = 0;
    bool ok = true;
    float acc[64];
    float held_amax = 0.0f;
    for (int u = blockIdx.x; ok && u < total_units; u += gridDim.x, ++unit_count) {
      int g, n, m;
      decode_unit(u, sh.prefix, p.n_groups, p.n_units, g, n, m);
      const int valid = p.group_rows[g] - m * kBM;
      const int64_t grow = (int64_t)p.group_start[g] + m * kBM + row;
      const bool live = row < valid;
      const float* sa_ptr = p.a_s + (live ? grow : 0) * kb_n;
      // weight block scales: up -> W_gate block n and W_up block n (rows 2n,
      // 2n+1 of s13); down -> W_down block n
      const float* sb0 = p.b_s + ((int64_t)g * b_blocks + (kUp ? 2 * n : n)) * kb_n;
      const float* sb1 = p.b_s + ((int64_t)g * b_blocks + (kUp ? 2 * n + 1 : n)) * kb_n;
      for (int sub = 0; ok && sub < kSub; ++sub) {
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0.0f;
        float sa_next = __ldg(sa_ptr);
        float sb0_next = __ldg(sb0);
        float sb1_next = kUp ? __ldg(sb1) : sb0_next;
        for (int kb = 0; kb < kb_n; ++kb, ++kbi) {
          const float sa = sa_next, s0 = sb0_next, s1 = sb1_next;
          if (kb + 1 < kb_n) {
            sa_next = __ldg(sa_ptr + kb + 1);
            sb0_next = __ldg(sb0 + kb + 1);
            sb1_next = kUp ? __ldg(sb1 + kb + 1) : sb0_next;
          }
          const float inv0 = __frcp_rn(sa * s0);
          const float inv1 = kUp ? __frcp_rn(sa * s1) : inv0;
          const int buf = kbi & (kTmemBufs - 1);
          // the result is made warp-uniform: tcgen05.ld below is warp-collective
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.tfull[buf]),
                                                 (uint32_t)(kbi / kTmemBufs) & 1u, abort, p.status));
          if (!ok) break;
          tc_fence_after();
          const uint32_t t0 = lane_addr + (uint32_t)(buf * kBN);
          float pa[16], pb[16], qa[16], qb[16];
          tmem_ld16(t0 + col_a, pa);
          tmem_ld16(t0 + col_a + 16, pb);
          tmem_ld16(t0 + col_b, qa);
          tmem_ld16(t0 + col_b + 16, qb);
          tmem_wait_ld_tied(pa, pb);
          tmem_wait_ld_tied(qa, qb);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&sh.tempty[buf]));
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            acc[i] = fmaf(pa[i], inv0, acc[i]);
            acc[16 + i] = fmaf(pb[i], inv0, acc[16 + i]);
            acc[32 + i] = fmaf(qa[i], inv1, acc[32 + i]);
            acc[48 + i] = fmaf(qb[i], inv1, acc[48 + i]);
          }
        }
        if (!ok) break;

        if (kUp) {
          // h = silu(G) * U for this thread's 32 channels of the sub-tile
          float amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float h = silu(acc[i]) * acc[32 + i];
            acc[i] = h;
            amax = fmaxf(amax, fabsf(h));
          }
          if (sub == 0) {
            // keep this half until the other half of the 128-channel tile is done
#pragma unroll
            for (int j = 0; j < 8; ++j)
              reinterpret_cast<float4*>(my_hold)[j] =
                  make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            held_amax = amax;
            continue;
          }
          // 1x128 re-quantisation: the tile amax needs both halves of this
          // thread's channels and the other epilogue group's share of the row
          amax = fmaxf(amax, held_amax);
          const int par = unit_count & 1;
          sh.amax[par][eg][row] = amax;
          mbar_arrive(smem_u32(&sh.xchg));
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.xchg), xchg_phase, abort, p.status));
          if (!ok) break;
          xchg_phase ^= 1u;
          amax = fmaxf(sh.amax[par][0][row], sh.amax[par][1][row]);
          const float s = tile_scale(amax);
          if (live) {
            // channels 128n + 32eg + j (sub-tile 0) and 128n + 64 + 32eg + j (sub-tile 1)
            uint8_t* dst = p.h_q + grow * p.I + n * kBM + 32 * eg;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              float hv[16];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 v = reinterpret_cast<const float4*>(my_hold)[4 * j + q];
                hv[4 * q] = v.x;
                hv[4 * q + 1] = v.y;
                hv[4 * q + 2] = v.z;
                hv[4 * q + 3] = v.w;
              }
              reinterpret_cast<uint4*>(dst)[j] = quant16(hv, s);
              reinterpret_cast<uint4*>(dst + 64)[j] = quant16(acc + 16 * j, s);
            }
            if (eg == 0) p.h_s[grow * (p.I / kBM) + n] = s;
          }
        } else {
          if (live) {
            float4* dst = reinterpret_cast<float4*>(p.y + grow * p.H + n * kBN + 64 * eg);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              dst[j] = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemBufs * kBN);
}

template <bool kUp>
cudaError_t launch(const GemmArgs& a, const CUtensorMap& ma, const CUtensorMap& mb,
                   cudaStream_t stream, int sm_count, int64_t unit_bound) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kUp>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<kUp>::kDynSmem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  int grid = sm_count;
  if (unit_bound < grid) grid = (int)(unit_bound > 0 ? unit_bound : 1);
  grouped_gemm_kernel<kUp><<<grid, kThreads, Cfg<kUp>::kDynSmem, stream>>>(ma, mb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_expert_up(const GroupedGemm& gg, const uint8_t* a_q, const float* a_s,
                             const uint8_t* w13, const float* s13, uint8_t* h_q, float* h_s,
                             cudaStream_t stream, int sm_count) {
  CUtensorMap ma, mb;
  cudaError_t e = make_tmap_u8(&ma, a_q, gg.H, gg.rows, kBK, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, w13, gg.H, (int64_t)gg.n_groups * 2 * gg.I, kBK, kBN);
  if (e != cudaSuccess) return e;
  GemmArgs a{};
  a.group_rows = gg.group_rows;
  a.group_start = gg.group_start;
  a.n_groups = gg.n_groups;
  a.kblocks = gg.H / kBK;
  a.n_units = gg.I / kBM;
  a.b_rows = 2 * gg.I;
  a.rows = gg.rows;
  a.a_s = a_s;
  a.b_s = s13;
  a.h_q = h_q;
  a.h_s = h_s;
  a.I = gg.I;
  a.H = gg.H;
  a.status = gg.status;
  const int64_t bound = (gg.rows / kBM + gg.n_groups) * (int64_t)a.n_units;
  return launch<true>(a, ma, mb, stream, sm_count, bound);
}

cudaError_t launch_expert_down(const GroupedGemm& gg, const uint8_t* h_q, const float* h_s,
                               const uint8_t* w2, const float* s2, float* y,
                               cudaStream_t stream, int sm_count) {
  CUtensorMap ma, mb;
  cudaError_t e = make_tmap_u8(&ma, h_q, gg.I, gg.rows, kBK, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, w2, gg.I, (int64_t)gg.n_groups * gg.H, kBK, kBN);
  if (e != cudaSuccess) return e;
  GemmArgs a{};
  a.group_rows = gg.group_rows;
  a.group_start = gg.group_start;
  a.n_groups = gg.n_groups;
  a.kblocks = gg.I / kBK;
  a.n_units = gg.H / kBN;
  a.b_rows = gg.H;
  a.rows = gg.rows;
  a.a_s = h_s;
  a.b_s = s2;
  a.y = y;
  a.I = gg.I;
  a.H = gg.H;
  a.status = gg.status;
  const int64_t bound = (gg.rows / kBM + gg.n_groups) * (int64_t)a.n_units;
  return launch<false>(a, ma, mb, stream, sm_count, bound);
}

}  // namespace moe
