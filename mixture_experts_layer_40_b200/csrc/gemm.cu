// Grouped FP8 E4M3 expert GEMMs on tcgen05 tensor cores (sm_100a), issued
// as 2-SM pair MMAs (cta_group::2).
//
// Numerics follow "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
// Multi-Token Prediction, and FP8 Training at 671B Scale" (trishampatil.com),
// section V "Four details", items 1-2: E4M3 operands with one scale per 1x128
// activation tile and per 128x128 weight block, and partial sums promoted to
// fp32 every N_C = 128 products. The pages' H800 design promotes on CUDA cores
// while a second WGMMA group computes. Here every 128-deep k-block is summed
// by the tensor core into its own TMEM buffer (two buffers, ping-pong) and
// eight promotion warps per SM read it back with tcgen05.ld and add
// partial * 1/(s_a s_b) into fp32 register totals while the tensor core fills
// the other buffer.
//
// A cluster of two CTAs (two SMs) computes one 256-row x 256-column tile:
// each CTA loads its 128 rows of A and its 128 rows (half the columns) of B
// into its own shared memory, the even CTA issues the pair MMA (M=256, N=256,
// K=32) that reads both halves, and each CTA's TMEM receives the 128 x 256
// accumulator of its own rows. Against a one-SM 128 x 256 tile this halves the
// weight bytes every SM loads and reads per MMA, which is what bounds the
// one-SM version (shared-memory and L2 traffic, not the tensor core).
//
// Per CTA, 384 threads (three warpgroups):
//   warp 0     TMA producer for this CTA's halves; the completion of both
//              CTAs' loads is counted on the even CTA's stage barrier
//   warp 1     TMEM allocator (pair allocation) and, in the even CTA, the MMA
//              issuer; the MMA commits arrive on both CTAs' barriers
//   warps 2-3  idle (they only complete the first warpgroup)
//   warps 4-11 promotion + epilogue on this CTA's 128 rows; warp w reads TMEM
//              lanes 32*(w%4)..+31; each warpgroup owns half of the 256 columns
// The first warpgroup gives registers back (setmaxnreg) so that each epilogue
// thread can hold 128 fp32 totals plus two 16-column chunks in flight.
// Work units are (group, n-tile, m-tile) with m fastest, so the m-tiles of one
// expert's weight tile run back to back and the weight tile is read from HBM
// about once. Every wait is bounded; a time-out raises the status word, and
// the CTAs drain their in-flight copies and MMAs before TMEM is released.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kBMc = 128;       // rows per CTA
constexpr int kBMp = 256;       // rows per pair tile
constexpr int kBN = 256;        // columns per tile
constexpr int kBNc = kBN / 2;   // B rows held by each CTA
constexpr int kBK = 128;
constexpr int kStages = 6;
constexpr int kABytes = kBMc * kBK;
constexpr int kBBytes = kBNc * kBK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 384;
constexpr int kEpiWarps = 8;
constexpr int kMaxGroups = 1025;
constexpr uint32_t kIdesc = make_idesc(kBMp, kBN, 0u, 0u);  // E4M3 x E4M3 -> fp32
constexpr size_t kDynSmem = (size_t)kStages * kStageBytes + 1024;
// Register split: launched at kLaunchRegs per thread (384 x 168 = 64512);
// warpgroup 0 drops to kRegsCtl, the two epilogue warpgroups rise to kRegsEpi.
constexpr int kLaunchRegs = 168;
constexpr int kRegsCtl = 64;
constexpr int kRegsEpi = 216;
static_assert(128 * kRegsCtl + 256 * kRegsEpi <= kThreads * kLaunchRegs, "register split");

struct GemmArgs {
  const int32_t* group_rows;
  const int32_t* group_start;
  int32_t n_groups;
  int32_t kblocks;        // reduction depth / 128
  int32_t n_tiles;        // 256-wide output tiles per group
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

struct alignas(8) GemmShared {
  uint64_t full[kStages];   // even CTA: both CTAs' bytes of a stage have landed
  uint64_t empty[kStages];  // the pair MMA has consumed a stage (both CTAs)
  uint64_t tfull[2];        // a TMEM buffer holds a finished k-block (both CTAs)
  uint64_t tempty[2];       // even CTA: both CTAs have read a TMEM buffer
  uint64_t xchg;            // amax exchange between the two epilogue groups
  uint32_t tmem_base;
  int abort;
  int prefix[kMaxGroups + 1];
  float amax[2][2][kBMc];   // [tile parity][epilogue group][row]
};

MOE_DEV void decode_tile(int tile, const int* prefix, int n_groups, int n_tiles, int& g, int& n,
                         int& m) {
  int lo = 0, hi = n_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] * n_tiles <= tile) lo = mid; else hi = mid;
  }
  g = lo;
  const int mt = prefix[g + 1] - prefix[g];
  const int local = tile - prefix[g] * n_tiles;
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
  __shared__ GemmShared sh;
  extern __shared__ uint8_t dyn_smem[];
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();   // 0: even CTA (issues the MMAs), 1: odd
  const int pair = (int)cluster_id_x();
  const int n_pairs = (int)cluster_count_x();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      mbar_init(smem_u32(&sh.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sh.tfull[b]), 1);
      mbar_init(smem_u32(&sh.tempty[b]), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(&sh.xchg), kEpiWarps * 32);
    sh.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == 1) tmem_alloc_pair(smem_u32(&sh.tmem_base), 512);
  if (warp == 2) {
    // pair-tile (256-row) prefix over the groups; a group whose rows fall
    // outside the buffers or whose start is not 128-aligned is flagged and skipped
    int carry = 0;
    if (lane == 0) sh.prefix[0] = 0;
    for (int base = 0; base < p.n_groups; base += 32) {
      const int g = base + lane;
      int mt = 0;
      if (g < p.n_groups) {
        const int r = p.group_rows[g];
        const int st = p.group_start[g];
        const bool ok = r >= 0 && st >= 0 && (st % kBMc) == 0 && (int64_t)st + r <= p.rows;
        if (!ok) flag_status(p.status, kStatusBounds);
        mt = ok ? (r + kBMp - 1) / kBMp : 0;
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
  // both CTAs' barriers are initialised before any cross-CTA arrival
  cluster_sync();
  tc_fence_after();

  const uint32_t tmem_base = sh.tmem_base;
  const int total_tiles = sh.prefix[p.n_groups] * p.n_tiles;
  const int kb_n = p.kblocks;
  volatile int* abort = &sh.abort;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  }
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = policy_evict_first();
      int it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        int g, n, m;
        decode_tile(tile, sh.prefix, p.n_groups, p.n_tiles, g, n, m);
        const int a_row = p.group_start[g] + m * kBMp + (int)rank * kBMc;
        const int b_row = g * p.b_rows + n * kBN + (int)rank * kBNc;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort, p.status)) { ok = false; break; }
          const uint32_t full_even = map_to_rank(smem_u32(&sh.full[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(&sh.full[s]), 2 * kStageBytes);
          const uint32_t sa = ring + s * kStageBytes;
          tma_load_2d_pair(sa, &tm_a, kb * kBK, a_row, full_even, pol_a);
          tma_load_2d_pair(sa + kABytes, &tm_b, kb * kBK, b_row, full_even, pol_b);
        }
      }
      if (!ok && rank == 0) {
        // drain: every armed stage must land before the pair may exit
        for (int s = 0; s < kStages && s < it; ++s) {
          const int last = s + ((it - 1 - s) / kStages) * kStages;
          mbar_wait(smem_u32(&sh.full[s]), (uint32_t)(last / kStages) & 1u, nullptr, p.status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      int it = 0, kbi = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += n_pairs) {
        for (int kb = 0; kb < kb_n; ++kb, ++it, ++kbi) {
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
          for (int k4 = 0; k4 < kBK / 32; ++k4) {
            mma_f8_pair(d, smem_desc_sw128(sa + k4 * 32), smem_desc_sw128(sa + kABytes + k4 * 32),
                        kIdesc, k4 > 0 ? 1u : 0u);
          }
          mma_commit_pair(smem_u32(&sh.empty[s]), (uint16_t)0x3);
          mma_commit_pair(smem_u32(&sh.tfull[buf]), (uint16_t)0x3);
        }
      }
      if (!ok && kbi > 0) {
        const int last = kbi - 1;
        mbar_wait(smem_u32(&sh.tfull[last & 1]), (uint32_t)(last >> 1) & 1u, nullptr, p.status);
      }
    }
  } else if (warp >= 4) {
    // -------------------------------------------------------------- epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsEpi));
    const int ew = warp - 4;
    const int eg = ew >> 2;            // epilogue group 0 / 1
    const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    const int b_blocks = p.b_rows / kBMc;
    // columns owned by this thread: up -> gate [64eg, 64eg+64) and up
    // [128+64eg, ...); down -> [128eg, 128eg+128)
    const uint32_t c0 = kUp ? (uint32_t)(64 * eg) : (uint32_t)(128 * eg);
    const uint32_t c2 = kUp ? (uint32_t)(128 + 64 * eg) : (uint32_t)(128 * eg + 64);
    const uint32_t tempty_even0 = map_to_rank(smem_u32(&sh.tempty[0]), 0);
    const uint32_t tempty_even1 = map_to_rank(smem_u32(&sh.tempty[1]), 0);
    int kbi = 0;
    uint32_t xchg_phase = 0;
    int tile_count = 0;
    bool ok = true;
    float acc[128];
    for (int tile = pair; ok && tile < total_tiles; tile += n_pairs, ++tile_count) {
      int g, n, m;
      decode_tile(tile, sh.prefix, p.n_groups, p.n_tiles, g, n, m);
      const int row0 = m * kBMp + (int)rank * kBMc;   // first row of this CTA inside the group
      const int valid = p.group_rows[g] - row0;
      const int64_t grow = (int64_t)p.group_start[g] + row0 + row;
      const bool live = row < valid;
      const float* sa_ptr = p.a_s + (live ? grow : 0) * kb_n;
      const float* sb0 = p.b_s + ((int64_t)g * b_blocks + 2 * n + (kUp ? 0 : eg)) * kb_n;
      const float* sb1 = p.b_s + ((int64_t)g * b_blocks + 2 * n + 1) * kb_n;
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
      float sa_next = __ldg(sa_ptr);
      float sb0_next = __ldg(sb0);
      float sb1_next = kUp ? __ldg(sb1) : 0.0f;
      for (int kb = 0; kb < kb_n; ++kb, ++kbi) {
        const float sa = sa_next, s0 = sb0_next, s1 = sb1_next;
        if (kb + 1 < kb_n) {
          sa_next = __ldg(sa_ptr + kb + 1);
          sb0_next = __ldg(sb0 + kb + 1);
          if (kUp) sb1_next = __ldg(sb1 + kb + 1);
        }
        const float inv0 = __frcp_rn(sa * s0);
        const float inv1 = kUp ? __frcp_rn(sa * s1) : inv0;
        const int buf = kbi & 1;
        // the result is made warp-uniform: tcgen05.ld below is warp-collective
        ok = __all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&sh.tfull[buf]), (uint32_t)(kbi >> 1) & 1u, abort, p.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t t0 = lane_addr + (uint32_t)(buf * kBN);
        // four pairs of 16-column chunks; the next pair is in flight while the
        // current one is folded into the totals
        float pa[16], pb[16], qa[16], qb[16];
        tmem_ld16(t0 + c0, pa);
        tmem_ld16(t0 + c0 + 16, pb);
        tmem_wait_ld_tied(pa, pb);
        tmem_ld16(t0 + c0 + 32, qa);
        tmem_ld16(t0 + c0 + 48, qb);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          acc[i] = fmaf(pa[i], inv0, acc[i]);
          acc[16 + i] = fmaf(pb[i], inv0, acc[16 + i]);
        }
        tmem_wait_ld_tied(qa, qb);
        tmem_ld16(t0 + c2, pa);
        tmem_ld16(t0 + c2 + 16, pb);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          acc[32 + i] = fmaf(qa[i], inv0, acc[32 + i]);
          acc[48 + i] = fmaf(qb[i], inv0, acc[48 + i]);
        }
        tmem_wait_ld_tied(pa, pb);
        tmem_ld16(t0 + c2 + 32, qa);
        tmem_ld16(t0 + c2 + 48, qb);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          acc[64 + i] = fmaf(pa[i], inv1, acc[64 + i]);
          acc[80 + i] = fmaf(pb[i], inv1, acc[80 + i]);
        }
        tmem_wait_ld_tied(qa, qb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(buf ? tempty_even1 : tempty_even0);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          acc[96 + i] = fmaf(qa[i], inv1, acc[96 + i]);
          acc[112 + i] = fmaf(qb[i], inv1, acc[112 + i]);
        }
      }
      if (!ok) break;

      if (kUp) {
        // h = silu(G) * U for this thread's 64 channels, then 1x128 re-quantisation;
        // the tile amax needs the other group's half of the row
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float h = silu(acc[i]) * acc[64 + i];
          acc[i] = h;
          amax = fmaxf(amax, fabsf(h));
        }
        const int par = tile_count & 1;
        sh.amax[par][eg][row] = amax;
        mbar_arrive(smem_u32(&sh.xchg));
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.xchg), xchg_phase, abort, p.status));
        if (!ok) break;
        xchg_phase ^= 1u;
        amax = fmaxf(sh.amax[par][0][row], sh.amax[par][1][row]);
        const float s = tile_scale(amax);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(p.h_q + grow * p.I + n * kBMc + 64 * eg);
#pragma unroll
          for (int j = 0; j < 4; ++j) dst[j] = quant16(acc + 16 * j, s);
          if (eg == 0) p.h_s[grow * (p.I / kBMc) + n] = s;
        }
      } else {
        if (live) {
          float4* dst = reinterpret_cast<float4*>(p.y + grow * p.H + n * kBN + 128 * eg);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            dst[j] = make_float4(acc[4 * j + 0], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA releases the pair's TMEM while the other may still use it
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

template <bool kUp>
cudaError_t launch(const GemmArgs& a, const CUtensorMap& ma, const CUtensorMap& mb,
                   cudaStream_t stream, int sm_count, int64_t tile_bound) {
  static int max_pairs = 0;
  if (max_pairs == 0) {
    // the register split above is only safe if the kernel really was built
    // with kLaunchRegs registers per thread
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, grouped_gemm_kernel<kUp>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(grouped_gemm_kernel<kUp>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDynSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t probe = {};
    probe.gridDim = dim3((unsigned)(sm_count / 2 * 2));
    probe.blockDim = dim3(kThreads);
    probe.dynamicSmemBytes = kDynSmem;
    cudaLaunchAttribute cl;
    cl.id = cudaLaunchAttributeClusterDimension;
    cl.val.clusterDim.x = 2;
    cl.val.clusterDim.y = 1;
    cl.val.clusterDim.z = 1;
    probe.attrs = &cl;
    probe.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_kernel<kUp>, &probe);
    if (e != cudaSuccess || clusters < 1) return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
    max_pairs = clusters;
  }
  int pairs = max_pairs;
  if (tile_bound < pairs) pairs = (int)(tile_bound > 0 ? tile_bound : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kDynSmem;
  cfg.stream = stream;
  cudaLaunchAttribute cl;
  cl.id = cudaLaunchAttributeClusterDimension;
  cl.val.clusterDim.x = 2;
  cl.val.clusterDim.y = 1;
  cl.val.clusterDim.z = 1;
  cfg.attrs = &cl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<kUp>, ma, mb, a);
}

}  // namespace

cudaError_t launch_expert_up(const GroupedGemm& gg, const uint8_t* a_q, const float* a_s,
                             const uint8_t* w13, const float* s13, uint8_t* h_q, float* h_s,
                             cudaStream_t stream, int sm_count) {
  CUtensorMap ma, mb;
  cudaError_t e = make_tmap_u8(&ma, a_q, gg.H, gg.rows, kBK, kBMc);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, w13, gg.H, (int64_t)gg.n_groups * 2 * gg.I, kBK, kBNc);
  if (e != cudaSuccess) return e;
  GemmArgs a{};
  a.group_rows = gg.group_rows;
  a.group_start = gg.group_start;
  a.n_groups = gg.n_groups;
  a.kblocks = gg.H / kBK;
  a.n_tiles = 2 * gg.I / kBN;
  a.b_rows = 2 * gg.I;
  a.rows = gg.rows;
  a.a_s = a_s;
  a.b_s = s13;
  a.h_q = h_q;
  a.h_s = h_s;
  a.I = gg.I;
  a.H = gg.H;
  a.status = gg.status;
  const int64_t bound = (gg.rows / kBMp + gg.n_groups) * (int64_t)a.n_tiles;
  return launch<true>(a, ma, mb, stream, sm_count, bound);
}

cudaError_t launch_expert_down(const GroupedGemm& gg, const uint8_t* h_q, const float* h_s,
                               const uint8_t* w2, const float* s2, float* y,
                               cudaStream_t stream, int sm_count) {
  CUtensorMap ma, mb;
  cudaError_t e = make_tmap_u8(&ma, h_q, gg.I, gg.rows, kBK, kBMc);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, w2, gg.I, (int64_t)gg.n_groups * gg.H, kBK, kBNc);
  if (e != cudaSuccess) return e;
  GemmArgs a{};
  a.group_rows = gg.group_rows;
  a.group_start = gg.group_start;
  a.n_groups = gg.n_groups;
  a.kblocks = gg.I / kBK;
  a.n_tiles = gg.H / kBN;
  a.b_rows = gg.H;
  a.rows = gg.rows;
  a.a_s = h_s;
  a.b_s = s2;
  a.y = y;
  a.I = gg.I;
  a.H = gg.H;
  a.status = gg.status;
  const int64_t bound = (gg.rows / kBMp + gg.n_groups) * (int64_t)a.n_tiles;
  return launch<false>(a, ma, mb, stream, sm_count, bound);
}

}  // namespace moe
