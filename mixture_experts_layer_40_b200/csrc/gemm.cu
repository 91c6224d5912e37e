// Grouped FP8 E4M3 expert GEMMs on tcgen05 tensor cores (sm_100a).
//
// Numerics follow "DeepSeek-V3: Auxiliary-Loss-Free MoE Load Balancing,
// Multi-Token Prediction, and FP8 Training at 671B Scale" (trishampatil.com),
// section V "Four details", items 1-2: E4M3 operands with one scale per 1x128
// activation tile and per 128x128 weight block, and partial sums promoted to
// fp32 every N_C = 128 products. The pages' H800 design promotes on CUDA cores
// while a second WGMMA group computes; here every 128-deep k-block is
// accumulated by the tensor core into its own TMEM buffer (two buffers, ping-
// pong) and eight epilogue warps read it back with tcgen05.ld and add
// partial * 1/(s_a s_b) into fp32 register totals (packed in pairs, two-lane
// FMAs) while the tensor core fills the other buffer.
//
// One persistent CTA per SM, 384 threads (three warpgroups):
//   warp 0     TMA producer: A (128 rows x 128 B) and B (256 rows x 128 B)
//              k-block tiles into a 4-stage shared-memory ring
//   warp 1     TMEM allocator and MMA issuer (one thread): 4 MMAs of
//              M=128, N=256, K=32 per k-block into TMEM buffer (k-block & 1)
//   warps 2-3  idle (they only complete the first warpgroup)
//   warps 4-11 promotion + epilogue; warp w reads TMEM lanes 32*(w%4)..+31,
//              so each warpgroup covers the 128 rows of a tile and owns half
//              of its 256 columns
// The first warpgroup gives registers back (setmaxnreg) so that each epilogue
// thread can hold 128 fp32 totals plus a 64-column partial chunk.
// Tiles are (group, m-tile, n-tile) with n fastest: the n-tiles of one row
// tile run on neighbouring CTAs at the same time and share its A rows in L2.
// A group's last row tile with at most 64 rows runs M=64 MMAs (half the
// tensor-core work on padding rows); its rows sit in TMEM lanes 0-15 of each
// 32-lane sub-partition, and those tiles' rows are stored one by one.
// Both operands load with the default L2 policy: with the weight stream
// marked evict-first (and A evict-last) the HBM reads matched one full read
// of an expert's weights per row tile, i.e. the expert's second row tile
// never found them in L2, and the kernel was slower. Every wait is bounded; a time-out raises the status word and
// the CTA drains its in-flight copies and MMAs before releasing TMEM.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 128;
constexpr int kMaxStages = 4;
constexpr int kABytes = kBM * kBK;
constexpr int kBBytes = kBN * kBK;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 384;
constexpr int kEpiThreads = 256;
constexpr int kMaxGroups = 1025;
constexpr uint32_t kIdesc = make_idesc(kBM, kBN, 0u, 0u);  // E4M3 x E4M3 -> fp32
// a group's last row tile with at most 64 rows: M=64 MMAs, whose rows land in
// TMEM lanes (r mod 16) + 32 (r / 16), i.e. lanes 0-15 of each sub-partition
constexpr uint32_t kIdesc64 = make_idesc(kBM / 2, kBN, 0u, 0u);
// down epilogue: each epilogue warp stages 32 rows x kYCols fp32 columns of
// its output tile in shared memory (swizzled over the 128-byte box row), two
// buffers so that one TMA store is in flight while the next chunk is written
#ifndef MOE_YCOLS
#define MOE_YCOLS 32
#endif
#ifndef MOE_DOWN_STAGES
#define MOE_DOWN_STAGES 3
#endif
constexpr int kYCols = MOE_YCOLS;
constexpr int kYBufBytes = 32 * kYCols * 4;
// What the epilogue makes of a finished tile:
//   kEpiUp    SwiGLU of the gate/up halves, then the 1x128 E4M3 requant of h
//   kEpiF32   fp32 rows (the backward's GEMMs, and the stage entry point that
//             pins the accumulation against float64)
//   kEpiBf16  bf16 rows, rounded once from the fp32 totals (the layer's
//             expert outputs)
enum Epi : int { kEpiUp = 0, kEpiF32 = 1, kEpiBf16 = 2 };
// the up GEMM (56 k-blocks per tile at H = 7168) keeps a 4-stage ring; the
// down GEMMs give one stage to the output staging buffers
template <int kEpi>
struct Cfg {
  static constexpr bool up = kEpi == kEpiUp;
  static constexpr int stages = up ? kMaxStages : MOE_DOWN_STAGES;
  static constexpr size_t dyn_smem =
      (size_t)stages * kStageBytes + (up ? 0 : 8 * 2 * kYBufBytes) + 1024;
};
static_assert(Cfg<kEpiF32>::dyn_smem + 8192 <= 232448, "shared memory");
// Register split: launched at kLaunchRegs per thread (384 x 168 = 64512);
// warpgroup 0 drops to kRegsCtl, the two epilogue warpgroups rise to kRegsEpi.
// 128 * kRegsCtl + 256 * kRegsEpi must not exceed 384 * kLaunchRegs.
constexpr int kLaunchRegs = 168;
constexpr int kRegsCtl = 40;
constexpr int kRegsEpi = 232;
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
  float* y;               // kEpiF32: [rows, H] fp32
  __nv_bfloat16* yb;      // kEpiBf16: [rows, H] bf16
  int32_t H;
  uint32_t* status;
};

struct alignas(8) GemmShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t xchg;           // amax exchange between the two epilogue groups
  uint32_t tmem_base;
  int abort;
  int prefix[kMaxGroups + 1];
  float amax[2][2][kBM];   // [tile parity][epilogue group][row]
  int stage_m64[kMaxStages];  // the producer's flag for the MMA: a 64-row tile
};

MOE_DEV void decode_tile(int tile, const int* prefix, int n_groups, int n_tiles, int& g, int& n,
                         int& m) {
  int lo = 0, hi = n_groups;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] * n_tiles <= tile) lo = mid; else hi = mid;
  }
  g = lo;
  const int local = tile - prefix[g] * n_tiles;
  m = local / n_tiles;
  n = local - m * n_tiles;
}

// silu(a) = a * sigmoid(a) with the hardware exp2 and reciprocal (a few ulp;
// the accurate library forms made the up GEMM's tile epilogue 6x longer).
// For a < -88, exp(-a) is +inf and the quotient is -0.
MOE_DEV float silu(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_y, const GemmArgs p) {
  constexpr bool kUp = kEpi == kEpiUp;
  constexpr int kSt = Cfg<kEpi>::stages;
  __shared__ GemmShared sh;
  extern __shared__ uint8_t dyn_smem[];
  const uint32_t ring = (smem_u32(dyn_smem) + 1023u) & ~1023u;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      mbar_init(smem_u32(&sh.empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
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
    if (!kUp) prefetch_tensormap(&tm_y);
  }
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), 512);
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
  const int total_tiles = sh.prefix[p.n_groups] * p.n_tiles;
  const int kb_n = p.kblocks;
  volatile int* abort = &sh.abort;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
  }
  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        int g, n, m;
        decode_tile(tile, sh.prefix, p.n_groups, p.n_tiles, g, n, m);
        const int a_row = p.group_start[g] + m * kBM;
        const int b_row = g * p.b_rows + n * kBN;
        const int m64 = (p.group_rows[g] - m * kBM) <= kBM / 2 ? 1 : 0;
        for (int kb = 0; kb < kb_n; ++kb, ++it) {
          const int s = it % kSt;
          const uint32_t ph = (uint32_t)(it / kSt) & 1u;
          if (!mbar_wait(smem_u32(&sh.empty[s]), ph ^ 1u, abort, p.status)) { ok = false; break; }
          sh.stage_m64[s] = m64;  // ordered before the MMA's read by the full barrier
          const uint32_t full = smem_u32(&sh.full[s]);
          mbar_arrive_expect_tx(full, kStageBytes);
          const uint32_t sa = ring + s * kStageBytes;
          tma_load_2d(sa, &tm_a, kb * kBK, a_row, full);
          tma_load_2d(sa + kABytes, &tm_b, kb * kBK, b_row, full);
        }
      }
      if (!ok) {
        // drain: every armed stage must land before the CTA may exit
        for (int s = 0; s < kSt && s < it; ++s) {
          const int last = s + ((it - 1 - s) / kSt) * kSt;
          mbar_wait(smem_u32(&sh.full[s]), (uint32_t)(last / kSt) & 1u, nullptr, p.status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int it = 0, kbi = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
        for (int kb = 0; kb < kb_n; ++kb, ++it, ++kbi) {
          const int buf = kbi & 1;
          const uint32_t use = (uint32_t)(kbi >> 1);
          if (!mbar_wait(smem_u32(&sh.tempty[buf]), (use & 1u) ^ 1u, abort, p.status)) { ok = false; break; }
          tc_fence_after();
          const int s = it % kSt;
          const uint32_t ph = (uint32_t)(it / kSt) & 1u;
          if (!mbar_wait(smem_u32(&sh.full[s]), ph, abort, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = ring + s * kStageBytes;
          const uint32_t d = tmem_base + (uint32_t)(buf * kBN);
          const uint64_t da = smem_desc_sw128(sa), db = smem_desc_sw128(sa + kABytes);
          const uint32_t idesc = *reinterpret_cast<volatile int*>(&sh.stage_m64[s]) ? kIdesc64 : kIdesc;
#pragma unroll
          for (int k4 = 0; k4 < kBK / 32; ++k4) {
            // +32 bytes along K = +2 in the descriptor's 16-byte address field
            mma_f8(d, da + (uint64_t)(2 * k4), db + (uint64_t)(2 * k4), idesc, k4 > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&sh.tfull[buf]));
          mma_commit(smem_u32(&sh.empty[s]));
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
    const uint32_t ybuf = ring + (uint32_t)(kSt * kStageBytes + ew * 2 * kYBufBytes);
    const int b_blocks = p.b_rows / kBM;
    int kbi = 0;
    uint32_t xchg_phase = 0;
    int tile_count = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++tile_count) {
      uint64_t acc2[64];  // the 128 fp32 totals as packed pairs
      int g, n, m;
      decode_tile(tile, sh.prefix, p.n_groups, p.n_tiles, g, n, m);
      const int valid_rows = p.group_rows[g] - m * kBM;
      // a 64-row tile: lanes 0-15 of each sub-partition hold rows 16q + lane
      const bool m64 = valid_rows <= kBM / 2;
      const int r_in = m64 ? (lane < 16 ? 16 * quarter + lane : kBM) : row;
      const int valid = m64 ? 0 : valid_rows;  // 64-row tiles store row by row
      const int64_t grow = (int64_t)p.group_start[g] + m * kBM + r_in;
      const bool live = r_in < valid_rows;
      const float* sa_ptr = p.a_s + (live ? grow : 0) * kb_n;
      const float* sb0 = p.b_s + ((int64_t)g * b_blocks + 2 * n + (kUp ? 0 : eg)) * kb_n;
      const float* sb1 = p.b_s + ((int64_t)g * b_blocks + 2 * n + 1) * kb_n;
#pragma unroll
      for (int i = 0; i < 64; ++i) acc2[i] = 0ull;
      float sa_next = ldg_early(sa_ptr);
      float sb0_next = ldg_early(sb0);
      float sb1_next = kUp ? ldg_early(sb1) : 0.0f;
      bool ok = true;
      for (int kb = 0; kb < kb_n; ++kb, ++kbi) {
        const float sa = sa_next, s0 = sb0_next, s1 = sb1_next;
        if (kb + 1 < kb_n) {
          sa_next = ldg_early(sa_ptr + kb + 1);
          sb0_next = ldg_early(sb0 + kb + 1);
          if (kUp) sb1_next = ldg_early(sb1 + kb + 1);
        }
        // 1/(s_a s_b) with the hardware reciprocal (<= 2 ulp)
        const float inv0 = __fdividef(1.0f, sa * s0);
        const float inv1 = kUp ? __fdividef(1.0f, sa * s1) : inv0;
        const uint64_t inv0x2 = splat_f32x2(inv0), inv1x2 = splat_f32x2(inv1);
        const int buf = kbi & 1;
        // the result is made warp-uniform: tcgen05.ld below is warp-collective
        ok = __all_sync(0xffffffffu,
                        mbar_wait(smem_u32(&sh.tfull[buf]), (uint32_t)(kbi >> 1) & 1u, abort, p.status));
        if (!ok) break;
        tc_fence_after();
        const uint32_t t0 = lane_addr + (uint32_t)(buf * kBN);
        // columns owned by this thread: up -> gate [64eg, 64eg+64) and up
        // [128+64eg, ...); down -> [128eg, 128eg+128)
        const uint32_t c0 = kUp ? (uint32_t)(64 * eg) : (uint32_t)(128 * eg);
        const uint32_t c2 = kUp ? (uint32_t)(128 + 64 * eg) : (uint32_t)(128 * eg + 64);
        float v[64];
        tmem_ld64(t0 + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 64; i += 2) fma_f32x2(acc2[i / 2], v[i], v[i + 1], inv0x2);
        tmem_ld64(t0 + c2, v);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sh.tempty[buf]));
#pragma unroll
        for (int i = 0; i < 64; i += 2) fma_f32x2(acc2[32 + i / 2], v[i], v[i + 1], inv1x2);
      }
      if (!ok) break;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 64; ++i) unpack_f32x2(acc2[i], acc[2 * i], acc[2 * i + 1]);

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
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&sh.xchg), xchg_phase, abort, p.status))) break;
        xchg_phase ^= 1u;
        amax = fmaxf(sh.amax[par][0][row], sh.amax[par][1][row]);
        const float s = tile_scale(amax);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(p.h_q + grow * p.I + n * kBM + 64 * eg);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 o;
            o.x = e4m3x4(__fmul_rn(acc[16 * j + 0], s), __fmul_rn(acc[16 * j + 1], s),
                         __fmul_rn(acc[16 * j + 2], s), __fmul_rn(acc[16 * j + 3], s));
            o.y = e4m3x4(__fmul_rn(acc[16 * j + 4], s), __fmul_rn(acc[16 * j + 5], s),
                         __fmul_rn(acc[16 * j + 6], s), __fmul_rn(acc[16 * j + 7], s));
            o.z = e4m3x4(__fmul_rn(acc[16 * j + 8], s), __fmul_rn(acc[16 * j + 9], s),
                         __fmul_rn(acc[16 * j + 10], s), __fmul_rn(acc[16 * j + 11], s));
            o.w = e4m3x4(__fmul_rn(acc[16 * j + 12], s), __fmul_rn(acc[16 * j + 13], s),
                         __fmul_rn(acc[16 * j + 14], s), __fmul_rn(acc[16 * j + 15], s));
            dst[j] = o;
          }
          if (eg == 0) p.h_s[grow * (p.I / kBM) + n] = s;
        }
      } else if (kEpi == kEpiBf16) {
        // bf16 rows (one rounding of the fp32 totals) out through shared
        // memory and TMA stores, 64 columns (128 bytes) of the warp's 32 rows
        // at a time, when all 32 rows belong to the group; a group's last,
        // partial 32 rows are stored directly, row by row, and padding rows
        // are never written
        const int q_live = valid - quarter * 32;
        const int y0 = p.group_start[g] + m * kBM + quarter * 32;
        const int x0 = n * kBN + 128 * eg;
        const uint32_t swz = (uint32_t)(lane & 7);
        if (q_live < 32) {
          if (live) {
            uint4* dst = reinterpret_cast<uint4*>(p.yb + grow * p.H + x0);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              dst[j] = make_uint4(pack_bf16x2(acc[8 * j + 0], acc[8 * j + 1]),
                                  pack_bf16x2(acc[8 * j + 2], acc[8 * j + 3]),
                                  pack_bf16x2(acc[8 * j + 4], acc[8 * j + 5]),
                                  pack_bf16x2(acc[8 * j + 6], acc[8 * j + 7]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const uint32_t buf_j = ybuf + (uint32_t)(j * kYBufBytes);
            // the store that last read this buffer (two chunks ago) is done
            if (lane == 0) bulk_wait_read_1();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint32_t dst = buf_j + (uint32_t)lane * 128u + (((uint32_t)c ^ swz) << 4);
              const int a0 = 64 * j + 8 * c;
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst),
                           "r"(pack_bf16x2(acc[a0 + 0], acc[a0 + 1])),
                           "r"(pack_bf16x2(acc[a0 + 2], acc[a0 + 3])),
                           "r"(pack_bf16x2(acc[a0 + 4], acc[a0 + 5])),
                           "r"(pack_bf16x2(acc[a0 + 6], acc[a0 + 7]))
                           : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tm_y, buf_j, x0 + 64 * j, y0);
              bulk_commit();
            }
          }
        }
      } else {
        // fp32 rows out through shared memory and TMA stores, 8 columns of
        // the warp's 32 rows at a time, when all 32 rows belong to the group;
        // a group's last, partial 32 rows are stored directly, row by row,
        // and padding rows are never written
        const int q_live = valid - quarter * 32;
        const int y0 = p.group_start[g] + m * kBM + quarter * 32;
        const int x0 = n * kBN + 128 * eg;
        // 128-byte-span swizzle: 16-byte chunk c of row r sits at c ^ (r / rows
        // per 128 bytes) within the row (32-, 64- and 128-byte modes alike)
        constexpr int kChunks = kYCols / 4;
        const uint32_t swz = (uint32_t)((lane / (32 / kYCols)) & (kChunks - 1));
        if (q_live < 32) {
          if (live) {
            float4* dst = reinterpret_cast<float4*>(p.y + grow * p.H + x0);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              dst[j] = make_float4(acc[4 * j + 0], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
          }
        } else {
#pragma unroll
        for (int j = 0; j < 128 / kYCols; ++j) {
          const uint32_t buf_j = ybuf + (uint32_t)((j & 1) * kYBufBytes);
          // the store that last read this buffer (two chunks ago) is done
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
            tma_store_2d(&tm_y, buf_j, x0 + kYCols * j, y0);
            bulk_commit();
          }
        }
        }
      }
    }
    if (!kUp && lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

template <int kEpi>
cudaError_t launch(const GemmArgs& a, const CUtensorMap& ma, const CUtensorMap& mb,
                   const CUtensorMap& my,
                   cudaStream_t stream, int sm_count, int64_t tile_bound) {
  // once per device: the register split above is only safe if the kernel
  // really was built with kLaunchRegs registers per thread, and the large
  // dynamic shared memory must be allowed on each device the kernel runs on
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, grouped_gemm_kernel<kEpi>);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(grouped_gemm_kernel<kEpi>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)Cfg<kEpi>::dyn_smem);
  });
  if (e != cudaSuccess) return e;
  int grid = sm_count;
  if (tile_bound < grid) grid = (int)(tile_bound > 0 ? tile_bound : 1);
  grouped_gemm_kernel<kEpi><<<grid, kThreads, Cfg<kEpi>::dyn_smem, stream>>>(ma, mb, my, a);
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
  const int64_t bound = (gg.rows / kBM + gg.n_groups) * (int64_t)a.n_tiles;
  return launch<kEpiUp>(a, ma, mb, ma, stream, sm_count, bound);
}

namespace {

GemmArgs down_args(const GroupedGemm& gg, const float* h_s, const float* s2) {
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
  a.I = gg.I;
  a.H = gg.H;
  a.status = gg.status;
  return a;
}

}  // namespace

cudaError_t launch_expert_down(const GroupedGemm& gg, const uint8_t* h_q, const float* h_s,
                               const uint8_t* w2, const float* s2, float* y,
                               cudaStream_t stream, int sm_count) {
  CUtensorMap ma, mb, my;
  cudaError_t e = make_tmap_u8(&ma, h_q, gg.I, gg.rows, kBK, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, w2, gg.I, (int64_t)gg.n_groups * gg.H, kBK, kBN);
  if (e != cudaSuccess) return e;
  e = make_tmap_f32(&my, y, gg.H, gg.rows, kYCols, 32);
  if (e != cudaSuccess) return e;
  GemmArgs a = down_args(gg, h_s, s2);
  a.y = y;
  const int64_t bound = (gg.rows / kBM + gg.n_groups) * (int64_t)a.n_tiles;
  return launch<kEpiF32>(a, ma, mb, my, stream, sm_count, bound);
}

cudaError_t launch_expert_down_bf16(const GroupedGemm& gg, const uint8_t* h_q, const float* h_s,
                                    const uint8_t* w2, const float* s2, __nv_bfloat16* y,
                                    cudaStream_t stream, int sm_count) {
  CUtensorMap ma, mb, my;
  cudaError_t e = make_tmap_u8(&ma, h_q, gg.I, gg.rows, kBK, kBM);
  if (e != cudaSuccess) return e;
  e = make_tmap_u8(&mb, w2, gg.I, (int64_t)gg.n_groups * gg.H, kBK, kBN);
  if (e != cudaSuccess) return e;
  e = make_tmap_bf16(&my, y, gg.H, gg.rows, 1, 64, 32);
  if (e != cudaSuccess) return e;
  GemmArgs a = down_args(gg, h_s, s2);
  a.yb = y;
  const int64_t bound = (gg.rows / kBM + gg.n_groups) * (int64_t)a.n_tiles;
  return launch<kEpiBf16>(a, ma, mb, my, stream, sm_count, bound);
}

}  // namespace moe
