// Backward of the expert path in FP8 ("DeepSeek-V3: Auxiliary-Loss-Free MoE
// Load Balancing, Multi-Token Prediction, and FP8 Training at 671B Scale",
// section V, Figure 6: the Dgrad GEMMs of every linear layer in E4M3 with
// fine-grained scales and fp32 accumulation; gating stays in high precision,
// so the router's own backward is left to the caller, who gets the gate
// gradients). The GEMMs are the forward's grouped FP8 kernel with the
// weights' 128x128 blocks transposed; the kernels here are the element-wise
// steps around them:
//   transpose_blocks    set-up: W [rows, cols] -> W^T per group, codes and
//                       block scales (a 128x128 block's scale is its own)
//   dy_rows_quantize    dY rows = g[t,k] dy[t] (routed) and dy[t] (shared),
//                       1x128-quantised into the forward's row order
//   swiglu_backward     dG = dh U silu'(G), dU = dh silu(G) from the
//                       recomputed [G|U] rows, 1x128-quantised in the
//                       gate/up-interleaved order of w13
//   gate_grad           dgates[t,k] = dy[t] . Y[row(t,k)]
#include "kernels.cuh"

namespace moe {

namespace {

// One CTA per 128x128 block of one group. The block comes in with 16-byte
// loads as 32-bit words, each thread transposes 4x4-byte sub-blocks in
// registers (byte permutes), and the transposed block goes out with 16-byte
// stores; both shared-memory arrays are padded to 33 words a row.
__global__ void __launch_bounds__(256) transpose_blocks_kernel(const uint8_t* __restrict__ w,
                                                               const float* __restrict__ s,
                                                               int64_t rows, int64_t cols,
                                                               uint8_t* __restrict__ wt,
                                                               float* __restrict__ st) {
  __shared__ uint32_t tin[kTile][kTile / 4 + 1];
  __shared__ uint32_t tout[kTile][kTile / 4 + 1];
  const int64_t cb = blockIdx.x, rb = blockIdx.y, g = blockIdx.z;
  const uint8_t* src = w + g * rows * cols + rb * kTile * cols + cb * kTile;
  // 128 rows x 8 chunks of 16 bytes
  for (int i = threadIdx.x; i < kTile * 8; i += blockDim.x) {
    const int r = i >> 3, q = i & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (int64_t)r * cols + 16 * q);
    tin[r][4 * q + 0] = v.x;
    tin[r][4 * q + 1] = v.y;
    tin[r][4 * q + 2] = v.z;
    tin[r][4 * q + 3] = v.w;
  }
  __syncthreads();
  // 32 x 32 sub-blocks of 4x4 bytes: word bj of source rows 4bi..4bi+3 becomes
  // word bi of destination rows 4bj..4bj+3
  for (int i = threadIdx.x; i < 32 * 32; i += blockDim.x) {
    const int bi = i >> 5, bj = i & 31;
    const uint32_t a0 = tin[4 * bi + 0][bj], a1 = tin[4 * bi + 1][bj];
    const uint32_t a2 = tin[4 * bi + 2][bj], a3 = tin[4 * bi + 3][bj];
    const uint32_t t0 = __byte_perm(a0, a1, 0x5140), t1 = __byte_perm(a2, a3, 0x5140);
    const uint32_t t2 = __byte_perm(a0, a1, 0x7362), t3 = __byte_perm(a2, a3, 0x7362);
    tout[4 * bj + 0][bi] = __byte_perm(t0, t1, 0x5410);
    tout[4 * bj + 1][bi] = __byte_perm(t0, t1, 0x7632);
    tout[4 * bj + 2][bi] = __byte_perm(t2, t3, 0x5410);
    tout[4 * bj + 3][bi] = __byte_perm(t2, t3, 0x7632);
  }
  __syncthreads();
  uint8_t* dst = wt + g * rows * cols + cb * kTile * rows + rb * kTile;
  for (int i = threadIdx.x; i < kTile * 8; i += blockDim.x) {
    const int r = i >> 3, q = i & 7;  // destination row r (a source column)
    *reinterpret_cast<uint4*>(dst + (int64_t)r * rows + 16 * q) =
        make_uint4(tout[r][4 * q + 0], tout[r][4 * q + 1], tout[r][4 * q + 2], tout[r][4 * q + 3]);
  }
  if (threadIdx.x == 0) {
    const int64_t rbn = rows / kTile, cbn = cols / kTile;
    st[g * rbn * cbn + cb * rbn + rb] = s[g * rbn * cbn + rb * cbn + cb];
  }
}

// 16 threads per 128-column tile of dy[t]; for each of the token's K + 1
// GEMM rows the tile is scaled by that row's gate (1 for the shared row),
// its amax reduced over the 16 threads and the codes written.
__global__ void __launch_bounds__(256) dy_rows_quantize_kernel(
    const uint4* __restrict__ dy, const float* __restrict__ gates, int T, int H, int K,
    const int32_t* __restrict__ token_row, int64_t routed_cap, uint8_t* __restrict__ q,
    float* __restrict__ qs, float* __restrict__ row_gate, uint32_t* __restrict__ status) {
  const int sub = threadIdx.x & 15;
  const int tiles_per_row = H / kTile;
  const int64_t n_tiles = (int64_t)T * tiles_per_row;
  for (int64_t base = (int64_t)blockIdx.x * 16; base < n_tiles; base += (int64_t)gridDim.x * 16) {
    const int64_t tile = base + (threadIdx.x >> 4);
    const bool live = tile < n_tiles;
    const int64_t t = live ? tile / tiles_per_row : 0;
    const int c = live ? (int)(tile - t * tiles_per_row) : 0;
    const uint4 v = live ? __ldg(dy + tile * 16 + sub) : make_uint4(0, 0, 0, 0);
    int my_row = -1;
    float my_gate = 0.0f;
    if (live && sub < K) {
      my_row = __ldg(token_row + t * K + sub);
      my_gate = __ldg(gates + t * K + sub);
    }
    const float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    // the tile's amax of |dy|, once: rounding is monotone, so the amax of the
    // rounded products |fp32(g * dy)| is fp32(|g| * amax |dy|) for every gate
    float amax_f = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax_f = fmaxf(amax_f, fabsf(f[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax_f = fmaxf(amax_f, __shfl_xor_sync(0xffffffffu, amax_f, o));
    for (int k = -1; k < K; ++k) {
      int64_t r = routed_cap + t;
      float g = 1.0f;
      if (k >= 0) {
        r = __shfl_sync(0xffffffffu, my_row, k, 16);
        g = __shfl_sync(0xffffffffu, my_gate, k, 16);
      }
      float d[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = __fmul_rn(g, f[i]);
      const float amax = __fmul_rn(fabsf(g), amax_f);
      if (!live) continue;
      if (k >= 0 && (r < 0 || r >= routed_cap)) {
        if (sub == 0) flag_status(status, kStatusBounds);
        continue;
      }
      const float s = tile_scale(amax);
      uint2 out;
      out.x = e4m3x4(__fmul_rn(d[0], s), __fmul_rn(d[1], s), __fmul_rn(d[2], s), __fmul_rn(d[3], s));
      out.y = e4m3x4(__fmul_rn(d[4], s), __fmul_rn(d[5], s), __fmul_rn(d[6], s), __fmul_rn(d[7], s));
      reinterpret_cast<uint2*>(q + r * H + (int64_t)c * kTile)[sub] = out;
      if (sub == 0) qs[r * tiles_per_row + c] = s;
      if (sub == 0 && c == 0 && row_gate != nullptr) row_gate[r] = g;
    }
  }
}

// 16 threads per (row, 128-channel block c): the block's 128 G and 128 U
// values sit at columns [256c, 256c + 128) and [256c + 128, 256c + 256) of the
// recomputed rows (w13's row order); dG and dU are quantised as two 1x128
// tiles at the same positions of the output rows.
__global__ void __launch_bounds__(256) swiglu_backward_kernel(
    const float* __restrict__ gu, const float* __restrict__ dh, int64_t rows, int I,
    uint8_t* __restrict__ q, float* __restrict__ qs) {
  // two units per thread per round: their six 16-byte loads each are issued
  // before either is used
  constexpr int kU = 2;
  const int sub = threadIdx.x & 15;
  const int blocks = I / kTile;
  const int64_t n_units = rows * blocks;
  const int64_t step = (int64_t)gridDim.x * 16;
  for (int64_t base = (int64_t)blockIdx.x * 16; base < n_units; base += step * kU) {
    float4 g0[kU], g1[kU], u0[kU], u1[kU], h0[kU], h1[kU];
    int64_t unit[kU];
#pragma unroll
    for (int v = 0; v < kU; ++v) {
      unit[v] = base + v * step + (threadIdx.x >> 4);
      const bool live = unit[v] < n_units;
      const int64_t r = live ? unit[v] / blocks : 0;
      const int c = live ? (int)(unit[v] - r * blocks) : 0;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4* gp = reinterpret_cast<const float4*>(gu + r * 2 * I + (int64_t)c * 2 * kTile);
      const float4* hp = reinterpret_cast<const float4*>(dh + r * I + (int64_t)c * kTile);
      g0[v] = live ? __ldg(gp + 2 * sub) : z;
      g1[v] = live ? __ldg(gp + 2 * sub + 1) : z;
      u0[v] = live ? __ldg(gp + 32 + 2 * sub) : z;
      u1[v] = live ? __ldg(gp + 32 + 2 * sub + 1) : z;
      h0[v] = live ? __ldg(hp + 2 * sub) : z;
      h1[v] = live ? __ldg(hp + 2 * sub + 1) : z;
    }
#pragma unroll
    for (int v = 0; v < kU; ++v) {
      const bool live = unit[v] < n_units;
      const int64_t r = live ? unit[v] / blocks : 0;
      const int c = live ? (int)(unit[v] - r * blocks) : 0;
      const float gv[8] = {g0[v].x, g0[v].y, g0[v].z, g0[v].w, g1[v].x, g1[v].y, g1[v].z, g1[v].w};
      const float uv[8] = {u0[v].x, u0[v].y, u0[v].z, u0[v].w, u1[v].x, u1[v].y, u1[v].z, u1[v].w};
      const float hv[8] = {h0[v].x, h0[v].y, h0[v].z, h0[v].w, h1[v].x, h1[v].y, h1[v].z, h1[v].w};
      float dg[8], du[8];
      float ag = 0.0f, au = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // sigmoid with the hardware exp2 and reciprocal, as the forward's SiLU
        const float sg = __fdividef(1.0f, 1.0f + __expf(-gv[i]));
        const float dsilu = sg * (1.0f + gv[i] * (1.0f - sg));
        dg[i] = hv[i] * uv[i] * dsilu;
        du[i] = hv[i] * (gv[i] * sg);
        ag = fmaxf(ag, fabsf(dg[i]));
        au = fmaxf(au, fabsf(du[i]));
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        ag = fmaxf(ag, __shfl_xor_sync(0xffffffffu, ag, o));
        au = fmaxf(au, __shfl_xor_sync(0xffffffffu, au, o));
      }
      if (!live) continue;
      const float sg_ = tile_scale(ag), su = tile_scale(au);
      uint2 og, ou;
      og.x = e4m3x4(__fmul_rn(dg[0], sg_), __fmul_rn(dg[1], sg_), __fmul_rn(dg[2], sg_), __fmul_rn(dg[3], sg_));
      og.y = e4m3x4(__fmul_rn(dg[4], sg_), __fmul_rn(dg[5], sg_), __fmul_rn(dg[6], sg_), __fmul_rn(dg[7], sg_));
      ou.x = e4m3x4(__fmul_rn(du[0], su), __fmul_rn(du[1], su), __fmul_rn(du[2], su), __fmul_rn(du[3], su));
      ou.y = e4m3x4(__fmul_rn(du[4], su), __fmul_rn(du[5], su), __fmul_rn(du[6], su), __fmul_rn(du[7], su));
      uint8_t* row = q + r * 2 * I + (int64_t)c * 2 * kTile;
      reinterpret_cast<uint2*>(row)[sub] = og;
      reinterpret_cast<uint2*>(row + kTile)[sub] = ou;
      if (sub == 0) {
        qs[r * 2 * blocks + 2 * c] = sg_;
        qs[r * 2 * blocks + 2 * c + 1] = su;
      }
    }
  }
}

// One warp per (token, slot): dgates[t, k] = dy[t] . Y[token_row[t, k]] in fp32
// (lane-strided partial sums, then a fixed butterfly).
__global__ void __launch_bounds__(256) gate_grad_kernel(const __nv_bfloat16* __restrict__ dy,
                                                        const __nv_bfloat16* __restrict__ y_rows,
                                                        const int32_t* __restrict__ token_row,
                                                        int T, int H, int K, int64_t routed_cap,
                                                        float* __restrict__ dgates,
                                                        uint32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < (int64_t)T * K;
       p += warps) {
    const int64_t t = p / K;
    const int64_t r = token_row[p];
    if (r < 0 || r >= routed_cap) {
      if (lane == 0) flag_status(status, kStatusBounds);
      continue;
    }
    const uint2* d2 = reinterpret_cast<const uint2*>(dy + t * H);
    const uint2* y2 = reinterpret_cast<const uint2*>(y_rows + r * H);
    float acc = 0.0f;
    for (int i = lane; i < H / 4; i += 32) {
      const uint2 d = __ldg(d2 + i);
      const uint2 yv = __ldg(y2 + i);
      acc = fmaf(bf16_lo(d.x), bf16_lo(yv.x), acc);
      acc = fmaf(bf16_hi(d.x), bf16_hi(yv.x), acc);
      acc = fmaf(bf16_lo(d.y), bf16_lo(yv.y), acc);
      acc = fmaf(bf16_hi(d.y), bf16_hi(yv.y), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dgates[p] = acc;
  }
}

// Column tiles for the weight gradients: 128 GEMM rows x 1 channel. One CTA
// per 128-row block and 32 channels (128 channels for the bf16 sources): the
// values (computed on the fly from the source with 16-byte loads, 0 on
// padding rows) go through shared memory, 8 threads reduce each channel's
// amax over the 128 rows, and each writes 16 codes of the channel's
// transposed row. A operands keep the scale ([C, R/128]); B
// operands store its inverse, block-major ([R/128, C]), for the per-column
// promotion of the weight-gradient GEMM.
enum ColSource { kColDy = 0, kColX = 1, kColH = 2, kColDgu = 3 };

struct ColArgs {
  const int32_t* row_token;   // [routed_cap] token of each routed GEMM row, -1 on padding
  int64_t routed_cap;         // rows from here on are the shared expert's: token r - routed_cap
  int T;
  const float* row_gate;      // [R] gate of the row's slot (1: shared row)
  const __nv_bfloat16* src;   // dy or x [T, C] (kColDy, kColX)
  const float* gu;            // [R, 2I] recomputed G/U rows (kColH, kColDgu)
  const float* dh;            // [R, I] (kColDgu)
  int64_t R;                  // GEMM rows (multiple of 128)
  int C;                      // channels of the output
  int I;
  uint8_t* codes;             // [C, R]
  float* scales;              // A: [C, R/128]; B: inverse, [R/128, C]
  bool b_operand;
};

template <int kSrc>
MOE_DEV float col_value(const ColArgs& a, int64_t r, int c) {
  const int64_t rs = r - a.routed_cap;
  const int t = r < a.routed_cap ? a.row_token[r] : (rs < a.T ? (int)rs : -1);
  if (t < 0) return 0.0f;
  if (kSrc == kColDy) return __fmul_rn(a.row_gate[r], __bfloat162float(a.src[(int64_t)t * a.C + c]));
  if (kSrc == kColX) return __bfloat162float(a.src[(int64_t)t * a.C + c]);
  if (kSrc == kColH) {
    const float* row = a.gu + r * 2 * a.I + (int64_t)(c / 128) * 256 + c % 128;
    const float g = row[0], u = row[128];
    const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
    return g * sg * u;
  }
  // kColDgu: channel c of w13's order; block c / 256 holds 128 gate then 128 up
  const int j = c % 256, ch = (c / 256) * 128 + (j % 128);
  const float* row = a.gu + r * 2 * a.I + (int64_t)(c / 256) * 256 + (j % 128);
  const float g = row[0], u = row[128];
  const float d = a.dh[r * a.I + ch];
  const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
  return j < 128 ? d * u * (sg * (1.0f + g * (1.0f - sg))) : d * (g * sg);
}

// The token of GEMM row r (-1 on padding rows).
MOE_DEV int col_token(const ColArgs& a, int64_t r) {
  const int64_t rs = r - a.routed_cap;
  return r < a.routed_cap ? a.row_token[r] : (rs < a.T ? (int)rs : -1);
}

// The values of 4 consecutive channels c .. c+3 (one 128-channel block) of
// GEMM row r from the fp32 sources, with 16-byte loads; same arithmetic as
// col_value.
template <int kSrc>
MOE_DEV void col_values4(const ColArgs& a, int64_t r, int c, float (&v)[4]) {
  if (kSrc == kColH) {
    const float* row = a.gu + r * 2 * a.I + (int64_t)(c / 128) * 256 + c % 128;
    const float4 g4 = *reinterpret_cast<const float4*>(row);
    const float4 u4 = *reinterpret_cast<const float4*>(row + 128);
    const float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float sg = __fdividef(1.0f, 1.0f + __expf(-g[j]));
      v[j] = g[j] * sg * u[j];
    }
  } else {
    const int jj = c % 256, ch = (c / 256) * 128 + (jj % 128);
    const float* row = a.gu + r * 2 * a.I + (int64_t)(c / 256) * 256 + (jj % 128);
    const float4 g4 = *reinterpret_cast<const float4*>(row);
    const float4 u4 = *reinterpret_cast<const float4*>(row + 128);
    const float4 d4 = *reinterpret_cast<const float4*>(a.dh + r * a.I + ch);
    const float g[4] = {g4.x, g4.y, g4.z, g4.w}, u[4] = {u4.x, u4.y, u4.z, u4.w};
    const float d[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float sg = __fdividef(1.0f, 1.0f + __expf(-g[j]));
      v[j] = jj < 128 ? d[j] * u[j] * (sg * (1.0f + g[j] * (1.0f - sg))) : d[j] * (g[j] * sg);
    }
  }
}

// Codes and scale of each of the 32 channels c0.. of one 128-row block from
// vals (8 threads per channel: the amax over the 128 rows, then 16 codes each).
MOE_DEV void quantize_col_block(const ColArgs& a, const float (*vals)[33], int64_t rb, int c0) {
  const int c = threadIdx.x >> 3, part = threadIdx.x & 7;
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(vals[part * 16 + i][c]));
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (c0 + c >= a.C) return;
  const float s = tile_scale(amax);
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    w[k] = e4m3x4(__fmul_rn(vals[part * 16 + 4 * k][c], s), __fmul_rn(vals[part * 16 + 4 * k + 1][c], s),
                  __fmul_rn(vals[part * 16 + 4 * k + 2][c], s), __fmul_rn(vals[part * 16 + 4 * k + 3][c], s));
  reinterpret_cast<uint4*>(a.codes + (int64_t)(c0 + c) * a.R + rb * kTile)[part] =
      make_uint4(w[0], w[1], w[2], w[3]);
  if (part == 0) {
    if (a.b_operand)
      a.scales[rb * a.C + c0 + c] = __fdiv_rn(1.0f, s);
    else
      a.scales[(int64_t)(c0 + c) * (a.R / kTile) + rb] = s;
  }
}

// bf16 sources (dY scaled by the row's gate, x): one CTA per 128-row block
// and 128 channels, the four 32-channel blocks' 16-byte loads all issued
// before the first is used.
template <int kSrc>
__global__ void __launch_bounds__(256) quantize_cols_bf16_kernel(const ColArgs a) {
  __shared__ float vals[kTile][33];
  const int64_t rb = blockIdx.x;
  const int cb = blockIdx.y * 128;
  const int q = threadIdx.x & 3;  // channels 8q .. 8q + 7 of each 32-channel block
  uint4 u[2][4];
  float gate[2];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t gr = rb * kTile + half * 64 + (threadIdx.x >> 2);
    const int t = col_token(a, gr);
    gate[half] = (kSrc == kColDy && t >= 0) ? a.row_gate[gr] : 1.0f;
#pragma unroll
    for (int blk = 0; blk < 4; ++blk)
      u[half][blk] = t >= 0 ? *reinterpret_cast<const uint4*>(a.src + (int64_t)t * a.C + cb +
                                                              32 * blk + 8 * q)
                            : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint4 v = u[half][blk];
      const float b[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                          bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
      const int r = half * 64 + (threadIdx.x >> 2);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        vals[r][8 * q + j] = kSrc == kColDy ? __fmul_rn(gate[half], b[j]) : b[j];
    }
    __syncthreads();
    quantize_col_block(a, vals, rb, cb + 32 * blk);
    __syncthreads();
  }
}

template <int kSrc>
__global__ void __launch_bounds__(256) quantize_cols_kernel(const ColArgs a) {
  __shared__ float vals[kTile][33];
  const int64_t rb = blockIdx.x;
  const int c0 = blockIdx.y * 32;
  if ((kSrc == kColH || kSrc == kColDgu) && c0 + 32 <= a.C) {
    // whole 32-channel block of an fp32 source: 16-byte loads (4 channels)
    const int q = threadIdx.x & 7;  // channels c0 + 4q .. + 3
#pragma unroll
    for (int quarter = 0; quarter < 4; ++quarter) {
      const int r = quarter * 32 + (threadIdx.x >> 3);
      const int64_t gr = rb * kTile + r;
      float f[4] = {0, 0, 0, 0};
      if (col_token(a, gr) >= 0) col_values4<kSrc>(a, gr, c0 + 4 * q, f);
#pragma unroll
      for (int j = 0; j < 4; ++j) vals[r][4 * q + j] = f[j];
    }
  } else {
    for (int i = threadIdx.x; i < kTile * 32; i += blockDim.x) {
      const int r = i >> 5, c = i & 31;
      vals[r][c] = (c0 + c < a.C) ? col_value<kSrc>(a, rb * kTile + r, c0 + c) : 0.0f;
    }
  }
  __syncthreads();
  quantize_col_block(a, vals, rb, c0);
}

int grid_for(int64_t units, int per_cta, int sm_count) {
  int64_t blocks = (units + per_cta - 1) / per_cta;
  const int64_t cap = (int64_t)sm_count * 8;
  if (blocks > cap) blocks = cap;
  return (int)(blocks > 0 ? blocks : 1);
}

}  // namespace

cudaError_t launch_transpose_blocks(const uint8_t* w, const float* s, int64_t groups, int64_t rows,
                                    int64_t cols, uint8_t* wt, float* st, cudaStream_t stream) {
  if (groups == 0) return cudaSuccess;
  dim3 grid((unsigned)(cols / kTile), (unsigned)(rows / kTile), (unsigned)groups);
  transpose_blocks_kernel<<<grid, 256, 0, stream>>>(w, s, rows, cols, wt, st);
  return cudaGetLastError();
}

cudaError_t launch_dy_rows_quantize(const void* dy, const float* gates, int T, int H, int K,
                                    const int32_t* token_row, int64_t routed_cap, uint8_t* q,
                                    float* qs, float* row_gate, uint32_t* status,
                                    cudaStream_t stream, int sm_count) {
  const int64_t n_tiles = (int64_t)T * (H / kTile);
  if (n_tiles == 0) return cudaSuccess;
  dy_rows_quantize_kernel<<<grid_for(n_tiles, 16, sm_count), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(dy), gates, T, H, K, token_row, routed_cap, q, qs, row_gate,
      status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_cols(int source, const int32_t* row_token, int64_t routed_cap, int T,
                                 const float* row_gate, const void* src, const float* gu,
                                 const float* dh, int64_t R, int C, int I, uint8_t* codes,
                                 float* scales, bool b_operand, cudaStream_t stream) {
  if (R == 0 || C == 0) return cudaSuccess;
  ColArgs a{row_token, routed_cap, T, row_gate, static_cast<const __nv_bfloat16*>(src), gu, dh,
            R, C, I, codes, scales, b_operand};
  dim3 grid((unsigned)(R / kTile), (unsigned)((C + 31) / 32));
  const bool bf16_wide = (source == kColDy || source == kColX) && C % 128 == 0;
  dim3 grid128((unsigned)(R / kTile), (unsigned)(C / 128));
  switch (source) {
    case kColDy:
      if (bf16_wide) quantize_cols_bf16_kernel<kColDy><<<grid128, 256, 0, stream>>>(a);
      else quantize_cols_kernel<kColDy><<<grid, 256, 0, stream>>>(a);
      break;
    case kColX:
      if (bf16_wide) quantize_cols_bf16_kernel<kColX><<<grid128, 256, 0, stream>>>(a);
      else quantize_cols_kernel<kColX><<<grid, 256, 0, stream>>>(a);
      break;
    case kColH: quantize_cols_kernel<kColH><<<grid, 256, 0, stream>>>(a); break;
    default: quantize_cols_kernel<kColDgu><<<grid, 256, 0, stream>>>(a); break;
  }
  return cudaGetLastError();
}

cudaError_t launch_swiglu_backward(const float* gu, const float* dh, int64_t rows, int I,
                                   uint8_t* q, float* qs, cudaStream_t stream, int sm_count) {
  const int64_t units = rows * (I / kTile);
  if (units == 0) return cudaSuccess;
  swiglu_backward_kernel<<<grid_for(units, 16, sm_count), 256, 0, stream>>>(gu, dh, rows, I, q,
                                                                           qs);
  return cudaGetLastError();
}

cudaError_t launch_gate_grad(const void* dy, const __nv_bfloat16* y_rows, const int32_t* token_row, int T,
                             int H, int K, int64_t routed_cap, float* dgates, uint32_t* status,
                             cudaStream_t stream, int sm_count) {
  const int64_t pairs = (int64_t)T * K;
  if (pairs == 0) return cudaSuccess;
  gate_grad_kernel<<<grid_for(pairs, 8, sm_count), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(dy), y_rows, token_row, T, H, K, routed_cap, dgates,
      status);
  return cudaGetLastError();
}

}  // namespace moe
