// FP8 E4M3 fine-grained quantisers: 1x128 activation tiles (online) and
// 128x128 weight blocks (set-up). Rule of "DeepSeek-V3 Technical Report"
// (deepforge.srivtx.xyz), "Per-tile FP8 scaling": scale = 448 / amax,
// code = round_to_e4m3(x * scale).
#include "kernels.cuh"

namespace moe {

// One 128-column tile per 16 threads; each thread owns 8 consecutive bf16
// (one 128-bit load) and writes 8 codes (one 64-bit store). HBM-bound: reads
// 2 bytes and writes 1 byte per element plus 4 bytes per 128 elements.
__global__ void __launch_bounds__(256) quantize_1x128_kernel(const uint4* __restrict__ x,
                                                             int64_t n_tiles,
                                                             uint2* __restrict__ q,
                                                             float* __restrict__ scales) {
  const int sub = threadIdx.x & 15;
  // the whole CTA iterates together so that every shuffle is warp-convergent
  for (int64_t base = (int64_t)blockIdx.x * 16; base < n_tiles; base += (int64_t)gridDim.x * 16) {
    const int64_t tile = base + (threadIdx.x >> 4);
    const bool live = tile < n_tiles;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (live) v = __ldcs(x + tile * 16 + sub);
    float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = tile_scale(amax);
    if (live) {
      uint2 out;
      out.x = e4m3x4(__fmul_rn(f[0], s), __fmul_rn(f[1], s), __fmul_rn(f[2], s), __fmul_rn(f[3], s));
      out.y = e4m3x4(__fmul_rn(f[4], s), __fmul_rn(f[5], s), __fmul_rn(f[6], s), __fmul_rn(f[7], s));
      q[tile * 16 + sub] = out;
      if (sub == 0) scales[tile] = s;
    }
  }
}

// One CTA per 128x128 block: 256 threads hold 16 float4 each in registers,
// reduce the block amax through shared memory, then write the codes.
__global__ void __launch_bounds__(256) quantize_128x128_kernel(const float4* __restrict__ w,
                                                               int64_t cols, int64_t col_blocks,
                                                               uint32_t* __restrict__ q,
                                                               float* __restrict__ scales) {
  __shared__ float red[8];
  const int64_t rb = blockIdx.y, cb = blockIdx.x;
  const int64_t cols4 = cols >> 2;
  float4 v[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int f = threadIdx.x + 256 * i;  // float4 index inside the block
    const int r = f >> 5, c4 = f & 31;
    v[i] = __ldcs(w + (rb * kTile + r) * cols4 + cb * 32 + c4);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = tile_scale(amax);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int f = threadIdx.x + 256 * i;
    const int r = f >> 5, c4 = f & 31;
    q[(rb * kTile + r) * cols4 + cb * 32 + c4] =
        e4m3x4(__fmul_rn(v[i].x, s), __fmul_rn(v[i].y, s), __fmul_rn(v[i].z, s), __fmul_rn(v[i].w, s));
  }
  if (threadIdx.x == 0) scales[rb * col_blocks + cb] = s;
}

// The layer's activation quantiser, fused with the permutation: the codes and
// the scale of each 1x128 tile of token t go to the shared expert's GEMM row
// routed_cap + t and to the token's K routed GEMM rows token_row[t, k], so x
// is read once and no second pass copies rows. Same tiling as above; lane k
// of a tile's 16 threads fetches the k-th destination row.
__global__ void __launch_bounds__(256) quantize_scatter_kernel(
    const uint4* __restrict__ x, int T, int H, int K, const int32_t* __restrict__ token_row,
    int64_t routed_cap, uint8_t* __restrict__ a_q, float* __restrict__ a_s,
    uint32_t* __restrict__ status) {
  // 8 threads per tile, 16 consecutive elements each (two 128-bit loads, one
  // 128-bit store of codes per destination row); four tiles in flight
  constexpr int kPerThread = 4;
  const int sub = threadIdx.x & 7;
  const int tiles_per_row = H / kTile;
  const int64_t n_tiles = (int64_t)T * tiles_per_row;
  const int64_t step = (int64_t)gridDim.x * 32;
  for (int64_t base = (int64_t)blockIdx.x * 32; base < n_tiles; base += step * kPerThread) {
    uint4 v0[kPerThread], v1[kPerThread];
    int row_a[kPerThread], row_b[kPerThread];   // destinations k = sub and k = sub + 8
    int64_t tile[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      tile[u] = base + u * step + (threadIdx.x >> 3);
      const bool live = tile[u] < n_tiles;
      const int64_t t = live ? tile[u] / tiles_per_row : 0;
      v0[u] = live ? __ldcs(x + tile[u] * 16 + 2 * sub) : make_uint4(0, 0, 0, 0);
      v1[u] = live ? __ldcs(x + tile[u] * 16 + 2 * sub + 1) : make_uint4(0, 0, 0, 0);
      row_a[u] = (live && sub < K) ? __ldg(token_row + t * K + sub) : -1;
      row_b[u] = (live && sub + 8 < K) ? __ldg(token_row + t * K + sub + 8) : -1;
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const bool live = tile[u] < n_tiles;
      const int64_t t = live ? tile[u] / tiles_per_row : 0;
      const int c = live ? (int)(tile[u] - t * tiles_per_row) : 0;
      float f[16] = {bf16_lo(v0[u].x), bf16_hi(v0[u].x), bf16_lo(v0[u].y), bf16_hi(v0[u].y),
                     bf16_lo(v0[u].z), bf16_hi(v0[u].z), bf16_lo(v0[u].w), bf16_hi(v0[u].w),
                     bf16_lo(v1[u].x), bf16_hi(v1[u].x), bf16_lo(v1[u].y), bf16_hi(v1[u].y),
                     bf16_lo(v1[u].z), bf16_hi(v1[u].z), bf16_lo(v1[u].w), bf16_hi(v1[u].w)};
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float s = tile_scale(amax);
      uint4 out;
      out.x = e4m3x4(__fmul_rn(f[0], s), __fmul_rn(f[1], s), __fmul_rn(f[2], s), __fmul_rn(f[3], s));
      out.y = e4m3x4(__fmul_rn(f[4], s), __fmul_rn(f[5], s), __fmul_rn(f[6], s), __fmul_rn(f[7], s));
      out.z = e4m3x4(__fmul_rn(f[8], s), __fmul_rn(f[9], s), __fmul_rn(f[10], s), __fmul_rn(f[11], s));
      out.w = e4m3x4(__fmul_rn(f[12], s), __fmul_rn(f[13], s), __fmul_rn(f[14], s), __fmul_rn(f[15], s));
      for (int k = -1; k < K; ++k) {
        int64_t r = routed_cap + t;
        if (k >= 0) {
          const int ra = __shfl_sync(0xffffffffu, row_a[u], k & 7, 8);
          const int rb = __shfl_sync(0xffffffffu, row_b[u], k & 7, 8);
          r = k < 8 ? ra : rb;
          if (live && (r < 0 || r >= routed_cap)) {
            if (sub == 0) flag_status(status, kStatusBounds);
            continue;
          }
        }
        if (live) {
          reinterpret_cast<uint4*>(a_q + r * H + (int64_t)c * kTile)[sub] = out;
          if (sub == 0) a_s[r * tiles_per_row + c] = s;
        }
      }
    }
  }
}

cudaError_t launch_quantize_scatter(const void* x, int T, int H, int K, const int32_t* token_row,
                                    int64_t routed_cap, uint8_t* a_q, float* a_s,
                                    uint32_t* status, cudaStream_t stream, int sm_count) {
  const int64_t n_tiles = (int64_t)T * (H / kTile);
  if (n_tiles == 0) return cudaSuccess;
  int64_t blocks = (n_tiles + 31) / 32;
  const int64_t cap = (int64_t)sm_count * 8;
  if (blocks > cap) blocks = cap;
  quantize_scatter_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(x), T, H, K, token_row, routed_cap, a_q, a_s, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_1x128(const void* x, int64_t rows, int64_t cols, uint8_t* q,
                                  float* scales, cudaStream_t stream, int sm_count) {
  const int64_t n_tiles = rows * (cols / kTile);
  if (n_tiles == 0) return cudaSuccess;
  int64_t blocks = (n_tiles + 15) / 16;
  const int64_t cap = (int64_t)sm_count * 8;
  if (blocks > cap) blocks = cap;
  quantize_1x128_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(x), n_tiles, reinterpret_cast<uint2*>(q), scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_128x128(const float* w, int64_t rows, int64_t cols, uint8_t* q,
                                    float* scales, cudaStream_t stream) {
  dim3 grid((unsigned)(cols / kTile), (unsigned)(rows / kTile));
  quantize_128x128_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(w), cols,
                                                    cols / kTile, reinterpret_cast<uint32_t*>(q),
                                                    scales);
  return cudaGetLastError();
}

}  // namespace moe
