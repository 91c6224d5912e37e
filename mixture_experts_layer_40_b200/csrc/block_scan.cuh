// Block-wide prefix sums over one value per thread (up to 1024 threads),
// used by the permutation and the expert-parallel dispatch plan. Every
// thread of the block must call them (they synchronise the block).
#pragma once

#include "common.cuh"

namespace moe {

// Exclusive prefix sum of a 0/1 flag. Returns this thread's prefix; *total
// receives the block sum. warp_sums: shared int[33].
MOE_DEV int block_scan_flag(bool flag, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[warp] = __popc(ballot);
  __syncthreads();
  if (warp == 0) {
    int v = lane < nwarps ? warp_sums[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane < nwarps) warp_sums[lane] = incl - v;
    if (lane == 31) warp_sums[32] = incl;
  }
  __syncthreads();
  const int res = warp_sums[warp] + in_warp;
  *total = warp_sums[32];
  __syncthreads();
  return res;
}

// Exclusive prefix sum of v over the block. warp_sums: shared int[33].
MOE_DEV int block_scan_int(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? warp_sums[lane] : 0;
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < nwarps) warp_sums[lane] = wi - w;
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  const int res = warp_sums[warp] + incl - v;
  *total = warp_sums[32];
  __syncthreads();
  return res;
}

}  // namespace moe
