// Host-side helpers of the C ABI entry points: sizes, alignment, workspace
// addressing and the mapping of CUDA errors to moe_status codes.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_capi.h"

namespace moe {

inline int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// A typed pointer `off` bytes into a workspace.
template <typename T>
inline T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Bump allocator over a workspace: each region starts on a 256-byte boundary.
struct Carver {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t a = off;
    off = (size_t)round_up((int64_t)(off + bytes), 256);
    return a;
  }
};

}  // namespace moe
