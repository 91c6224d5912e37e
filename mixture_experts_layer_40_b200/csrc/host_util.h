// Host-side helpers of the C ABI entry points: sizes, alignment, workspace
// addressing and the mapping of CUDA errors to moe_status codes.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <mutex>

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

// An NVTX range over a host scope (entry points and the forward's stages), for
// timeline profilers; without a profiler attached the calls do nothing. The
// range covers the host-side enqueue, not the kernels' execution.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// A set-up step (kernel attributes) done once per device: the first call
// with a device current runs it, later calls on that device skip it. A step
// that fails is retried by the next call. Safe to use from several host
// threads. Function attributes belong to the device's context, so a process
// that resets a device (cudaDeviceReset) must not call the library on that
// device again.
class DeviceOnce {
 public:
  template <typename F>
  cudaError_t run(F&& setup) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done_[dev].load(std::memory_order_acquire)) return cudaSuccess;
    std::lock_guard<std::mutex> lock(mu_);
    if (done_[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    e = setup();
    if (e == cudaSuccess) done_[dev].store(true, std::memory_order_release);
    return e;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::mutex mu_;
  std::atomic<bool> done_[kMaxDevices] = {};
};

}  // namespace moe
