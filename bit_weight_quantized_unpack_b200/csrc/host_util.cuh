// Host-side helpers shared by the launchers: per-device caches of the SM count and of the
// large-shared-memory opt-in of each kernel.
//
// Both facts belong to a device, not to the process: a process that drives two GPUs must
// query the SM count of each and opt every kernel in on each device's context before its
// first launch there. The caches are indexed by device ordinal (0..63) and use atomics, so
// that threads making their first calls at the same time agree.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace wq {

constexpr int kMaxDevices = 64;

// SM count of the current device (0 if the query fails).
inline int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// Sets `kernel`'s dynamic shared-memory limit to `bytes` on the current device, once per
// device; `done` is one bit per device ordinal, owned by the caller (one per kernel).
template <class Kernel>
cudaError_t ensure_smem_limit(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return cudaSuccess;
}

}  // namespace wq
