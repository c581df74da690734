// Host-side launch helpers: per-host-thread launch accounting and per-device caches.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace p3d {
extern thread_local int g_launches;
inline void count_launch(int n = 1) { g_launches += n; }
inline void reset_launches() { g_launches = 0; }

constexpr int kMaxCachedDevices = 64;

// Number of SMs of the current device (looked up once per device; a device beyond the cache is
// looked up on every call).
inline int sm_count() {
  static std::atomic<int> cache[kMaxCachedDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev >= 0 && dev < kMaxCachedDevices) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int v = 0;
  cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
  v = v > 0 ? v : 148;
  if (dev >= 0 && dev < kMaxCachedDevices) cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// Cycle budget of every bounded device-side wait of the tensor-core kernels, read at each
// launch. The default (4e9 SM cycles, about 2 s at 1.97 GHz) is far above any legitimate wait;
// pack3d_testing_set_wait_budget lowers it so that a test can make a wait run out.
constexpr long long kDefaultWaitBudget = 4000000000LL;
inline std::atomic<long long>& wait_budget_store() {
  static std::atomic<long long> v{kDefaultWaitBudget};
  return v;
}
inline long long wait_budget_cycles() { return wait_budget_store().load(std::memory_order_relaxed); }

// Raises the dynamic shared-memory limit of `func` to `bytes` on the current device, once per
// device (`done` is the kernel's own bit mask of devices already set; setting the attribute
// twice from two host threads is harmless).
inline cudaError_t smem_attr_once(const void* func, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const bool cacheable = dev >= 0 && dev < kMaxCachedDevices;
  if (cacheable && ((done.load(std::memory_order_acquire) >> dev) & 1ull)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && cacheable) done.fetch_or(1ull << dev, std::memory_order_release);
  return e;
}
}  // namespace p3d
