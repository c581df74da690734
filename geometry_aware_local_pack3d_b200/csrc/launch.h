// Per-host-thread count of kernel launches issued by the last public call.
#pragma once

#include <cuda_runtime.h>

namespace p3d {
extern thread_local int g_launches;
inline void count_launch(int n = 1) { g_launches += n; }
inline void reset_launches() { g_launches = 0; }

// Number of SMs of the current device (looked up once per process).
inline int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    n = v > 0 ? v : 148;
  }
  return n;
}
}  // namespace p3d
