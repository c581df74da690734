// pack3d_attn_bwd_noalloc: the backward pass with its scratch memory taken from a buffer that
// lives inside this library, for callers that cannot allocate device memory themselves.
//
// pack3d_attn_bwd needs a caller-provided workspace (rotated q/k, the two D row terms and the
// summary gradients). Some callers cannot call cudaMalloc to make one: a host framework that
// owns every device allocation through its own pool and does not let libraries allocate, or a
// latency-critical loop that cannot accept cudaMalloc's implicit device synchronisation. This
// entry point serves them from a fixed, file-scope device array instead; it allocates nothing.
//
// The array is a __device__ symbol, so host code cannot use its name as a device address. The
// first call on each device (with that device current) looks its address up once with
// cudaGetSymbolAddress; later calls reuse the cached pointer. That first call should therefore
// come before any stream capture on the device.
//
// Every call shares the one array and leaves its last contents there. The backward kernels
// overwrite every workspace element they read, so nothing needs clearing between calls; calls
// whose work overlaps on the GPU (different streams, no ordering) race on the array.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace p3d {
pack3d_status check_common(const pack3d_index* idx, int dtype, int batch, int heads);
pack3d_status kv_group_of(int heads, int kv_heads, int* group);
}

namespace {
constexpr size_t kScratchBytes = PACK3D_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
pack3d_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PACK3D_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PACK3D_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || !p) return PACK3D_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PACK3D_OK;
}
}  // namespace

extern "C" pack3d_status pack3d_attn_bwd_noalloc(
    const pack3d_index* idx, const void* q, const void* k, const void* v, const void* gate,
    const void* ksum, const void* vsum, const void* o_loc, const void* o_glob,
    const float* lse_loc, const float* lse_glob, const void* dO, int dtype, int batch, int heads,
    int kv_heads, float scale, uint32_t flags, void* dq, void* dk, void* dv, void* dgate,
    void* stream) {
  // a rejected call launches nothing: the launch count reads 0 afterwards, and argument errors
  // are the ones pack3d_attn_bwd reports for the same arguments
  p3d::reset_launches();
  const pack3d_status common = p3d::check_common(idx, dtype, batch, heads);
  if (common != PACK3D_OK) return common;
  int group = 1;
  const pack3d_status kv = p3d::kv_group_of(heads, kv_heads, &group);
  if (kv != PACK3D_OK) return kv;
  const size_t need = pack3d_bwd_workspace_bytes(idx, dtype, batch, heads, kv_heads);
  if (need > kScratchBytes) return PACK3D_ERR_WORKSPACE;  // problem too large for the buffer
  void* ws = nullptr;
  const pack3d_status st = scratch_address(&ws);
  if (st != PACK3D_OK) return st;
  return pack3d_attn_bwd(idx, q, k, v, gate, ksum, vsum, o_loc, o_glob, lse_loc, lse_glob, dO,
                         dtype, batch, heads, kv_heads, scale, flags, dq, dk, dv, dgate, ws,
                         kScratchBytes, stream);
}
