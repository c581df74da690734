// Shared device helpers of the PACK3D CUDA path (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pack3d.h"

namespace p3d {

constexpr int kNbr = 27;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// status word slots (pack3d_index::status[0])
constexpr int kStatusFirstError = 0;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

struct Coord {
  int z, y, x;
};
__device__ __forceinline__ Coord decode(int32_t c) {
  return Coord{c >> 20, (c >> 10) & 1023, c & 1023};
}
__device__ __forceinline__ int coord_axis(const Coord& c, int a) {
  return a == 0 ? c.z : (a == 1 ? c.y : c.x);
}

// Records the first device-detected error in the status word (never traps).
__device__ __forceinline__ void set_status(int32_t* status, int code) {
  if (status) atomicCAS(status + kStatusFirstError, 0, code);
}

// (cos, sin) of coordinate value `cv` on axis `a` for rotation pair p of that axis third;
// the table is [3 axes][rows][pairs] (each axis carries its own coordinate scale).
__device__ __forceinline__ int rope_slot(int rows, int pairs, int a, int cv, int p) {
  return (a * rows + cv) * pairs + p;
}
__device__ __forceinline__ float2 rope_cs(const float* rope, int rows, int pairs, int a, int cv,
                                          int p) {
  return reinterpret_cast<const float2*>(rope)[rope_slot(rows, pairs, a, cv, p)];
}

// Is summary `m`'s box within Chebyshev distance 1 of coordinate c? The box of summary
// (mz, my, mx) spans [m_a * ext_a, m_a * ext_a + ext_a - 1] per axis (its part outside the grid
// cannot change the answer: the cube around a token reaches at most one site past the grid).
__device__ __forceinline__ bool block_is_near(const pack3d_index& ix, int m, const Coord& c) {
  const int ngx = ix.sum_grid[2], ngy = ix.sum_grid[1];
  const int mx = m % ngx, my = (m / ngx) % ngy, mz = m / (ngx * ngy);
  const int ez = ix.sum_ext[0], ey = ix.sum_ext[1], ex = ix.sum_ext[2];
  const int lz = mz * ez, ly = my * ey, lx = mx * ex;
  return lz <= c.z + 1 && lz + ez - 1 >= c.z - 1 && ly <= c.y + 1 && ly + ey - 1 >= c.y - 1 &&
         lx <= c.x + 1 && lx + ex - 1 >= c.x - 1;
}

// A summary with no member present takes part in no softmax.
__device__ __forceinline__ bool summary_empty(const pack3d_index& ix, int m) {
  return (ix.empty[m >> 5] >> (m & 31)) & 1u;
}

// Summary-grid coordinates of the summaries whose box meets the cube [c-1, c+1]^3 (clipped to
// the grid): [z0, z1] x [y0, y1] x [x0, x1]; empty ranges when `on` is false.
struct ExclBox {
  int z0, z1, y0, y1, x0, x1;
};
__device__ __forceinline__ ExclBox excl_box(const pack3d_index& ix, const Coord& c, bool on) {
  ExclBox e{0, -1, 0, -1, 0, -1};
  if (!on) return e;
  const pack3d_geom& g = ix.geom;
  e.z0 = max(c.z - 1, 0) / ix.sum_ext[0]; e.z1 = min(c.z + 1, g.gz - 1) / ix.sum_ext[0];
  e.y0 = max(c.y - 1, 0) / ix.sum_ext[1]; e.y1 = min(c.y + 1, g.gy - 1) / ix.sum_ext[1];
  e.x0 = max(c.x - 1, 0) / ix.sum_ext[2]; e.x1 = min(c.x + 1, g.gx - 1) / ix.sum_ext[2];
  return e;
}

// GQA: query head bh = b * H + h reads the keys, values and summaries of KV head
// b * H_kv + h / G = bh / G, G = H / H_kv query heads per KV head.
__host__ __device__ __forceinline__ int64_t kv_of(int64_t bh, int group) { return bh / group; }

__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + __expf(-a)); }

// Summary tiles: the M summaries of each (batch, head) are stored in tiles of 64 (zero padded
// to a whole tile); a tile holds d/8 columns, each 64 summaries x 8 consecutive elements. This
// is the no-swizzle tensor-core operand layout of a 64-summary chunk, so one contiguous copy
// moves a chunk into shared memory. Element (bh, m, e) lives at this element offset:
__host__ __device__ __forceinline__ int64_t sum_index(int64_t bh, int64_t m, int e, int d,
                                                      int64_t m_tiles) {
  return ((bh * m_tiles + (m >> 6)) * (d >> 3) + (e >> 3)) * 512 + (m & 63) * 8 + (e & 7);
}
__host__ __device__ __forceinline__ int64_t sum_tiles(int64_t m) { return (m + 63) >> 6; }

// Phase timestamps for one CTA, compiled in only by a tracing build (P3D_TRACE_ENABLED):
// the kernels mark their handoffs with P3D_TRACE(slot); normal builds emit nothing.
#ifdef P3D_TRACE_ENABLED
#ifndef P3D_TRACE_CTA
#define P3D_TRACE_CTA 0
#endif
static __device__ unsigned long long g_trace[4096];
#define P3D_TRACE(slot)                                                            \
  do {                                                                             \
    if (blockIdx.x == (P3D_TRACE_CTA)) {                                           \
      unsigned long long t_;                                                       \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                       \
      g_trace[(slot) & 4095] = t_;                                                 \
    }                                                                              \
  } while (0)
// SM clock next to the global timer, for measuring the clock a kernel actually runs at
#define P3D_TRACE_CLK(slot)                                                        \
  do {                                                                             \
    if (blockIdx.x == (P3D_TRACE_CTA)) {                                           \
      unsigned long long t_;                                                       \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                       \
      g_trace[(slot) & 4095] = t_;                                                 \
      g_trace[((slot) + 1) & 4095] = (unsigned long long)clock64();                \
    }                                                                              \
  } while (0)
// SM clock only (fine-grained intervals inside one role)
#define P3D_TRACE_C(slot)                                                          \
  do {                                                                             \
    if (blockIdx.x == (P3D_TRACE_CTA))                                             \
      g_trace[(slot) & 4095] = (unsigned long long)clock64();                      \
  } while (0)
#else
#define P3D_TRACE_C(slot) \
  do {                    \
  } while (0)
#define P3D_TRACE_CLK(slot) \
  do {                      \
  } while (0)
#define P3D_TRACE(slot) \
  do {                  \
  } while (0)
#endif

}  // namespace p3d
