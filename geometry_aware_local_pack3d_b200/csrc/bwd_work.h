// Backward workspace: one caller buffer carved into 256-byte-aligned arrays.
#pragma once

#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include "pack3d.h"

namespace p3d {

// Most query ranges the tensor-core summary-gradient kernel splits each (batch, head) into (the
// launch picks the count that fills whole waves of SMs); the partial sums are added in split
// order into the first range's slot before the summary gradients are un-pooled.
constexpr int kDsumSplitMax = 8;

struct BwdWork {
  void* qr;     // [BH, N, d]  rotated q, in the I/O type (bf16 or fp32)
  void* kr;     // [BH, N, d]  rotated k, in the I/O type
  float* Dl;    // [BH, N]     <g dO, o_loc>
  float* Dg;    // [BH, N]     <(1 - g) dO, o_glob>
  float* dks;   // [nsplit][BH, M, d]  gradient of the key summaries (per query range)
  float* dvs;   // [nsplit][BH, M, d]  gradient of the value summaries
  int nsplit;   // partials the un-pooling adds (1: reduced in place, or the CUDA-core path)
  // tensor-core path only (null otherwise)
  __nv_bfloat16* qtb;   // [BH, N, d]  rotated q, bf16 (the qr array itself)
  __nv_bfloat16* dogb;  // [BH, N, d]  (1 - g) dO, bf16
  float* dqg;           // [BH, N, d]  global branch's part of dq~ (rotated space)
  // GQA only (null with one query head per KV head): each query head's dk, dv in float32,
  // summed over the query heads of a KV head by k_bwd_gqa_reduce
  float* dkp;           // [BH, N, d]
  float* dvp;           // [BH, N, d]
};

inline size_t bwd_align(size_t x) { return (x + 255) & ~(size_t)255; }

// Bytes of workspace for I/O elements of `el` bytes; `tc` (bf16 only) adds the tensor-core
// path's arrays; `kv_group` > 1 (GQA) adds the per-query-head key gradients. `bh` counts query
// heads.
inline size_t bwd_workspace_bytes_for(const pack3d_index& ix, int64_t bh, size_t el, bool tc,
                                      int kv_group) {
  const size_t D = ix.geom.head_dim, rows = (size_t)bh * ix.n, sums = (size_t)bh * ix.m;
  const int ns = tc ? kDsumSplitMax : 1;
  size_t b = 2 * bwd_align(el * rows * D) + 2 * bwd_align(sizeof(float) * rows) +
             2 * bwd_align(sizeof(float) * ns * sums * D);
  if (tc) b += bwd_align(sizeof(__nv_bfloat16) * rows * D) + bwd_align(sizeof(float) * rows * D);
  if (kv_group > 1) b += 2 * bwd_align(sizeof(float) * rows * D);
  return b;
}

inline BwdWork bwd_carve(const pack3d_index& ix, int64_t bh, void* ws, size_t el, bool tc,
                         int kv_group) {
  const size_t D = ix.geom.head_dim, rows = (size_t)bh * ix.n, sums = (size_t)bh * ix.m;
  char* p = static_cast<char*>(ws);
  BwdWork w;
  w.nsplit = 1;
  const int ns = tc ? kDsumSplitMax : 1;
  w.qr = p; p += bwd_align(el * rows * D);
  w.kr = p; p += bwd_align(el * rows * D);
  w.Dl = reinterpret_cast<float*>(p); p += bwd_align(sizeof(float) * rows);
  w.Dg = reinterpret_cast<float*>(p); p += bwd_align(sizeof(float) * rows);
  w.dks = reinterpret_cast<float*>(p); p += bwd_align(sizeof(float) * ns * sums * D);
  w.dvs = reinterpret_cast<float*>(p); p += bwd_align(sizeof(float) * ns * sums * D);
  w.qtb = w.dogb = nullptr;
  w.dqg = nullptr;
  w.dkp = w.dvp = nullptr;
  if (tc) {  // bf16 I/O: qr already holds the rotated q in bf16
    w.qtb = static_cast<__nv_bfloat16*>(w.qr);
    w.dogb = reinterpret_cast<__nv_bfloat16*>(p); p += bwd_align(sizeof(__nv_bfloat16) * rows * D);
    w.dqg = reinterpret_cast<float*>(p); p += bwd_align(sizeof(float) * rows * D);
  }
  if (kv_group > 1) {
    w.dkp = reinterpret_cast<float*>(p); p += bwd_align(sizeof(float) * rows * D);
    w.dvp = reinterpret_cast<float*>(p);
  }
  return w;
}

}  // namespace p3d
