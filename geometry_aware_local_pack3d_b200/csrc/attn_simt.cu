// PACK3D attention on CUDA cores in float32: the general path for every supported dtype and
// head_dim (float32 I/O always runs here), forward and backward.
//
// Forward (project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contracts 1-3;
// paper summary §3.2, §3.3, §3.5):
//   k_local_fwd   one thread per query: exact softmax over the <= 27 coordinate neighbours,
//                 keys rotated on the fly from the rotation table, offsets in canonical order.
//   k_global_fwd  one thread per query: online softmax over all summaries, staged through
//                 shared memory in chunks (every thread reads the same summary: broadcast),
//                 optional exclude_near mask, and the sigmoid mixer fused in the epilogue.
// Backward (paper summary §3.4), one warp per row, lanes over head dims:
//   k_bwd_prep    rotated q, k; dgate; D_loc = <g dO, o_loc>, D_glob = <(1-g) dO, o_glob>.
//   k_bwd_dsum    dK_sum[m] = sum_i dS_im q~_i and dV_sum[m] = sum_i P_im (1-g_i) dO_i.
//   k_bwd_dq      dq = R(c)^T (sum_j dS_ij k~_j + sum_m dS_im K_sum[m]); 4 lanes per row.
//   k_bwd_dkv     dk, dv gathered over the key's own neighbourhood (the 3x3x3 relation is
//                 symmetric, so no scatter/atomics) plus 1/|S| of its block's summary grads;
//                 4 lanes per row.
// On the bf16 tensor-core path the global branch's summary gradients and its part of dq come
// from the kernels of bwd_tc.cu instead of k_bwd_dsum and the summary loop of k_bwd_dq.
// Every reduction order depends on coordinates (offset order, canonical slots, summary ids),
// never on memory slots, except the sums over all queries in k_bwd_dsum.
#include <math.h>

#include "bwd_work.h"

#include "common.cuh"
#include "launch.h"
#include "vec.cuh"

namespace p3d {

// ------------------------------------------------------------------------------ helpers
template <typename T, int D>
__device__ __forceinline__ void load_row(const T* __restrict__ p, float (&x)[D]) {
  constexpr int E = Vec<T>::E;
#pragma unroll
  for (int c = 0; c < D / E; ++c) {
    float t[E];
    Vec<T>::load(p + c * E, t);
#pragma unroll
    for (int e = 0; e < E; ++e) x[c * E + e] = t[e];
  }
}

template <typename T, int D>
__device__ __forceinline__ void store_row(T* p, const float (&x)[D]) {
  constexpr int E = Vec<T>::E;
#pragma unroll
  for (int c = 0; c < D / E; ++c) {
    float t[E];
#pragma unroll
    for (int e = 0; e < E; ++e) t[e] = x[c * E + e];
    Vec<T>::store(p + c * E, t);
  }
}

// x <- R(c) x (sign = +1) or R(c)^T x (sign = -1), rotation table in global memory.
template <int D>
__device__ __forceinline__ void rotate_row(const pack3d_index& ix, const Coord& c,
                                           float (&x)[D], float sign) {
  constexpr int DA = D / 3;
#pragma unroll
  for (int e = 0; e < D; e += 2) {
    const int axis = e / DA, p = (e % DA) / 2;
    const float2 cs = rope_cs(ix.rope, ix.rope_rows, ix.rope_pairs, axis, coord_axis(c, axis), p);
    const float sn = sign * cs.y;
    const float x0 = x[e], x1 = x[e + 1];
    x[e] = x0 * cs.x - x1 * sn;
    x[e + 1] = x0 * sn + x1 * cs.x;
  }
}

// ------------------------------------------------------------------------ local forward
template <typename T, int D>
__global__ void __launch_bounds__(128) k_local_fwd(pack3d_index ix, const T* __restrict__ q,
                                                   const T* __restrict__ k,
                                                   const T* __restrict__ v, float scale,
                                                   int kv_group, T* __restrict__ o_loc,
                                                   float* __restrict__ lse_loc) {
  const int64_t bh = blockIdx.y;
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= ix.n) return;
  const int64_t rowbase = bh * ix.n;
  const int64_t kvbase = kv_of(bh, kv_group) * ix.n;  // keys and values of the KV head
  const Coord ci = decode(ix.coord[i]);
  float qr[D];
  load_row<T, D>(q + (rowbase + i) * D, qr);
  rotate_row<D>(ix, ci, qr, 1.f);

  const float sl2 = scale * kLog2e;
  float s[kNbr];
  float mx = -INFINITY;
#pragma unroll
  for (int o = 0; o < kNbr; ++o) {
    const int j = ix.nbr[i * kNbr + o];
    s[o] = -INFINITY;
    if (j < 0) continue;
    float kr[D];
    load_row<T, D>(k + (kvbase + j) * D, kr);
    rotate_row<D>(ix, decode(ix.coord[j]), kr, 1.f);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < D; ++e) dot = fmaf(qr[e], kr[e], dot);
    s[o] = dot * sl2;
    mx = fmaxf(mx, s[o]);
  }
  float l = 0.f;
  float acc[D];
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] = 0.f;
#pragma unroll
  for (int o = 0; o < kNbr; ++o) {
    const int j = ix.nbr[i * kNbr + o];
    if (j < 0) continue;
    const float p = exp2f(s[o] - mx);
    l += p;
    float vr[D];
    load_row<T, D>(v + (kvbase + j) * D, vr);
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] = fmaf(p, vr[e], acc[e]);
  }
  const float inv = 1.f / l;  // the query itself is always a neighbour: l >= 1
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] *= inv;
  store_row<T, D>(o_loc + (rowbase + i) * D, acc);
  if (lse_loc) lse_loc[rowbase + i] = (mx + log2f(l)) * kLn2;
}

// ------------------------------------------------------------------ global forward + mixer
template <typename T, int D, int CH>
__global__ void __launch_bounds__(128) k_global_fwd(
    pack3d_index ix, const T* __restrict__ q, const T* __restrict__ ksum,
    const T* __restrict__ vsum, const T* __restrict__ gate, const T* o_loc_in, float scale,
    int exclude_near, int kv_group, T* o, float* __restrict__ lse_glob,
    T* __restrict__ o_glob_out) {
  __shared__ float sk[CH][D];
  __shared__ float sv[CH][D];
  const int64_t bh = blockIdx.y;
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const bool live = i < ix.n;
  const int64_t rowbase = bh * ix.n;
  const int M = (int)ix.m;
  Coord ci{0, 0, 0};
  float qr[D];
  if (live) {
    ci = decode(ix.coord[i]);
    load_row<T, D>(q + (rowbase + i) * D, qr);
    rotate_row<D>(ix, ci, qr, 1.f);
  }
  const float sl2 = scale * kLog2e;
  float mx = -INFINITY, l = 0.f;
  float acc[D];
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] = 0.f;

  const int64_t MT = sum_tiles(M);
  for (int m0 = 0; m0 < M; m0 += CH) {
    const int cnt = min(CH, M - m0);
    __syncthreads();
    for (int t = threadIdx.x; t < cnt * D; t += blockDim.x) {
      const int64_t off = sum_index(kv_of(bh, kv_group), m0 + t / D, t % D, D, MT);
      sk[t / D][t % D] = to_f(ksum[off]);
      sv[t / D][t % D] = to_f(vsum[off]);
    }
    __syncthreads();
    if (!live) continue;
    for (int mm = 0; mm < cnt; ++mm) {
      if (summary_empty(ix, m0 + mm)) continue;  // no member: in no softmax
      if (exclude_near && block_is_near(ix, m0 + mm, ci)) continue;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < D; ++e) dot = fmaf(qr[e], sk[mm][e], dot);
      const float sc = dot * sl2;
      if (sc > mx) {
        const float corr = exp2f(mx - sc);  // exp2(-inf) = 0 on the first hit
        l *= corr;
#pragma unroll
        for (int e = 0; e < D; ++e) acc[e] *= corr;
        mx = sc;
      }
      const float p = exp2f(sc - mx);
      l += p;
#pragma unroll
      for (int e = 0; e < D; ++e) acc[e] = fmaf(p, sv[mm][e], acc[e]);
    }
  }
  if (!live) return;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] *= inv;
  if (lse_glob) lse_glob[rowbase + i] = l > 0.f ? (mx + log2f(l)) * kLn2 : -INFINITY;
  if (o_glob_out) store_row<T, D>(o_glob_out + (rowbase + i) * D, acc);
  // mixer (paper summary §3.3): o = g o_loc + (1 - g) o_glob, g = sigmoid(a)
  const float a = to_f(gate[rowbase + i]);
  const float g = 1.f / (1.f + expf(-a));
  float ol[D];
  load_row<T, D>(o_loc_in + (rowbase + i) * D, ol);
#pragma unroll
  for (int e = 0; e < D; ++e) acc[e] = g * ol[e] + (1.f - g) * acc[e];
  store_row<T, D>(o + (rowbase + i) * D, acc);
}

// ------------------------------------------------------------------------------ backward
// Warp-per-row layout: lane owns dims e = lane + 32 * t, t < KT.
template <int D> struct WarpRow {
  static constexpr int KT = (D + 31) / 32;
  float x[KT];
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

template <typename T, int D>
__device__ __forceinline__ void wr_load(const T* __restrict__ p, WarpRow<D>& r, int lane) {
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) {
    const int e = lane + 32 * t;
    r.x[t] = e < D ? to_f(p[e]) : 0.f;
  }
}
template <typename T, int D>
__device__ __forceinline__ void wr_load_sum(const T* __restrict__ base, int64_t bh, int64_t m,
                                            int64_t mt, WarpRow<D>& r, int lane) {
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) {
    const int e = lane + 32 * t;
    r.x[t] = e < D ? to_f(base[sum_index(bh, m, e, D, mt)]) : 0.f;
  }
}
template <int D>
__device__ __forceinline__ void wr_load_f(const float* __restrict__ p, WarpRow<D>& r, int lane) {
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) {
    const int e = lane + 32 * t;
    r.x[t] = e < D ? p[e] : 0.f;
  }
}
template <typename T, int D>
__device__ __forceinline__ void wr_store(T* p, const WarpRow<D>& r, int lane) {
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) {
    const int e = lane + 32 * t;
    if (e < D) p[e] = from_f<T>(r.x[t]);
  }
}
template <int D>
__device__ __forceinline__ float wr_dot(const WarpRow<D>& a, const WarpRow<D>& b) {
  float s = 0.f;
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) s = fmaf(a.x[t], b.x[t], s);
  return warp_sum(s);
}
// r <- R(c) r or R(c)^T r; the pair partner of dim e is e ^ 1, held by lane ^ 1.
template <int D>
__device__ __forceinline__ void wr_rotate(const pack3d_index& ix, const Coord& c, WarpRow<D>& r,
                                          int lane, float sign) {
  constexpr int DA = D / 3;
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) {
    const int e = lane + 32 * t;
    const float partner = __shfl_xor_sync(0xffffffffu, r.x[t], 1);
    if (e < D) {
      const int axis = e / DA, p = (e % DA) / 2;
      const float2 cs =
          rope_cs(ix.rope, ix.rope_rows, ix.rope_pairs, axis, coord_axis(c, axis), p);
      const float sn = sign * cs.y;
      // even e: x0' = x0 c - x1 s ; odd e: x1' = x0 s + x1 c
      r.x[t] = (e & 1) ? fmaf(partner, sn, r.x[t] * cs.x) : fmaf(-partner, sn, r.x[t] * cs.x);
    }
  }
}

// Group layout for the neighbour loops of the backward: kGL = 4 lanes per row, 8 rows per
// warp; lane g of a group owns the KD = d/4 consecutive dims [g KD, g KD + KD), read and
// written as 16-byte vectors (8-byte ones when a lane's share is 24 bytes). Dot products reduce
// over the 4 lanes in 2 shuffle steps, and every rotation pair (2p, 2p+1) stays in one lane.
constexpr int kGL = 4;
template <int D> struct GRow {
  static constexpr int KD = D / kGL;
  static_assert(KD % 2 == 0, "a lane must own whole rotation pairs");
  float x[KD];
};
// Bytes per vector access of a lane's KD elements of type T: the largest of 16, 8, 4 dividing
// the lane's share (the share starts on a multiple of it, as rows are 16-byte aligned).
template <typename T, int KD> constexpr int gr_chunk() {
  return (KD * (int)sizeof(T)) % 16 == 0 ? 16 : ((KD * (int)sizeof(T)) % 8 == 0 ? 8 : 4);
}
template <typename T> struct Unpack;
template <> struct Unpack<float> {
  __device__ __forceinline__ static void to_f(uint32_t w, float* x, int& n) { x[n++] = __uint_as_float(w); }
  __device__ __forceinline__ static uint32_t from_f(const float* x, int& n) { return __float_as_uint(x[n++]); }
};
template <> struct Unpack<__nv_bfloat16> {
  __device__ __forceinline__ static void to_f(uint32_t w, float* x, int& n) {
    x[n++] = __uint_as_float(w << 16);
    x[n++] = __uint_as_float(w & 0xffff0000u);
  }
  __device__ __forceinline__ static uint32_t from_f(const float* x, int& n) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[n], x[n + 1]);
    n += 2;
    return *reinterpret_cast<const uint32_t*>(&h);
  }
};
template <typename T, int D>
__device__ __forceinline__ void gr_load(const T* __restrict__ row, GRow<D>& r, int g) {
  constexpr int KD = GRow<D>::KD, CH = gr_chunk<T, KD>(), WORDS = CH / 4;
  const uint32_t* p = reinterpret_cast<const uint32_t*>(row + g * KD);
  int n = 0;
#pragma unroll
  for (int c = 0; c < KD * (int)sizeof(T) / CH; ++c) {
    uint32_t w[4];
    if (CH == 16) {
      const uint4 t = __ldg(reinterpret_cast<const uint4*>(p) + c);
      w[0] = t.x; w[1] = t.y; w[2] = t.z; w[3] = t.w;
    } else if (CH == 8) {
      const uint2 t = __ldg(reinterpret_cast<const uint2*>(p) + c);
      w[0] = t.x; w[1] = t.y;
    } else {
      w[0] = __ldg(p + c);
    }
#pragma unroll
    for (int k = 0; k < WORDS; ++k) Unpack<T>::to_f(w[k], r.x, n);
  }
}
template <typename T, int D>
__device__ __forceinline__ void gr_store(T* row, const GRow<D>& r, int g) {
  constexpr int KD = GRow<D>::KD, CH = gr_chunk<T, KD>(), WORDS = CH / 4;
  uint32_t* p = reinterpret_cast<uint32_t*>(row + g * KD);
  int n = 0;
#pragma unroll
  for (int c = 0; c < KD * (int)sizeof(T) / CH; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < WORDS; ++k) w[k] = Unpack<T>::from_f(r.x, n);
    if (CH == 16)
      reinterpret_cast<uint4*>(p)[c] = make_uint4(w[0], w[1], w[2], w[3]);
    else if (CH == 8)
      reinterpret_cast<uint2*>(p)[c] = make_uint2(w[0], w[1]);
    else
      p[c] = w[0];
  }
}
__device__ __forceinline__ float group_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}
template <int D>
__device__ __forceinline__ float gr_dot(const GRow<D>& a, const GRow<D>& b) {
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < GRow<D>::KD; ++k) s = fmaf(a.x[k], b.x[k], s);
  return group_sum(s);
}
// r <- R(c) r (sign 1) or R(c)^T r (sign -1)
template <int D>
__device__ __forceinline__ void gr_rotate(const pack3d_index& ix, const Coord& c, GRow<D>& r,
                                          int g, float sign) {
  constexpr int DA = D / 3;
#pragma unroll
  for (int k = 0; k < GRow<D>::KD; k += 2) {
    const int e = g * GRow<D>::KD + k;
    const int axis = e / DA, p = (e % DA) / 2;
    const float2 cs = rope_cs(ix.rope, ix.rope_rows, ix.rope_pairs, axis, coord_axis(c, axis), p);
    const float sn = sign * cs.y, x0 = r.x[k], x1 = r.x[k + 1];
    r.x[k] = x0 * cs.x - x1 * sn;
    r.x[k + 1] = x0 * sn + x1 * cs.x;
  }
}

// Row prologue, one pass over the rows of q, k, dO, o_loc and o_glob with 16-byte pieces: each
// row is read by a group of G lanes (G = C rounded up to a power of two, C = 16-byte pieces
// per row), a warp takes 32 / G rows at a time and the warps walk the rows persistently. The
// rotation table, read at every row's coordinate, sits in shared memory when it fits (a grid
// extent up to 170 at d = 96). The pair rotation is x0' = x0 c - x1 s, x1' = x0 s + x1 c with
// one rounding of the product and one of the fma, and the row sums reduce over the group's
// lanes with xor shuffles.
template <typename T, int D> struct PrepShape {
  static constexpr int kC = D / Vec<T>::E;
  static constexpr int kG = kC <= 8 ? 8 : (kC <= 16 ? 16 : 32);
};
constexpr int kPrepThreads = 256;
constexpr int kPrepTableMax = 65536;

template <typename T, int D>
__device__ __forceinline__ void prep_rotate(float (&x)[Vec<T>::E], const float2* cs) {
#pragma unroll
  for (int e = 0; e < Vec<T>::E; e += 2) {
    const float2 r = cs[e / 2];
    const float x0 = x[e], x1 = x[e + 1];
    x[e] = fmaf(-x1, r.y, x0 * r.x);
    x[e + 1] = fmaf(x0, r.y, x1 * r.x);
  }
}

template <typename T, int D, bool kTab>
__global__ void __launch_bounds__(kPrepThreads) k_bwd_prep(pack3d_index ix, const T* __restrict__ q,
                                                           const T* __restrict__ k,
                                                           const T* __restrict__ gate,
                                                           const T* __restrict__ o_loc,
                                                           const T* __restrict__ o_glob,
                                                           const T* __restrict__ dO, int64_t rows,
                                                           int kv_group, BwdWork w,
                                                           T* __restrict__ dgate) {
  constexpr int E = Vec<T>::E;
  constexpr int C = PrepShape<T, D>::kC, G = PrepShape<T, D>::kG, RPW = 32 / G;
  constexpr int DA = D / 3;
  static_assert(DA % E == 0, "a 16-byte piece must stay inside one axis third");
  extern __shared__ __align__(16) float prep_tab[];
  const float* rope = ix.rope;
  if constexpr (kTab) {
    const int n16 = 6 * ix.rope_rows * ix.rope_pairs / 4;
    for (int i = threadIdx.x; i < n16; i += blockDim.x)
      reinterpret_cast<float4*>(prep_tab)[i] = __ldg(reinterpret_cast<const float4*>(ix.rope) + i);
    __syncthreads();
    rope = prep_tab;
  }
  const int lane = threadIdx.x & 31, sub = lane / G, c = lane % G;
  const bool active = c < C;
  const int pc = active ? c : 0;  // an idle lane works on piece 0 and keeps nothing
  const int axis = (pc * E) / DA, p0 = ((pc * E) % DA) / 2;
  const float* tab_lane = rope + 2 * rope_slot(ix.rope_rows, ix.rope_pairs, axis, 0, p0);
  const int tab_row = 2 * ix.rope_pairs, csh = 20 - 10 * axis;
  const int64_t N = ix.n;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  T* qr = static_cast<T*>(w.qr);
  T* kr = static_cast<T*>(w.kr);
  for (int64_t r0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * RPW;
       r0 < rows; r0 += nwarps * RPW) {
    const int64_t row = r0 + sub;
    const bool live = row < rows;
    const bool ok = active && live;
    const int64_t i = live ? row % N : 0;
    const int64_t kvrow = kv_of(live ? row / N : 0, kv_group) * N + i;  // the key of the KV head
    float xq[E], xk[E], xd[E], xl[E], xg[E];
#pragma unroll
    for (int e = 0; e < E; ++e) xq[e] = xk[e] = xd[e] = xl[e] = xg[e] = 0.f;
    const int64_t off = (live ? row : 0) * D + pc * E;
    if (ok) {
      Vec<T>::load(q + off, xq);
      Vec<T>::load(k + kvrow * D + pc * E, xk);
      Vec<T>::load(dO + off, xd);
      Vec<T>::load(o_loc + off, xl);
      Vec<T>::load(o_glob + off, xg);
    }
    const int32_t cc = live ? __ldg(ix.coord + i) : 0;
    const float a = live ? to_f(gate[row]) : 0.f;
    // (cos, sin) of the piece's E / 2 pairs at the row's coordinate on this lane's axis
    float2 cs[E / 2];
    {
      const float4* cs4 = reinterpret_cast<const float4*>(tab_lane + tab_row * ((cc >> csh) & 1023));
#pragma unroll
      for (int h = 0; h < E / 4; ++h) {
        const float4 t4 = kTab ? cs4[h] : __ldg(cs4 + h);
        cs[2 * h] = make_float2(t4.x, t4.y);
        cs[2 * h + 1] = make_float2(t4.z, t4.w);
      }
    }
    prep_rotate<T, D>(xq, cs);
    prep_rotate<T, D>(xk, cs);
    const float g = 1.f / (1.f + expf(-a));
    float dl = 0.f, dgl = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dl = fmaf(xd[e], xl[e], dl);
      dgl = fmaf(xd[e], xg[e], dgl);
    }
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) {
      dl += __shfl_xor_sync(0xffffffffu, dl, o);
      dgl += __shfl_xor_sync(0xffffffffu, dgl, o);
    }
    if (ok) {
      Vec<T>::store(qr + off, xq);
      Vec<T>::store(kr + off, xk);
      if (w.dogb) {
        // tensor-core path: (1 - g) dO rows in bf16, an MMA operand (the rotated q is qr)
        uint32_t pk[E / 2];
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn((1.f - g) * xd[e], (1.f - g) * xd[e + 1]);
          pk[e / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        if constexpr (E == 8)
          *reinterpret_cast<uint4*>(w.dogb + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        else
          *reinterpret_cast<uint2*>(w.dogb + off) = make_uint2(pk[0], pk[1]);
      }
    }
    if (live && c == 0) {
      dgate[row] = from_f<T>((dl - dgl) * g * (1.f - g));
      w.Dl[row] = g * dl;
      w.Dg[row] = (1.f - g) * dgl;
    }
  }
}

template <typename T, int D, bool kTab>
cudaError_t launch_bwd_prep_as(const pack3d_index& ix, const T* q, const T* k, const T* gate,
                               const T* o_loc, const T* o_glob, const T* dO, int64_t rows,
                               int kv_group, const BwdWork& w, T* dgate, int smem,
                               cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t e =
      smem_attr_once(reinterpret_cast<const void*>(k_bwd_prep<T, D, kTab>), kPrepTableMax, attr_done);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_bwd_prep<T, D, kTab>, kPrepThreads,
                                                    smem);
  if (e != cudaSuccess) return e;
  occ = occ > 0 ? occ : 1;
  constexpr int RPW = 32 / PrepShape<T, D>::kG;
  const int64_t per_cta = (int64_t)(kPrepThreads / 32) * RPW;
  const int64_t need = (rows + per_cta - 1) / per_cta;
  const int64_t resident = (int64_t)occ * sm_count();
  const unsigned grid = (unsigned)(need < resident ? need : resident);
  if (grid == 0) return cudaSuccess;
  k_bwd_prep<T, D, kTab><<<grid, kPrepThreads, smem, s>>>(ix, q, k, gate, o_loc, o_glob, dO, rows,
                                                          kv_group, w, dgate);
  count_launch();
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_bwd_prep(const pack3d_index& ix, const T* q, const T* k, const T* gate,
                            const T* o_loc, const T* o_glob, const T* dO, int64_t rows,
                            int kv_group, const BwdWork& w, T* dgate, cudaStream_t s) {
  const int tab = 24 * ix.rope_rows * ix.rope_pairs;  // bytes: [3, rows, pairs] x (cos, sin)
  if (tab <= kPrepTableMax)
    return launch_bwd_prep_as<T, D, true>(ix, q, k, gate, o_loc, o_glob, dO, rows, kv_group, w,
                                          dgate, tab, s);
  return launch_bwd_prep_as<T, D, false>(ix, q, k, gate, o_loc, o_glob, dO, rows, kv_group, w,
                                         dgate, 0, s);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) k_bwd_dsum(pack3d_index ix, const T* __restrict__ ksum,
                                                  const T* __restrict__ vsum,
                                                  const T* __restrict__ gate,
                                                  const T* __restrict__ dO,
                                                  const float* __restrict__ lse_glob,
                                                  float scale, int exclude_near, int64_t bh_count,
                                                  int kv_group, BwdWork w) {
  const int lane = threadIdx.x & 31;
  const int64_t task = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t M = ix.m;
  if (task >= bh_count * M) return;
  const int64_t bh = task / M;
  const int m = (int)(task % M);
  WarpRow<D> km, vm, ak, av, x, d;
  wr_load_sum<T, D>(ksum, kv_of(bh, kv_group), m, sum_tiles(M), km, lane);
  wr_load_sum<T, D>(vsum, kv_of(bh, kv_group), m, sum_tiles(M), vm, lane);
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) ak.x[t] = av.x[t] = 0.f;
  for (int64_t i = 0; i < ix.n; ++i) {
    const int64_t row = bh * ix.n + i;
    const float lse = lse_glob[row];
    if (lse == -INFINITY) continue;
    if (exclude_near && block_is_near(ix, m, decode(ix.coord[i]))) continue;
    wr_load<T, D>(static_cast<const T*>(w.qr) + row * D, x, lane);
    wr_load<T, D>(dO + row * D, d, lane);
    const float g1 = 1.f - 1.f / (1.f + expf(-to_f(gate[row])));
    const float s = wr_dot<D>(x, km) * scale;
    const float p = expf(s - lse);
    const float dp = g1 * wr_dot<D>(d, vm);
    const float ds = p * (dp - w.Dg[row]) * scale;
#pragma unroll
    for (int t = 0; t < WarpRow<D>::KT; ++t) {
      ak.x[t] = fmaf(ds, x.x[t], ak.x[t]);
      av.x[t] = fmaf(p * g1, d.x[t], av.x[t]);
    }
  }
#pragma unroll
  for (int t = 0; t < WarpRow<D>::KT; ++t) {
    const int e = lane + 32 * t;
    if (e < D) {
      w.dks[task * D + e] = ak.x[t];
      w.dvs[task * D + e] = av.x[t];
    }
  }
}

// dq = R(c)^T (sum_j dS_ij k~_j + global part); kGL lanes per query row.
template <typename T, int D>
__global__ void __launch_bounds__(128, 4) k_bwd_dq(pack3d_index ix, const T* __restrict__ v,
                                                const T* __restrict__ ksum,
                                                const T* __restrict__ vsum,
                                                const T* __restrict__ gate,
                                                const T* __restrict__ dO,
                                                const float* __restrict__ lse_loc,
                                                const float* __restrict__ lse_glob, float scale,
                                                int exclude_near, int64_t rows, int kv_group,
                                                BwdWork w, T* __restrict__ dq) {
  const int g = threadIdx.x & (kGL - 1);
  const int64_t row0 = blockIdx.x * (int64_t)(blockDim.x / kGL) + threadIdx.x / kGL;
  const bool active = row0 < rows;  // inactive groups follow along on row 0 and store nothing
  const int64_t row = active ? row0 : 0;
  const int64_t bh = row / ix.n, i = row % ix.n;
  const int64_t rowbase = bh * ix.n, kvbase = kv_of(bh, kv_group) * ix.n;
  const Coord c = decode(ix.coord[i]);
  const float gt = 1.f / (1.f + expf(-to_f(gate[row])));
  const T* qr = static_cast<const T*>(w.qr);
  const T* kr = static_cast<const T*>(w.kr);
  GRow<D> q, d, acc, x, y;
  gr_load<T, D>(qr + row * D, q, g);
  gr_load<T, D>(dO + row * D, d, g);
#pragma unroll
  for (int k = 0; k < GRow<D>::KD; ++k) acc.x[k] = 0.f;
  // local branch
  const float ll = lse_loc[row], Dl = w.Dl[row];
  for (int o = 0; o < kNbr; ++o) {
    const int j = ix.nbr[i * kNbr + o];
    const int64_t rj = rowbase + (j >= 0 ? j : 0);
    gr_load<T, D>(kr + rj * D, x, g);
    gr_load<T, D>(v + (kvbase + (j >= 0 ? j : 0)) * D, y, g);
    const float sd = gr_dot<D>(q, x), dp = gr_dot<D>(d, y);
    const float p = j >= 0 ? expf(sd * scale - ll) : 0.f;
    const float ds = p * (gt * dp - Dl) * scale;
#pragma unroll
    for (int k = 0; k < GRow<D>::KD; ++k) acc.x[k] = fmaf(ds, x.x[k], acc.x[k]);
  }
  // global branch (computed by the tensor-core kernel into the workspace on that path)
  if (w.dqg) {
    gr_load<float, D>(w.dqg + row * D, x, g);
#pragma unroll
    for (int k = 0; k < GRow<D>::KD; ++k) acc.x[k] += x.x[k];
  } else {
    const float lg = lse_glob[row], Dg = w.Dg[row];
    if (lg != -INFINITY) {
      const int M = (int)ix.m;
      const int64_t mt = sum_tiles(M);
      for (int m = 0; m < M; ++m) {
        if (summary_empty(ix, m)) continue;
        if (exclude_near && block_is_near(ix, m, c)) continue;
#pragma unroll
        for (int k = 0; k < GRow<D>::KD; ++k) {
          const int e = g * GRow<D>::KD + k;
          x.x[k] = to_f(ksum[sum_index(kv_of(bh, kv_group), m, e, D, mt)]);
          y.x[k] = to_f(vsum[sum_index(kv_of(bh, kv_group), m, e, D, mt)]);
        }
        const float p = expf(gr_dot<D>(q, x) * scale - lg);
        const float ds = p * ((1.f - gt) * gr_dot<D>(d, y) - Dg) * scale;
#pragma unroll
        for (int k = 0; k < GRow<D>::KD; ++k) acc.x[k] = fmaf(ds, x.x[k], acc.x[k]);
      }
    }
  }
  gr_rotate<D>(ix, c, acc, g, -1.f);
  if (active) gr_store<T, D>(dq + row * D, acc, g);
}

// dk, dv of key j: gathered over its own neighbourhood (the 3x3x3 relation is symmetric, so
// no scatter/atomics) plus its weight in its summary's mean (1 / (members present in its block
// x non-empty blocks in its summary's group)) times the summary gradients; kGL lanes per
// key row. With summary-centre RoPE the summary's key gradient first goes back through the
// summary's rotation R(centre)^T and is added after the local part's inverse rotation. With
// GQA each query head's dk, dv go to float32 partials that k_bwd_gqa_reduce sums.
template <typename T, int D>
__global__ void __launch_bounds__(128, 4) k_bwd_dkv(pack3d_index ix, const T* __restrict__ v,
                                                 const T* __restrict__ gate,
                                                 const T* __restrict__ dO,
                                                 const float* __restrict__ lse_loc, float scale,
                                                 int64_t rows, int kv_group, BwdWork w,
                                                 T* __restrict__ dk, T* __restrict__ dv) {
  const int g = threadIdx.x & (kGL - 1);
  const int64_t row0 = blockIdx.x * (int64_t)(blockDim.x / kGL) + threadIdx.x / kGL;
  const bool active = row0 < rows;
  const int64_t row = active ? row0 : 0;
  const int64_t bh = row / ix.n, j = row % ix.n;
  const int64_t rowbase = bh * ix.n;
  const Coord c = decode(ix.coord[j]);
  const T* qr = static_cast<const T*>(w.qr);
  const T* kr = static_cast<const T*>(w.kr);
  GRow<D> kj, vj, ak, av, x, d;
  gr_load<T, D>(kr + row * D, kj, g);
  gr_load<T, D>(v + (kv_of(bh, kv_group) * ix.n + j) * D, vj, g);
#pragma unroll
  for (int k = 0; k < GRow<D>::KD; ++k) ak.x[k] = av.x[k] = 0.f;
  for (int o = 0; o < kNbr; ++o) {
    const int i = ix.nbr[j * kNbr + o];
    const int64_t ri = rowbase + (i >= 0 ? i : 0);
    gr_load<T, D>(qr + ri * D, x, g);
    gr_load<T, D>(dO + ri * D, d, g);
    const float gt = 1.f / (1.f + expf(-to_f(gate[ri])));
    const float sd = gr_dot<D>(x, kj), dp = gr_dot<D>(d, vj);
    const float p = i >= 0 ? expf(sd * scale - lse_loc[ri]) : 0.f;
    const float ds = p * (gt * dp - w.Dl[ri]) * scale;
#pragma unroll
    for (int k = 0; k < GRow<D>::KD; ++k) {
      ak.x[k] = fmaf(ds, x.x[k], ak.x[k]);
      av.x[k] = fmaf(p * gt, d.x[k], av.x[k]);
    }
  }
  // un-pool: the token's weight in its summary's (two-stage) mean times the summary's
  // gradient (per-query-range partials summed in range order)
  const int t = ix.sum_of[j];
  const float wt = 1.f / ((float)ix.count[ix.block_of[j]] * (float)ix.count2[t]);
  const int64_t part = (int64_t)(rows / ix.n) * ix.m * D;
  GRow<D> sk, sv;
#pragma unroll
  for (int k = 0; k < GRow<D>::KD; ++k) sk.x[k] = sv.x[k] = 0.f;
  for (int sp = 0; sp < w.nsplit; ++sp) {
    gr_load<float, D>(w.dks + sp * part + (bh * ix.m + t) * D, x, g);
    gr_load<float, D>(w.dvs + sp * part + (bh * ix.m + t) * D, d, g);
#pragma unroll
    for (int k = 0; k < GRow<D>::KD; ++k) {
      sk.x[k] += x.x[k];
      sv.x[k] += d.x[k];
    }
  }
#pragma unroll
  for (int k = 0; k < GRow<D>::KD; ++k) av.x[k] = fmaf(sv.x[k], wt, av.x[k]);
  if (ix.geom.summary_rope == PACK3D_ROPE_CENTRE) {
    gr_rotate<D>(ix, c, ak, g, -1.f);
    // R(centre_t)^T of the summary's key gradient, pair e/2 of dims (e, e+1)
    const float2* rc = reinterpret_cast<const float2*>(ix.rope_c) + (int64_t)t * (D / 2);
#pragma unroll
    for (int k = 0; k < GRow<D>::KD; k += 2) {
      const float2 cs = rc[(g * GRow<D>::KD + k) / 2];
      const float x0 = sk.x[k], x1 = sk.x[k + 1];
      ak.x[k] = fmaf(x0 * cs.x + x1 * cs.y, wt, ak.x[k]);
      ak.x[k + 1] = fmaf(x1 * cs.x - x0 * cs.y, wt, ak.x[k + 1]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < GRow<D>::KD; ++k) ak.x[k] = fmaf(sk.x[k], wt, ak.x[k]);
    gr_rotate<D>(ix, c, ak, g, -1.f);
  }
  if (active) {
    if (w.dkp) {
      gr_store<float, D>(w.dkp + row * D, ak, g);
      gr_store<float, D>(w.dvp + row * D, av, g);
    } else {
      gr_store<T, D>(dk + row * D, ak, g);
      gr_store<T, D>(dv + row * D, av, g);
    }
  }
}

// GQA: dk, dv of a KV head = the sum, in head order, of its query heads' float32 partials.
template <typename T>
__global__ void __launch_bounds__(256) k_bwd_gqa_reduce(const float* __restrict__ dkp,
                                                        const float* __restrict__ dvp,
                                                        int64_t kv_elems, int64_t per_head,
                                                        int kv_group, T* __restrict__ dk,
                                                        T* __restrict__ dv) {
  const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (e >= kv_elems) return;
  const int64_t bhk = e / per_head, off = e % per_head;
  float sk = 0.f, sv = 0.f;
  for (int gq = 0; gq < kv_group; ++gq) {
    const int64_t src = (bhk * kv_group + gq) * per_head + off;
    sk += dkp[src];
    sv += dvp[src];
  }
  dk[e] = from_f<T>(sk);
  dv[e] = from_f<T>(sv);
}

// ------------------------------------------------------------------------------ launchers
size_t bwd_workspace_bytes(const pack3d_index& ix, int64_t bh, int dtype, bool tc,
                           int kv_group) {
  return bwd_workspace_bytes_for(ix, bh, dtype == PACK3D_BF16 ? 2 : 4, tc, kv_group);
}

cudaError_t bwd_tc_dispatch(const pack3d_index& ix, const BwdWork& w, const void* ksum,
                            const void* vsum, const float* lse_glob, int64_t bh, int kv_group,
                            float scale, int excl, cudaStream_t s);
cudaError_t bwd_local_dq_tc_dispatch(const pack3d_index& ix, const BwdWork& w, const void* v,
                                     const void* dO, const void* gate, const float* lse_loc,
                                     int64_t bh, int kv_group, float scale, void* dq,
                                     cudaStream_t s);
cudaError_t bwd_local_dkv_tc_dispatch(const pack3d_index& ix, const BwdWork& w, const void* v,
                                      const void* dO, const void* gate, const float* lse_loc,
                                      int64_t bh, int kv_group, float scale, void* dk, void* dv,
                                      cudaStream_t s);

template <typename T, int D>
cudaError_t bwd_simt(const pack3d_index& ix, const void* q, const void* k, const void* v,
                     const void* gate, const void* ksum, const void* vsum, const void* o_loc,
                     const void* o_glob, const float* lse_loc, const float* lse_glob,
                     const void* dO, int64_t bh, int kv_group, float scale, int excl, void* dq,
                     void* dk, void* dv, void* dgate, void* ws, bool tc, cudaStream_t s) {
  const BwdWork w = bwd_carve(ix, bh, ws, sizeof(T), tc, kv_group);
  const int64_t rows = bh * ix.n;
  const unsigned mb = (unsigned)((bh * ix.m + 3) / 4);
  const T* tq = static_cast<const T*>(q);
  const T* tk = static_cast<const T*>(k);
  const T* tv = static_cast<const T*>(v);
  const T* tg = static_cast<const T*>(gate);
  const T* tdo = static_cast<const T*>(dO);
  {
    const cudaError_t e = launch_bwd_prep<T, D>(ix, tq, tk, tg, static_cast<const T*>(o_loc),
                                                static_cast<const T*>(o_glob), tdo, rows,
                                                kv_group, w, static_cast<T*>(dgate), s);
    if (e != cudaSuccess) return e;
  }
  if (tc) {
    // the global branch's summary gradients and its part of dq on tensor cores
    const cudaError_t e =
        bwd_tc_dispatch(ix, w, ksum, vsum, lse_glob, bh, kv_group, scale, excl, s);
    if (e != cudaSuccess) return e;
  } else {
    k_bwd_dsum<T, D><<<mb, 128, 0, s>>>(ix, static_cast<const T*>(ksum),
                                         static_cast<const T*>(vsum), tg, tdo, lse_glob, scale,
                                         excl, bh, kv_group, w);
    count_launch();
  }
  const unsigned gb = (unsigned)((rows + 128 / kGL - 1) / (128 / kGL));  // kGL lanes per row
  if (tc) {
    // bf16: the local branch on tensor cores -- dq~ plus the global part, R(c)^T -> dq; dk~, dv
    // plus the un-pooled summary gradients, R(c)^T -> dk
    cudaError_t e =
        bwd_local_dq_tc_dispatch(ix, w, v, dO, gate, lse_loc, bh, kv_group, scale, dq, s);
    if (e != cudaSuccess) return e;
    e = bwd_local_dkv_tc_dispatch(ix, w, v, dO, gate, lse_loc, bh, kv_group, scale, dk, dv, s);
    if (e != cudaSuccess) return e;
  } else {
    k_bwd_dq<T, D><<<gb, 128, 0, s>>>(ix, tv, static_cast<const T*>(ksum),
                                       static_cast<const T*>(vsum), tg, tdo, lse_loc, lse_glob,
                                       scale, excl, rows, kv_group, w, static_cast<T*>(dq));
    k_bwd_dkv<T, D><<<gb, 128, 0, s>>>(ix, tv, tg, tdo, lse_loc, scale, rows, kv_group, w,
                                        static_cast<T*>(dk), static_cast<T*>(dv));
    count_launch(2);
  }
  if (kv_group > 1) {
    const int64_t kv_elems = rows / kv_group * D;
    k_bwd_gqa_reduce<T><<<(unsigned)((kv_elems + 255) / 256), 256, 0, s>>>(
        w.dkp, w.dvp, kv_elems, ix.n * (int64_t)D, kv_group, static_cast<T*>(dk),
        static_cast<T*>(dv));
    count_launch();
  }
  return cudaGetLastError();
}

// Global branch + mixer only, over a given local output (which `o` may alias).
cudaError_t global_simt_dispatch(const pack3d_index& ix, const void* q, const void* gate,
                                 const void* ksum, const void* vsum, const void* o_loc,
                                 int dtype, int64_t bh, int kv_group, float scale, int excl,
                                 void* o, float* lse_glob, void* o_glob, cudaStream_t s) {
  const dim3 grid((unsigned)((ix.n + 127) / 128), (unsigned)bh);
  const int d = ix.geom.head_dim;
#define P3D_GLB(T, D)                                                                          \
  k_global_fwd<T, D, 32><<<grid, 128, 0, s>>>(                                                 \
      ix, static_cast<const T*>(q), static_cast<const T*>(ksum), static_cast<const T*>(vsum), \
      static_cast<const T*>(gate), static_cast<const T*>(o_loc), scale, excl, kv_group,       \
      static_cast<T*>(o), lse_glob, static_cast<T*>(o_glob))
  if (dtype == PACK3D_BF16) {
    if (d == 96) P3D_GLB(__nv_bfloat16, 96); else P3D_GLB(__nv_bfloat16, 48);
  } else {
    if (d == 96) P3D_GLB(float, 96); else P3D_GLB(float, 48);
  }
#undef P3D_GLB
  count_launch();
  return cudaGetLastError();
}

cudaError_t local_simt_dispatch(const pack3d_index& ix, const void* q, const void* k,
                                const void* v, int dtype, int64_t bh, int kv_group, float scale,
                                void* o_loc, float* lse_loc, cudaStream_t s) {
  const dim3 grid((unsigned)((ix.n + 127) / 128), (unsigned)bh);
  const int d = ix.geom.head_dim;
#define P3D_LOC(T, D)                                                                         \
  k_local_fwd<T, D><<<grid, 128, 0, s>>>(ix, static_cast<const T*>(q), static_cast<const T*>(k), \
                                          static_cast<const T*>(v), scale, kv_group,           \
                                          static_cast<T*>(o_loc), lse_loc)
  if (dtype == PACK3D_BF16) {
    if (d == 96) P3D_LOC(__nv_bfloat16, 96); else P3D_LOC(__nv_bfloat16, 48);
  } else {
    if (d == 96) P3D_LOC(float, 96); else P3D_LOC(float, 48);
  }
#undef P3D_LOC
  count_launch();
  return cudaGetLastError();
}

cudaError_t bwd_simt_dispatch(const pack3d_index& ix, const void* q, const void* k,
                              const void* v, const void* gate, const void* ksum,
                              const void* vsum, const void* o_loc, const void* o_glob,
                              const float* lse_loc, const float* lse_glob, const void* dO,
                              int dtype, int64_t bh, int kv_group, float scale, int excl,
                              void* dq, void* dk, void* dv, void* dgate, void* ws, bool tc,
                              cudaStream_t s) {
  const int d = ix.geom.head_dim;
#define P3D_BWD(T, D)                                                                         \
  bwd_simt<T, D>(ix, q, k, v, gate, ksum, vsum, o_loc, o_glob, lse_loc, lse_glob, dO, bh,      \
                 kv_group, scale, excl, dq, dk, dv, dgate, ws, tc, s)
  if (dtype == PACK3D_BF16) return d == 96 ? P3D_BWD(__nv_bfloat16, 96) : P3D_BWD(__nv_bfloat16, 48);
  return d == 96 ? P3D_BWD(float, 96) : P3D_BWD(float, 48);
#undef P3D_BWD
}

}  // namespace p3d
