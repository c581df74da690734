// Block summaries (project page "Geometry Matters in Packed 3D Attention", Chapter 3 "Rotate
// first, then pool"; paper summary §3.2 and §B.5), written in summary tiles (see sum_index in
// common.cuh; the tail of the last tile is written as zeros).
//
//   block mean   Kb[m] = (1/|S_m|) sum_{s} R(c_j) k[b,h,j],  Vb[m] = (1/|S_m|) sum_{s} v[b,h,j]
//                with j = members[m][s] (canonical slot s), over the members present;
//   summary      ksum[t] = (1/count2[t]) sum over the non-empty blocks m of group t of Kb[m]
//                (second pooling stage, note under Figure 1 of the project page; with no
//                second stage each group is one block), likewise vsum.
// Summary-centre RoPE (project page Ch.3 "One block, two ways to summarize it"; paper summary
// §B.7-§B.8): the unrotated keys are pooled the same way and ksum[t] is rotated once by the
// angles of the centre of t's box (rope_c table). An empty summary is written as zeros.
//
// With a k_rot buffer the rotated key rows R(c_j) k[b,h,j] are written out as well (every
// token is the member of exactly one block, so each row is written once), for the local branch
// to gather without rotating.
//
// HBM-bound: every k and v row is read exactly once with 16-byte vector loads. One warp per
// summary: lane l handles 16-byte chunk (l % C) of member rows s = l / C, l / C + R, ...
// (C chunks per row, R = 32 / C rows per pass); the R partial sums are then combined in fixed
// order with warp shuffles. Absent members (and the zero padding of the last summary tile)
// contribute with weight 0. The summation order depends on canonical slots and group slots
// only, never on memory slots, so a coordinate-carrying repack gives bit-identical summaries.
#include "common.cuh"
#include "launch.h"
#include "vec.cuh"

namespace p3d {

template <typename T, int D>
__global__ void __launch_bounds__(128, 6) k_summarize(pack3d_index ix, const T* __restrict__ k,
                                                   const T* __restrict__ v, int64_t bh_count,
                                                   T* __restrict__ ksum, T* __restrict__ vsum,
                                                   T* __restrict__ krot) {
  constexpr int E = Vec<T>::E;
  constexpr int C = D / E;       // chunks per row
  constexpr int R = 32 / C;      // member rows per pass
  constexpr int DA = D / 3;      // axis third
  static_assert(DA % E == 0, "a 16-byte chunk must stay inside one axis third");
  const int lane = threadIdx.x & 31;
  const int64_t task = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t M = ix.m;
  const int64_t MT = sum_tiles(M);
  if (task >= bh_count * MT * 64) return;
  const int64_t bh = task / (MT * 64);
  const int m = (int)(task % (MT * 64));  // m >= M: zero padding of the last tile
  const int vol = ix.block_volume, gv = ix.group_volume;
  const bool centre = ix.geom.summary_rope == PACK3D_ROPE_CENTRE;
  const int r = lane / C, c = lane % C;
  const bool active = r < R;
  const int axis = (c * E) / DA;
  const int p0 = ((c * E) % DA) / 2;

  float ak[E], av[E];
#pragma unroll
  for (int e = 0; e < E; ++e) ak[e] = av[e] = 0.f;

  const T* kb = k + bh * ix.n * D;
  const T* vb = v + bh * ix.n * D;
  for (int t = 0; t < gv; ++t) {
    // the group's block t (warp-uniform); without a second stage the block is the summary
    // itself, so no table lookup stands before the member loads
    const int blk = m < M ? (gv == 1 ? m : ix.groups[(int64_t)m * gv + t]) : -1;
    if (blk < 0) continue;
    // each member present carries 1 / (members present in the block): the sum over the
    // block's members is then its mean (the count's load overlaps the member loads)
    const int cnt = ix.count[blk];
    const float inv = cnt > 0 ? 1.0f / (float)cnt : 0.f;
    // Members are taken 32 at a time: lane l fetches the slot and coordinate of member b0 + l
    // once, and every lane then reads them by shuffle, so the 16-byte k/v loads of many
    // members are independent and in flight together (the loop body has no branch).
    for (int b0 = 0; b0 < vol; b0 += 32) {
      int jl = -1;
      int32_t cl = 0;
      if (b0 + lane < vol) {
        jl = ix.members[(int64_t)blk * vol + b0 + lane];
        if (jl >= 0) cl = ix.coord[jl];
      }
#pragma unroll 8
      for (int i = 0; i < (32 + R - 1) / R; ++i) {
        const int sl = r + R * i;  // member b0 + sl, canonical-slot order within this lane
        const int j = __shfl_sync(0xffffffffu, jl, sl & 31);
        const int32_t cc = __shfl_sync(0xffffffffu, cl, sl & 31);
        const bool use = active && sl < 32 && b0 + sl < vol && j >= 0;
        const int64_t row = use ? j : 0;
        const float wgt = use ? inv : 0.f;
        const int cv = coord_axis(decode(cc), axis);
        float xk[E], xv[E], rk[E];
        Vec<T>::load(kb + row * D + c * E, xk);
        Vec<T>::load(vb + row * D + c * E, xv);
        // (cos, sin) of the piece's E / 2 rotation pairs: E * 4 contiguous bytes of the table
        // (p0 is a multiple of E / 2, so the 16-byte loads are aligned)
        float2 csv[E / 2];
        {
          const float4* cs4 = reinterpret_cast<const float4*>(
              ix.rope + 2 * rope_slot(ix.rope_rows, ix.rope_pairs, axis, use ? cv : 0, p0));
#pragma unroll
          for (int h = 0; h < E / 4; ++h) {
            const float4 t4 = __ldg(cs4 + h);
            csv[2 * h] = make_float2(t4.x, t4.y);
            csv[2 * h + 1] = make_float2(t4.z, t4.w);
          }
        }
#pragma unroll
        for (int e = 0; e < E; e += 2) {
          const float2 cs = csv[e / 2];
          rk[e] = xk[e] * cs.x - xk[e + 1] * cs.y;
          rk[e + 1] = xk[e] * cs.y + xk[e + 1] * cs.x;
          ak[e] = fmaf(wgt, centre ? xk[e] : rk[e], ak[e]);
          ak[e + 1] = fmaf(wgt, centre ? xk[e + 1] : rk[e + 1], ak[e + 1]);
          av[e] = fmaf(wgt, xv[e], av[e]);
          av[e + 1] = fmaf(wgt, xv[e + 1], av[e + 1]);
        }
        if (krot && use) Vec<T>::store(krot + bh * ix.n * D + row * D + c * E, rk);
      }
    }
  }
  // combine the R partial sums in the fixed order r = 0, 1, ..., R-1 (each lane's own
  // partials are read, never a value already combined in an earlier step)
  float pk[E], pv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    pk[e] = ak[e];
    pv[e] = av[e];
  }
#pragma unroll
  for (int rr = 1; rr < R; ++rr) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      ak[e] += __shfl_sync(0xffffffffu, pk[e], (lane + rr * C) & 31);
      av[e] += __shfl_sync(0xffffffffu, pv[e], (lane + rr * C) & 31);
    }
  }
  if (r == 0) {
    const int cnt2 = m < M ? ix.count2[m] : 0;
    const float inv = cnt2 > 0 ? 1.0f / (float)cnt2 : 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      ak[e] *= inv;
      av[e] *= inv;
    }
    if (centre && m < M) {
      // rotate the pooled key once, by the angles of the summary's box centre
      const float2* rc = reinterpret_cast<const float2*>(ix.rope_c) + (int64_t)m * (D / 2);
#pragma unroll
      for (int e = 0; e < E; e += 2) {
        const float2 cs = rc[(c * E + e) / 2];
        const float x0 = ak[e], x1 = ak[e + 1];
        ak[e] = x0 * cs.x - x1 * cs.y;
        ak[e + 1] = x0 * cs.y + x1 * cs.x;
      }
    }
    Vec<T>::store(ksum + sum_index(bh, m, c * E, D, MT), ak);
    Vec<T>::store(vsum + sum_index(bh, m, c * E, D, MT), av);
  }
}

template <typename T, int D>
cudaError_t launch_summarize(const pack3d_index& ix, const void* k, const void* v, int64_t bh,
                             void* ksum, void* vsum, void* krot, cudaStream_t s) {
  const int64_t tasks = bh * sum_tiles(ix.m) * 64;
  const unsigned blocks = (unsigned)((tasks + 3) / 4);
  k_summarize<T, D><<<blocks, 128, 0, s>>>(ix, static_cast<const T*>(k), static_cast<const T*>(v),
                                            bh, static_cast<T*>(ksum), static_cast<T*>(vsum),
                                            static_cast<T*>(krot));
  count_launch();
  return cudaGetLastError();
}

// krot may be null (summaries only)
cudaError_t summarize_dispatch(const pack3d_index& ix, const void* k, const void* v, int dtype,
                               int64_t bh, void* ksum, void* vsum, void* krot, cudaStream_t s) {
  const int d = ix.geom.head_dim;
  if (dtype == PACK3D_BF16) {
    if (d == 96) return launch_summarize<__nv_bfloat16, 96>(ix, k, v, bh, ksum, vsum, krot, s);
    return launch_summarize<__nv_bfloat16, 48>(ix, k, v, bh, ksum, vsum, krot, s);
  }
  if (d == 96) return launch_summarize<float, 96>(ix, k, v, bh, ksum, vsum, krot, s);
  return launch_summarize<float, 48>(ix, k, v, bh, ksum, vsum, krot, s);
}

}  // namespace p3d
