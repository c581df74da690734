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
// HBM-bound: every k and v row is read exactly once. Each warp is persistent and walks the
// summaries w, w + (warps in the grid), ... as one stream of member chunks (CH = 16 canonical
// slots, 32 when R below does not divide 16; a block of more members is several chunks, and
// with a second stage the group's blocks follow each other). A chunk's k and v rows are staged
// into the warp's shared memory by 16-byte cp.async copies (absent members are zero-filled
// without a read), double-buffered: while the warp sums chunk f the rows of chunk f + 1 are in
// flight, and the table lookups of chunks f + 2 (member slots) and f + 3 (group slot) are issued
// ahead, so no load sits on the warp's path. The rotation table, read for every member row,
// is copied into shared memory once per CTA when it fits (up to 64 KB; a larger table is read
// through L1). The sum itself: lane l handles 16-byte piece
// (l % C) of member rows s = l / C, l / C + R, ... (C pieces per row, R = 32 / C rows per pass);
// the R partial sums are then combined in fixed order with warp shuffles. Absent members (and
// the zero padding of the last summary tile) are zero rows. The summation order depends on
// canonical slots and group slots only, never on memory slots, so a coordinate-carrying repack
// gives bit-identical summaries.
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "vec.cuh"

namespace p3d {

// One member chunk on its way through a warp's pipeline.
struct SumChunk {
  int64_t bh;   // (batch, KV head) of the chunk's summary
  int m;        // summary within the head (m >= M: zero padding of the last tile)
  int b;        // chunk within the block
  int blk;      // first-stage block (-1: none)
  bool last;    // last chunk of its summary
  int jl;       // slot of member CH b + lane (-1: absent or lane >= CH)
  int32_t cl;   // its packed coordinate (0 when absent)
  float inv;    // 1 / (members present in the block), 0 for an empty block
};

template <typename T, int D>
struct SumShape {
  static constexpr int kC = D / Vec<T>::E;             // 16-byte pieces per row
  static constexpr int kR = 32 / kC;                   // member rows per pass
  static constexpr int kCH = 16 % kR == 0 ? 16 : 32;   // members per chunk
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kTileBytes = kCH * kRowBytes;   // one tensor's rows of a chunk
  static constexpr int kBufBytes = 2 * kTileBytes;     // k and v
  static constexpr int kWarpBytes = 2 * kBufBytes;     // double-buffered
  // warps per CTA at most (16 keeps the registers at 128 a thread)
  static constexpr int kMaxWarps = kWarpBytes <= 12288 ? 16 : 8;
};

// The rotation table is copied into each CTA's shared memory when it is at most this large
// (a grid extent up to 170 at d = 96); a larger table is read through the L1 cache.
constexpr int kSumTableSmemMax = 65536;
constexpr int kSumSmemMax = 232448;  // dynamic shared memory of one CTA at most

// kTab: the rotation table sits in shared memory (after the warps' staging buffers);
// kCentre: summary-centre RoPE (the unrotated keys are pooled).
template <typename T, int D, bool kTab, bool kCentre>
__global__ void __launch_bounds__(32 * SumShape<T, D>::kMaxWarps, 1)
    k_summarize(pack3d_index ix, const T* __restrict__ k, const T* __restrict__ v,
                int64_t bh_count, T* __restrict__ ksum, T* __restrict__ vsum,
                T* __restrict__ krot) {
  using S = SumShape<T, D>;
  constexpr int E = Vec<T>::E;
  constexpr int C = S::kC;
  constexpr int R = S::kR;
  constexpr int CH = S::kCH;
  constexpr int DA = D / 3;      // axis third
  static_assert(DA % E == 0, "a 16-byte chunk must stay inside one axis third");
  static_assert((CH * C) % 32 == 0, "a chunk's pieces must spread evenly over the lanes");
  extern __shared__ __align__(16) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int W = blockDim.x >> 5;
  uint8_t* const wbuf = smem + (threadIdx.x >> 5) * S::kWarpBytes;
  const int64_t M = ix.m;
  const int64_t MT = sum_tiles(M);
  const int64_t per_bh = MT * 64;
  const int64_t tasks = bh_count * per_bh;
  const int64_t nwarps = (int64_t)gridDim.x * W;
  const int64_t w0 = (int64_t)blockIdx.x * W + (threadIdx.x >> 5);
  const float* rope = ix.rope;
  if constexpr (kTab) {
    // every member row needs (cos, sin) at its own coordinate: the table is read ~D / 2 times
    // per row, so it is served from shared memory
    float* tab = reinterpret_cast<float*>(smem + W * S::kWarpBytes);
    const int n16 = 6 * ix.rope_rows * ix.rope_pairs / 4;  // 16-byte pieces of the table
    for (int i = threadIdx.x; i < n16; i += blockDim.x)
      reinterpret_cast<float4*>(tab)[i] = __ldg(reinterpret_cast<const float4*>(ix.rope) + i);
    __syncthreads();
    rope = tab;
  }
  if (w0 >= tasks) return;
  const int vol = ix.block_volume, gv = ix.group_volume;
  const int nb = (vol + CH - 1) / CH;
  const int64_t nchunks = ((tasks - 1 - w0) / nwarps + 1) * (int64_t)(gv * nb);
  const int r = lane / C, c = lane % C;
  const bool active = r < R;
  const int axis = (c * E) / DA;
  const int p0 = ((c * E) % DA) / 2;
  // this lane's (cos, sin) pairs p0 .. p0 + E/2 - 1 of its axis: row cv of the axis starts
  // 2 * pairs * cv floats on (the coordinate field of the axis sits at bit 20 - 10 * axis)
  const float* tab_lane = rope + 2 * rope_slot(ix.rope_rows, ix.rope_pairs, axis, 0, p0);
  const int tab_row = 2 * ix.rope_pairs;
  const int csh = 20 - 10 * axis;
  const int64_t nd = ix.n * D;

  // cursor of the chunk stream (task, group slot, chunk within the block)
  int64_t a_task = w0;
  int a_t = 0, a_b = 0;
  // group slot and summary of the next chunk of the stream
  auto stage_a = [&](SumChunk& x) {
    x.bh = a_task / per_bh;
    x.m = (int)(a_task - x.bh * per_bh);
    x.b = a_b;
    x.last = a_t == gv - 1 && a_b == nb - 1;
    x.blk = x.m < M ? (gv == 1 ? x.m : ix.groups[(int64_t)x.m * gv + a_t]) : -1;
    if (++a_b == nb) {
      a_b = 0;
      if (++a_t == gv) {
        a_t = 0;
        a_task += nwarps;
      }
    }
  };
  // member slot of lane's member
  auto stage_b = [&](SumChunk& x) {
    const int s = x.b * CH + lane;
    x.jl = (x.blk >= 0 && lane < CH && s < vol) ? ix.members[(int64_t)x.blk * vol + s] : -1;
  };
  // the rows' copies into `buf`, the members' coordinates and the block's weight
  auto stage_c = [&](SumChunk& x, uint8_t* buf) {
    const T* kg = k + x.bh * nd;
    const T* vg = v + x.bh * nd;
#pragma unroll
    for (int i = 0; i < CH * C / 32; ++i) {
      const int p = lane + 32 * i;  // piece (member sm, 16-byte column q) of the chunk
      const int sm = p / C, q = p - (p / C) * C;
      const int j = __shfl_sync(0xffffffffu, x.jl, sm);
      const int64_t row = j >= 0 ? j : 0;
      tc::cp_async16(buf + sm * S::kRowBytes + q * 16, kg + row * D + q * E, j >= 0);
      tc::cp_async16(buf + S::kTileBytes + sm * S::kRowBytes + q * 16, vg + row * D + q * E,
                     j >= 0);
    }
    x.cl = x.jl >= 0 ? ix.coord[x.jl] : 0;
    const int cnt = x.blk >= 0 ? ix.count[x.blk] : 0;
    x.inv = cnt > 0 ? 1.0f / (float)cnt : 0.f;
  };

  float ak[E], av[E];
#pragma unroll
  for (int e = 0; e < E; ++e) ak[e] = av[e] = 0.f;

  SumChunk s0, s1, s2, s3;
  stage_a(s0);
  if (nchunks > 1) stage_a(s1);
  if (nchunks > 2) stage_a(s2);
  stage_b(s0);
  if (nchunks > 1) stage_b(s1);
  stage_c(s0, wbuf);
  tc::cp_async_commit();
  for (int64_t f = 0; f < nchunks; ++f) {
    if (f + 1 < nchunks) stage_c(s1, wbuf + ((f + 1) & 1) * S::kBufBytes);
    tc::cp_async_commit();
    if (f + 2 < nchunks) stage_b(s2);
    if (f + 3 < nchunks) stage_a(s3);
    tc::cp_async_wait_group<1>();
    __syncwarp();
    // sum chunk f: rows in canonical-slot order within this lane. An absent member's rows are
    // zeros, so it adds exactly nothing (x + w * 0 = x; no partial sum is ever -0); a lane past
    // the chunk's last row (when R does not divide CH) reads row 0 with weight 0.
    const T* ks = reinterpret_cast<const T*>(wbuf + (f & 1) * S::kBufBytes);
    const T* vs = reinterpret_cast<const T*>(wbuf + (f & 1) * S::kBufBytes + S::kTileBytes);
    T* kr = krot ? krot + s0.bh * nd : nullptr;
    const float w = s0.inv;
#pragma unroll 4
    for (int i = 0; i < (CH + R - 1) / R; ++i) {
      const int sl = r + R * i;
      const bool row_ok = active && sl < CH;
      const int src = row_ok ? sl : 0;
      const float wr = row_ok ? w : 0.f;
      const int j = __shfl_sync(0xffffffffu, s0.jl, src);
      const int32_t cc = __shfl_sync(0xffffffffu, s0.cl, src);
      float xk[E], xv[E], rk[E];
      Vec<T>::load_shared(ks + src * D + c * E, xk);
      Vec<T>::load_shared(vs + src * D + c * E, xv);
      // (cos, sin) of the piece's E / 2 rotation pairs: E * 4 contiguous bytes of the table
      // (p0 is a multiple of E / 2, so the 16-byte loads are aligned); an absent member has
      // coordinate 0
      float2 csv[E / 2];
      {
        const float4* cs4 =
            reinterpret_cast<const float4*>(tab_lane + tab_row * ((cc >> csh) & 1023));
#pragma unroll
        for (int h = 0; h < E / 4; ++h) {
          const float4 t4 = kTab ? cs4[h] : __ldg(cs4 + h);
          csv[2 * h] = make_float2(t4.x, t4.y);
          csv[2 * h + 1] = make_float2(t4.z, t4.w);
        }
      }
#pragma unroll
      for (int e = 0; e < E; e += 2) {
        const float2 cs = csv[e / 2];
        rk[e] = xk[e] * cs.x - xk[e + 1] * cs.y;
        rk[e + 1] = xk[e] * cs.y + xk[e + 1] * cs.x;
        ak[e] = fmaf(wr, kCentre ? xk[e] : rk[e], ak[e]);
        ak[e + 1] = fmaf(wr, kCentre ? xk[e + 1] : rk[e + 1], ak[e + 1]);
        av[e] = fmaf(wr, xv[e], av[e]);
        av[e + 1] = fmaf(wr, xv[e + 1], av[e + 1]);
      }
      if (kr && row_ok && j >= 0) Vec<T>::store(kr + (int64_t)j * D + c * E, rk);
    }
    if (s0.last) {
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
      const int m = s0.m;
      if (r == 0) {
        const int cnt2 = m < M ? ix.count2[m] : 0;
        const float inv = cnt2 > 0 ? 1.0f / (float)cnt2 : 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          ak[e] *= inv;
          av[e] *= inv;
        }
        if (kCentre && m < M) {
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
        Vec<T>::store(ksum + sum_index(s0.bh, m, c * E, D, MT), ak);
        Vec<T>::store(vsum + sum_index(s0.bh, m, c * E, D, MT), av);
      }
#pragma unroll
      for (int e = 0; e < E; ++e) ak[e] = av[e] = 0.f;
    }
    // every lane is done with this buffer before chunk f + 2's copies refill it
    __syncwarp();
    s0 = s1;
    s1 = s2;
    s2 = s3;
  }
}

template <typename T, int D, bool kTab, bool kCentre>
cudaError_t launch_summarize_as(const pack3d_index& ix, const void* k, const void* v, int64_t bh,
                                void* ksum, void* vsum, void* krot, int warps, int smem,
                                cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  const void* fn = reinterpret_cast<const void*>(k_summarize<T, D, kTab, kCentre>);
  cudaError_t e = smem_attr_once(fn, kSumSmemMax, attr_done);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_summarize<T, D, kTab, kCentre>,
                                                    32 * warps, smem);
  if (e != cudaSuccess) return e;
  occ = occ > 0 ? occ : 1;
  // persistent: at most one wave of CTAs, each warp walks its share of the summaries
  const int64_t tasks = bh * sum_tiles(ix.m) * 64;
  const int64_t need = (tasks + warps - 1) / warps;
  const int64_t resident = (int64_t)occ * sm_count();
  const unsigned blocks = (unsigned)(need < resident ? need : resident);
  if (blocks == 0) return cudaSuccess;
  k_summarize<T, D, kTab, kCentre><<<blocks, 32 * warps, smem, s>>>(
      ix, static_cast<const T*>(k), static_cast<const T*>(v), bh, static_cast<T*>(ksum),
      static_cast<T*>(vsum), static_cast<T*>(krot));
  count_launch();
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_summarize(const pack3d_index& ix, const void* k, const void* v, int64_t bh,
                             void* ksum, void* vsum, void* krot, cudaStream_t s) {
  using S = SumShape<T, D>;
  const int tab = 24 * ix.rope_rows * ix.rope_pairs;  // bytes: [3, rows, pairs] x (cos, sin)
  const bool in_smem = tab <= kSumTableSmemMax;
  const int room = kSumSmemMax - (in_smem ? tab : 0);
  // with the rotated keys written as well, 12 warps of 16 share the SM's memory traffic best
  // (65,536- and 262,144-token fields); the summaries alone run best with 16
  const int cap = (krot && S::kMaxWarps == 16) ? 12 : S::kMaxWarps;
  int warps = room / S::kWarpBytes;
  warps = warps > cap ? cap : warps;
  const int smem = warps * S::kWarpBytes + (in_smem ? tab : 0);
  const bool centre = ix.geom.summary_rope == PACK3D_ROPE_CENTRE;
  if (in_smem)
    return centre ? launch_summarize_as<T, D, true, true>(ix, k, v, bh, ksum, vsum, krot, warps,
                                                          smem, s)
                  : launch_summarize_as<T, D, true, false>(ix, k, v, bh, ksum, vsum, krot,
                                                           warps, smem, s);
  return centre ? launch_summarize_as<T, D, false, true>(ix, k, v, bh, ksum, vsum, krot, warps,
                                                         smem, s)
                : launch_summarize_as<T, D, false, false>(ix, k, v, bh, ksum, vsum, krot, warps,
                                                          smem, s);
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
