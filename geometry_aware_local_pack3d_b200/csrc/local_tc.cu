// Local branch of PACK3D attention on tcgen05 tensor cores (bf16 I/O, head_dim 48 or 96).
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 1: each query
// attends exactly to every token of its 3x3x3 coordinate neighbourhood (at most 27, fewer at
// the border), found by coordinate, never by adjacency in memory; paper summary §3.5: streamed
// online softmax, no gathered neighbour tensor in memory.
//
// Work unit: one 8x4x4 (z, y, x) coordinate brick of 128 queries of one (batch, head). A CTA
// (4 softmax warps, 3 gather warps, 1 MMA warp) is persistent and walks bricks with a grid
// stride; two CTAs share an SM. The brick's 10x6x6 halo of keys is streamed through shared
// memory in 5 chunks of two halo z-slices (72 keys, padded to 80). Rows are brick positions:
// row = 32 w + 16 dz + 4 y + x, so warp w holds brick z-slices 2w, 2w+1 and needs exactly halo
// chunks w and w + 1. Per chunk c:
//   S_c = q~ k~_c^T (SS MMA, 128 x 80, fp32 in TMEM)  ->  the two owning warps apply the
//   per-row 3x3x3 mask and the online softmax, the other warps write P = 0  ->
//   O += P_c v_c (TS MMA).
// The halo is gathered by coordinate (inverse map), rotated (axial RoPE) on the way into
// shared memory, and stored in the no-swizzle core-matrix layout; the gather warps run up to
// two chunks ahead and start on the next brick while the current one is still computing.
// TMEM: S (80 columns at column 0, P written over its first 40) + O (<= 96 columns at column
// 128) in a 256-column allocation per CTA. The epilogue reads O out of TMEM, hands it back to
// the MMA warp and only then writes o_loc.
// Every query sits at the same row, and every neighbour at the same column, whatever the
// packing, so a coordinate-carrying repack permutes the output bit for bit.
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace p3d {

namespace ltc {
constexpr int BZ = 8, BY = 4, BX = 4;  // brick
constexpr int HZ = BZ + 2, HY = BY + 2, HX = BX + 2;
constexpr int kSliceKeys = HY * HX;     // 36
constexpr int kChunkKeys = 2 * kSliceKeys;  // 72
constexpr int kChunkPad = 80;           // MMA N (multiple of 16)
constexpr int kChunks = HZ / 2;         // 5
constexpr int kThreads = 256;           // 4 softmax + 3 producer + 1 MMA warps
constexpr int kProd = 96;               // producer threads
constexpr uint32_t kTmemCols = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kRopeSmemBytes = 16384;  // rotation tables up to this size stay in shared memory

template <int D> struct Smem {
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kCBytes = kChunkPad * D * 2;  // one K or V chunk
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;               // [2 stages]
  static constexpr int kV = kK + 2 * kCBytes;           // [2 stages]
  static constexpr int kSlots = kV + 2 * kCBytes;           // 128 query + 360 halo slots
  static constexpr int kRope = kSlots + (128 + HZ * HY * HX) * 4;  // [22][D/6] (cos, sin)
  static constexpr int kRopeAll = kRope + (HZ + HY + HX) * (D / 6) * 8;  // whole table, if it fits
  static constexpr int kBar = kRopeAll + kRopeSmemBytes;
  static constexpr int kBytes = kBar + 128;
};

enum {
  B_QFULL = 0, B_QEMPTY = 1, B_KVFULL = 2, B_KVEMPTY = 4, B_SFULL = 6, B_PFULL = 7, B_PVDONE = 8,
  B_OFREE = 9, B_DRAIN = 10, B_COUNT = 11
};

struct Params {
  pack3d_index ix;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o_loc;
  float* lse_loc;  // optional
  float scale_log2;
  int nbz, nby, nbx;  // bricks per axis
  int64_t tiles;      // batch * heads * bricks
  int rope_in_smem;   // the whole rotation table is copied to shared memory once per CTA
  long long wait_budget;  // SM cycles of each bounded wait
};

// trace slots of the first four tiles a CTA processes (tracing builds only)
#define LTRACE(ti, off)                                    \
  do {                                                     \
    if ((ti) < 4) P3D_TRACE(3000 + (ti) * 200 + (off));    \
  } while (0)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}


// 16 bytes of one row: rotate 4 (x0, x1) pairs of axis third `axis` by coordinate value cv.
__device__ __forceinline__ uint4 rope16(uint4 x, const float* rope, int pairs, int cv, int p0) {
  const uint32_t xin[4] = {x.x, x.y, x.z, x.w};
  uint32_t xo[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 cs = rope_cs(rope, pairs, cv, p0 + k);
    const float e0 = __uint_as_float(xin[k] << 16);
    const float e1 = __uint_as_float(xin[k] & 0xffff0000u);
    xo[k] = tc::pack_bf16(e0 * cs.x - e1 * cs.y, e0 * cs.y + e1 * cs.x);
  }
  return make_uint4(xo[0], xo[1], xo[2], xo[3]);
}

}  // namespace ltc

template <int D>
__global__ void __launch_bounds__(ltc::kThreads, 2) k_local_tc(const ltc::Params P) {
  using namespace ltc;
  using S = Smem<D>;
  constexpr int KC = D / 8;
  constexpr int DA = D / 3;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBar + 8 * B_COUNT + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) P3D_TRACE(3000);
  if (tid == 0) P3D_TRACE_CLK(3910);
  tc::Abort ab{abort_flag, P.ix.status, P.wait_budget};
  const pack3d_geom& g = P.ix.geom;
  const int64_t N = P.ix.n;
  const int64_t bricks = (int64_t)P.nbz * P.nby * P.nbx;
  // tile t -> (batch*head, brick origin); consecutive tiles are neighbouring bricks of one
  // (batch, head), so the CTAs in flight share most of their halos in L2
  auto origin = [&](int64_t t, int64_t& bh, int& z0, int& y0, int& x0) {
    bh = t / bricks;
    const int64_t br = t % bricks;
    z0 = (int)(br / (P.nby * P.nbx)) * BZ;
    y0 = (int)((br / P.nbx) % P.nby) * BY;
    x0 = (int)(br % P.nbx) * BX;
  };

  if (tid == 0) {
    tc::mbar_init(&bars[B_QFULL], kProd);
    tc::mbar_init(&bars[B_QEMPTY], 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_KVFULL + i], kProd);
      tc::mbar_init(&bars[B_KVEMPTY + i], 1);
    }
    tc::mbar_init(&bars[B_SFULL], 1);
    tc::mbar_init(&bars[B_PFULL], 128);
    tc::mbar_init(&bars[B_PVDONE], 1);
    tc::mbar_init(&bars[B_OFREE], 128);
    tc::mbar_init(&bars[B_DRAIN], 1);
    abort_flag[0] = 0;
    tc::fence_mbar_init();
  }
  if (P.rope_in_smem) {
    const int n = P.ix.rope_rows * P.ix.rope_pairs * 2;
    float* dst = reinterpret_cast<float*>(smem + S::kRopeAll);
    for (int i = tid; i < n; i += kThreads) dst[i] = P.ix.rope[i];
  }
  if (warp == 7) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    // --------------------------------------------------------- softmax + epilogue (row = tid)
    const uint32_t o_col = 128, s_col = 0;
    uint32_t gc = 0;  // chunk counter over all tiles of this CTA
    int ti = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < P.tiles && ok; t += gridDim.x, ++ti) {
      // Lane-derived values are re-derived from opaque copies every tile: hoisting them (and
      // the many TMEM addresses and masks computed from them) out of the tile loop would keep
      // them all live across it and push the 80-column score row out of registers.
      int ln = lane;
      uint32_t tl = tbase;
      asm volatile("" : "+r"(ln), "+r"(tl));
      tl += (uint32_t)(warp * 32) << 16;
      const int dz = ln >> 4, qy = (ln >> 2) & 3, qx = ln & 3;
      int64_t bh;
      int z0, y0, x0;
      origin(t, bh, z0, y0, x0);
      const int cz = z0 + 2 * warp + dz, cy = y0 + qy, cx = x0 + qx;
      const bool valid = cz < g.gz && cy < g.gy && cx < g.gx;
      // the row's memory slot, requested now so that its latency hides behind the chunks
      const int slot = valid ? P.ix.inv[((int64_t)cz * g.gy + cy) * g.gx + cx] : -1;
      // neighbour bits over the two owned chunks: bit = part * 80 + (hz % 2) * 36 + hy * 6 + hx
      uint32_t nb[5] = {0u, 0u, 0u, 0u, 0u};
      if (valid) {
#pragma unroll
        for (int o = 0; o < 27; ++o) {
          const int ddz = o / 9 - 1, ddy = (o / 3) % 3 - 1, ddx = o % 3 - 1;
          const int z = cz + ddz, y = cy + ddy, x = cx + ddx;
          if (z < 0 || z >= g.gz || y < 0 || y >= g.gy || x < 0 || x >= g.gx) continue;
          const int hzr = dz + 1 + ddz;  // halo z relative to the warp's first chunk, 0..3
          const int bit = (hzr >> 1) * kChunkPad + (hzr & 1) * kSliceKeys +
                          (qy + 1 + ddy) * HX + (qx + 1 + ddx);
#pragma unroll
          for (int wd = 0; wd < 5; ++wd) nb[wd] |= (bit >> 5) == wd ? (1u << (bit & 31)) : 0u;
        }
      }
      float m_run = -INFINITY, l_run = 0.f;
      for (int c = 0; c < kChunks; ++c, ++gc) {
        if (!__all_sync(0xffffffffu, ab.wait(&bars[B_SFULL], gc & 1))) { ok = false; break; }
        if (lane == 0) LTRACE(ti, 40 + warp * 16 + c * 2);
        tc::tc_fence_after();
        const int part = c - warp;  // 0 or 1 when this warp owns chunk c
        if (part == 0 || part == 1) {
          // the 80 mask bits of this chunk as a 96-bit window (compile-time word indices below)
          uint32_t win[3];
          if (part == 0) {
            win[0] = nb[0]; win[1] = nb[1]; win[2] = nb[2];
          } else {
            win[0] = (nb[2] >> 16) | (nb[3] << 16);
            win[1] = (nb[3] >> 16) | (nb[4] << 16);
            win[2] = nb[4] >> 16;
          }
          // the chunk's 80 columns in registers; entries off the 3x3x3 cube become -inf, so the
          // row max and P = exp2(s * scale - m) need no further masking (raw scores; scale > 0)
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          uint32_t r[kChunkPad];
#pragma unroll
          for (int c0 = 0; c0 < kChunkPad; c0 += 16)
            tc::tmem_ld16(tl + s_col + c0, *reinterpret_cast<uint32_t(*)[16]>(&r[c0]));
          tc::tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < kChunkPad; ++k) {
            if (!((win[k >> 5] >> (k & 31)) & 1u)) r[k] = 0xff800000u;  // -inf off the cube
            mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(r[k]));
          }
          const float cmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * P.scale_log2;
          const float m_new = fmaxf(m_run, cmax);
          const bool need = m_new > m_run + kRescaleLog2;
          if (part == 1 && __any_sync(0xffffffffu, need)) {
            // O rows of this warp hold P_{c-1} v_{c-1} with the old max: rescale after PV_{c-1}
            if (!__all_sync(0xffffffffu, ab.wait(&bars[B_PVDONE], (gc - 1) & 1))) {
              ok = false;
              break;
            }
            tc::tc_fence_after();
            const float f = need ? ex2(m_run - m_new) : 1.f;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 16) {
              uint32_t r[16];
              tc::tmem_ld16(tl + o_col + c0, r);
              tc::tmem_wait_ld();
#pragma unroll
              for (int k = 0; k < 16; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * f);
              tc::tmem_st16(tl + o_col + c0, r);
            }
            tc::tmem_wait_st();
          }
          if (need) {
            l_run *= ex2(m_run - m_new);
            m_run = m_new;
          }
          const float m_use = m_run == -INFINITY ? 0.f : m_run;
          // P over the first 40 columns of S
          const float neg_m = -m_use;
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c0 = 0; c0 < kChunkPad; c0 += 16) {
            uint32_t p[8];
#pragma unroll
            for (int k = 0; k < 16; k += 2) {
              const float p0 = ex2(fmaf(__uint_as_float(r[c0 + k]), P.scale_log2, neg_m));
              const float p1 = ex2(fmaf(__uint_as_float(r[c0 + k + 1]), P.scale_log2, neg_m));
              ls[(k >> 1) & 3] += p0 + p1;
              p[k >> 1] = tc::pack_bf16(p0, p1);
            }
            ltc::tmem_st8(tl + s_col + (c0 >> 1), p);
          }
          const float lsum = (ls[0] + ls[1]) + (ls[2] + ls[3]);
          l_run += lsum;
        } else {
          const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
          for (int c0 = 0; c0 < kChunkPad / 2; c0 += 8) ltc::tmem_st8(tl + s_col + c0, z);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bars[B_PFULL]);
        if (lane == 0) LTRACE(ti, 40 + warp * 16 + c * 2 + 1);
      }
      if (!ok) break;
      // epilogue after the tile's last PV: O / l packed to bf16, O handed back to the MMA warp
      // for the next tile, then o_loc and lse_loc written
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_PVDONE], (gc - 1) & 1))) break;
      tc::tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      uint32_t ow[D / 2];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t r[16];
        tc::tmem_ld16(tl + o_col + c0, r);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ow[c0 / 2 + k] = tc::pack_bf16(__uint_as_float(r[2 * k]) * inv_l,
                                         __uint_as_float(r[2 * k + 1]) * inv_l);
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&bars[B_OFREE]);
      if (slot >= 0) {
        const int64_t bh = t / bricks;
        uint4* dst = reinterpret_cast<uint4*>(P.o_loc + (bh * N + slot) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          dst[c] = make_uint4(ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
        if (P.lse_loc)
          P.lse_loc[bh * N + slot] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
      if (lane == 0) LTRACE(ti, 150 + warp);
    }
    if (tid == 0) P3D_TRACE_CLK(3912);
  } else if (warp < 7) {
    // --------------------------------------------------------- producer: q tile, then k/v chunks
    // Per tile: the slots of the 128 queries and 360 halo keys and the rotation rows of the 22
    // coordinate values the brick touches are staged in shared memory; every row piece is then
    // a cp.async (many in flight at once) followed by an in-place rotation for q and k. The
    // producer runs ahead of the MMA warp by the two k/v stages and, across tiles, gathers the
    // next brick while the current one is still being computed.
    const int ptid = tid - 128;
    constexpr int PR = D / 6;  // rotation pairs per axis
    int32_t* slot_q = reinterpret_cast<int32_t*>(smem + S::kSlots);
    int32_t* slot_h = slot_q + 128;
    float2* rope_s = reinterpret_cast<float2*>(smem + S::kRope);  // [22][PR]
    volatile int* prod_ok = abort_flag + 1;                       // [2], used alternately
    int nwait = 0;
    // a bounded wait by one producer thread, its verdict shared with all 96
    auto pwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      volatile int* f = prod_ok + (nwait++ & 1);
      if (ptid == 0) *f = ab.wait(bar, parity) ? 1 : 0;
      asm volatile("bar.sync 1, 96;" ::: "memory");
      return *f != 0;
    };
    // rotation of one 16-byte piece (8 dims, 4 pairs) in place with table row `roff`
    auto rotate_piece = [&](uint8_t* ptr, int roff) {
      const uint4 x = *reinterpret_cast<uint4*>(ptr);
      const float4* cs4 = reinterpret_cast<const float4*>(rope_s + roff);
      const float4 ca = cs4[0], cb = cs4[1];
      const float cs[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
      const uint32_t xin[4] = {x.x, x.y, x.z, x.w};
      uint32_t xo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float e0 = __uint_as_float(xin[k] << 16);
        const float e1 = __uint_as_float(xin[k] & 0xffff0000u);
        xo[k] = tc::pack_bf16(e0 * cs[2 * k] - e1 * cs[2 * k + 1], e0 * cs[2 * k + 1] + e1 * cs[2 * k]);
      }
      *reinterpret_cast<uint4*>(ptr) = make_uint4(xo[0], xo[1], xo[2], xo[3]);
    };
    // table row of a piece: axis third of column kc, coordinate index along that axis
    auto rope_off = [&](int hz, int hy, int hx, int kc) {
      const int axis = (kc * 8) / DA, p0 = ((kc * 8) % DA) / 2;
      const int idx = axis == 0 ? hz : (axis == 1 ? HZ + hy : HZ + HY + hx);
      return idx * PR + p0;
    };
    // The (key, column) pieces a thread moves are the same in every chunk: their shared-memory
    // offset, key number and rotation-table row are packed once per thread into one word; a
    // z-third piece of chunk c adds 2c table rows.
    //   bits 0-9  : offset / 16 within a chunk stage (< 80 * 12 pieces)
    //   bits 10-16: key number + 1 (0: padding key of the 80-wide chunk)
    //   bits 17-29: rotation-table row offset (element pairs)
    //   bit  30   : z-third piece
    constexpr int NI = kChunkPad * KC / kProd;
    static_assert(NI * kProd == kChunkPad * KC, "pieces per chunk must split evenly");
    static_assert(kChunkPad * KC <= 1024 && kChunkKeys < 127 && (HZ + HY + HX) * PR < 8192,
                  "piece fields must fit their bit ranges");
    uint32_t pinfo[NI];
#pragma unroll
    for (int n = 0; n < NI; ++n) {
      int kk, kc;
      tc::PieceOrder<KC>::at(ptid + n * kProd, kk, kc);
      const int off16 = kc * kChunkPad + (kk >> 3) * 8 + (kk & 7);
      const int key1 = kk < kChunkKeys ? kk + 1 : 0;
      const int ro = rope_off(kk / kSliceKeys, (kk / HX) % HY, kk % HX, kc);
      const int zf = (kc * 8) / DA == 0 ? 1 : 0;
      pinfo[n] = (uint32_t)off16 | ((uint32_t)key1 << 10) | ((uint32_t)ro << 17) | ((uint32_t)zf << 30);
    }
    // halo chunk c of the current tile into the stage of chunk counter gi
    auto issue_chunk = [&](const __nv_bfloat16* kb, const __nv_bfloat16* vb, int c, uint32_t gi) {
      uint8_t* ks = smem + S::kK + (gi & 1) * S::kCBytes;
      uint8_t* vs = smem + S::kV + (gi & 1) * S::kCBytes;
#pragma unroll
      for (int n = 0; n < NI; ++n) {
        const int off16 = pinfo[n] & 1023, key1 = (pinfo[n] >> 10) & 127;
        const int slot = key1 ? slot_h[c * kChunkKeys + key1 - 1] : -1;
        const int64_t src = (int64_t)(slot >= 0 ? slot : 0) * D + (off16 / kChunkPad) * 8;
        tc::cp_async16(ks + off16 * 16, kb + src, slot >= 0);
        tc::cp_async16(vs + off16 * 16, vb + src, slot >= 0);
      }
      tc::cp_async_commit();
    };
    // after its copies landed: rotate k in place, publish
    auto finish_chunk = [&](int c, uint32_t gi) {
      uint8_t* ks = smem + S::kK + (gi & 1) * S::kCBytes;
#pragma unroll
      for (int n = 0; n < NI; ++n) {
        const int ro = ((pinfo[n] >> 17) & 8191) + ((pinfo[n] >> 30) ? 2 * c * PR : 0);
        // zero-filled pieces (absent or padding keys) rotate to zero
        rotate_piece(ks + (pinfo[n] & 1023) * 16, ro);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_KVFULL + (gi & 1)]);
    };
    uint32_t gc = 0;
    int ti = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < P.tiles && ok; t += gridDim.x, ++ti, gc += kChunks) {
      int64_t bh;
      int z0, y0, x0;
      origin(t, bh, z0, y0, x0);
      const __nv_bfloat16* qb = P.q + bh * N * D;
      const __nv_bfloat16* kb = P.k + bh * N * D;
      const __nv_bfloat16* vb = P.v + bh * N * D;
      if (ptid == 0) LTRACE(ti, 0);
      // every producer thread is done with the previous tile's slots and rotation rows
      asm volatile("bar.sync 1, 96;" ::: "memory");
#pragma unroll 4
      for (int i = ptid; i < 128 + HZ * kSliceKeys; i += kProd) {
        int z, y, x;
        if (i < 128) {
          const int w = i >> 5, l = i & 31;
          z = z0 + 2 * w + (l >> 4); y = y0 + ((l >> 2) & 3); x = x0 + (l & 3);
        } else {
          const int h = i - 128;
          z = z0 - 1 + h / kSliceKeys; y = y0 - 1 + (h / HX) % HY; x = x0 - 1 + h % HX;
        }
        const bool in = z >= 0 && z < g.gz && y >= 0 && y < g.gy && x >= 0 && x < g.gx;
        slot_q[i] = in ? P.ix.inv[((int64_t)z * g.gy + y) * g.gx + x] : -1;
      }
      if (ptid == 0) LTRACE(ti, 3);
      const float* rope = P.rope_in_smem ? reinterpret_cast<const float*>(smem + S::kRopeAll)
                                         : P.ix.rope;
      for (int i = ptid; i < (HZ + HY + HX) * PR; i += kProd) {
        const int idx = i / PR, pp = i % PR;
        const int cv = idx < HZ ? z0 - 1 + idx : (idx < HZ + HY ? y0 - 1 + idx - HZ : x0 - 1 + idx - HZ - HY);
        rope_s[i] = (cv >= 0 && cv < P.ix.rope_rows) ? rope_cs(rope, P.ix.rope_pairs, cv, pp)
                                                     : make_float2(0.f, 0.f);
      }
      asm volatile("bar.sync 1, 96;" ::: "memory");
      if (ptid == 0) LTRACE(ti, 1);
      // chunk 0 (its stage frees first), the q tile (free once the previous tile's last QK is
      // done), then chunk 1; all in flight before any is waited for
      if (gc >= 2 && !pwait(&bars[B_KVEMPTY + (gc & 1)], ((gc - 2) >> 1) & 1)) { ok = false; break; }
      if (ptid == 0) LTRACE(ti, 4);
      issue_chunk(kb, vb, 0, gc);
      if (ptid == 0) LTRACE(ti, 5);
      if (ti >= 1 && !pwait(&bars[B_QEMPTY], (ti - 1) & 1)) { ok = false; break; }
      if (ptid == 0) LTRACE(ti, 6);
      // q tile: row r <-> brick (2w + dz, y, x) <-> halo (2w + dz + 1, y + 1, x + 1)
      for (int i = ptid; i < 128 * KC; i += kProd) {
        int r, kc;
        tc::PieceOrder<KC>::at(i, r, kc);
        const int slot = slot_q[r];
        tc::cp_async16(smem + S::kQ + kc * 2048 + (r >> 3) * 128 + (r & 7) * 16,
                       qb + (int64_t)(slot >= 0 ? slot : 0) * D + kc * 8, slot >= 0);
      }
      tc::cp_async_commit();
      if (gc + 1 >= 2 && !pwait(&bars[B_KVEMPTY + ((gc + 1) & 1)], ((gc - 1) >> 1) & 1)) {
        ok = false;
        break;
      }
      if (ptid == 0) LTRACE(ti, 7);
      issue_chunk(kb, vb, 1, gc + 1);
      if (ptid == 0) LTRACE(ti, 8);
      tc::cp_async_wait_group<1>();  // chunk 0 and q have landed
      if (ptid == 0) LTRACE(ti, 9);
#pragma unroll 4
      for (int i = ptid; i < 128 * KC; i += kProd) {
        int r, kc;
        tc::PieceOrder<KC>::at(i, r, kc);
        const int w = r >> 5, l = r & 31;  // pieces of absent rows are zero and stay zero
        rotate_piece(smem + S::kQ + kc * 2048 + (r >> 3) * 128 + (r & 7) * 16,
                     rope_off(2 * w + (l >> 4) + 1, ((l >> 2) & 3) + 1, (l & 3) + 1, kc));
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_QFULL]);
      if (ptid == 0) LTRACE(ti, 2);
      finish_chunk(0, gc);
      if (ptid == 0) LTRACE(ti, 12);
      tc::cp_async_wait_group<0>();
      finish_chunk(1, gc + 1);
      if (ptid == 0) LTRACE(ti, 16);
      // halo chunks 2..4 reuse the two stages once the PV two chunks earlier has completed
      for (int c = 2; c < kChunks; ++c) {
        const uint32_t gi = gc + c;
        if (!pwait(&bars[B_KVEMPTY + (gi & 1)], ((gi - 2) >> 1) & 1)) { ok = false; break; }
        issue_chunk(kb, vb, c, gi);
        if (ptid == 0) LTRACE(ti, 10 + c * 4);
        tc::cp_async_wait_all();
        if (ptid == 0) LTRACE(ti, 10 + c * 4 + 1);
        finish_chunk(c, gi);
        if (ptid == 0) LTRACE(ti, 10 + c * 4 + 2);
      }
    }
    tc::cp_async_wait_all();  // nothing may still be landing in shared memory at exit
  } else if (warp == 7) {
    // --------------------------------------------------------- MMA issuer
    // The whole warp runs the schedule with warp-uniform values (descriptors formed once and
    // advanced by address offsets); one elected lane issues the MMAs and commits.
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0);
    const uint32_t id_qk = tc::idesc_bf16_f32(128, kChunkPad, false, false);
    const uint32_t id_pv = tc::idesc_bf16_f32(128, D, false, true);
    const uint64_t qd0 = tc::smem_desc(tc::smem_u32(smem + S::kQ), 2048, 128);
    const uint64_t kd0 = tc::smem_desc(tc::smem_u32(smem + S::kK), kChunkPad * 16, 128);
    const uint64_t vd0 = tc::smem_desc(tc::smem_u32(smem + S::kV), 128, kChunkPad * 16);
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    uint32_t gc = 0;
    int ti = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < P.tiles && ok; t += gridDim.x, ++ti) {
      if (!wwait(&bars[B_QFULL], ti & 1)) break;
      for (int c = 0; c < kChunks; ++c, ++gc) {
        const int st = gc & 1;
        if (!wwait(&bars[B_KVFULL + st], (gc >> 1) & 1)) { ok = false; break; }
        if (lane == 0) LTRACE(ti, 130 + c * 2);
        // S holds P of the previous chunk until its PV has completed
        if (gc >= 1 && !wwait(&bars[B_PVDONE], (gc - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t b0 = kd0 + (uint64_t)((st * S::kCBytes) >> 4);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            tc::mma_ss(tb, qd0 + (uint64_t)(ks * (4096 >> 4)),
                       b0 + (uint64_t)(ks * (2 * kChunkPad * 16 >> 4)), id_qk, ks > 0);
          tc::tc_commit(&bars[B_SFULL]);
          if (c == kChunks - 1) tc::tc_commit(&bars[B_QEMPTY]);  // q tile free for the next brick
        }
        __syncwarp();
        if (lane == 0) LTRACE(ti, 110 + c * 4);
        if (!wwait(&bars[B_PFULL], gc & 1)) { ok = false; break; }
        if (lane == 0) LTRACE(ti, 110 + c * 4 + 1);
        // the first PV of a tile overwrites O: the previous tile's epilogue must have read it
        if (c == 0 && ti >= 1 && !wwait(&bars[B_OFREE], (ti - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t v0 = vd0 + (uint64_t)((st * S::kCBytes) >> 4);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kChunkPad / 16; ++ks)
            tc::mma_ts(tb + 128, tb + ks * 8, v0 + (uint64_t)(ks * (256 >> 4)), id_pv,
                       (c > 0 || ks > 0) ? 1u : 0u);
          tc::tc_commit(&bars[B_PVDONE]);
          tc::tc_commit(&bars[B_KVEMPTY + st]);
        }
        __syncwarp();
        if (lane == 0) LTRACE(ti, 110 + c * 4 + 2);
      }
    }
    // every MMA this warp issued has completed once this commit arrives (bounded wait)
    if (tc::elect_one()) tc::tc_commit(&bars[B_DRAIN]);
    __syncwarp();
    if (!tc::mbar_wait(&bars[B_DRAIN], 0, 100000000LL))
      set_status(P.ix.status, PACK3D_ERR_TIMEOUT);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 7) {
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
}

template <int D>
cudaError_t launch_local_tc(const pack3d_index& ix, const void* q, const void* k, const void* v,
                            int64_t bh, float scale, void* o_loc, float* lse_loc,
                            cudaStream_t s) {
  using namespace ltc;
  static std::atomic<uint64_t> attr_done{0};
  if (smem_attr_once(reinterpret_cast<const void*>(k_local_tc<D>), Smem<D>::kBytes, attr_done) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  Params p;
  p.ix = ix;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o_loc = static_cast<__nv_bfloat16*>(o_loc);
  p.lse_loc = lse_loc;
  p.scale_log2 = scale * kLog2e;
  p.wait_budget = wait_budget_cycles();
  p.nbz = (ix.geom.gz + BZ - 1) / BZ;
  p.nby = (ix.geom.gy + BY - 1) / BY;
  p.nbx = (ix.geom.gx + BX - 1) / BX;
  p.tiles = bh * p.nbz * p.nby * p.nbx;
  p.rope_in_smem = (int64_t)ix.rope_rows * ix.rope_pairs * 8 <= kRopeSmemBytes ? 1 : 0;
  if (p.tiles <= 0) return cudaSuccess;
  // persistent: two CTAs per SM, each walking tiles blockIdx.x, blockIdx.x + gridDim.x, ...
  const int64_t cap = 2 * (int64_t)sm_count();
  const unsigned grid = (unsigned)(p.tiles < cap ? p.tiles : cap);
  k_local_tc<D><<<grid, kThreads, Smem<D>::kBytes, s>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t local_tc_dispatch(const pack3d_index& ix, const void* q, const void* k,
                              const void* v, int64_t bh, float scale, void* o_loc,
                              float* lse_loc, cudaStream_t s) {
  if (ix.geom.head_dim == 96) return launch_local_tc<96>(ix, q, k, v, bh, scale, o_loc, lse_loc, s);
  return launch_local_tc<48>(ix, q, k, v, bh, scale, o_loc, lse_loc, s);
}

}  // namespace p3d

#ifdef P3D_TRACE_ENABLED
extern "C" int p3d_trace_read_l(unsigned long long* host) {
  cudaDeviceSynchronize();
  return (int)cudaMemcpyFromSymbol(host, p3d::g_trace, sizeof(unsigned long long) * 4096);
}
extern "C" int p3d_trace_clear_l() {
  static unsigned long long z[4096];
  return (int)cudaMemcpyToSymbol(p3d::g_trace, z, sizeof(z));
}
#endif
