// Local branch of PACK3D attention on tcgen05 tensor cores (bf16 I/O, head_dim 48 or 96).
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 1: each query
// attends exactly to every token of its 3x3x3 coordinate neighbourhood (at most 27, fewer at
// the border), found by coordinate, never by adjacency in memory; paper summary §3.5: streamed
// online softmax, no gathered neighbour tensor in memory.
//
// A CTA (4 softmax warps, 3 gather warps, 1 MMA warp) owns one 8x4x4 (z, y, x) coordinate brick of 128 queries of one (batch, head). Its
// 10x6x6 halo of keys is streamed through shared memory in 5 chunks of two halo z-slices
// (72 keys, padded to 80). Rows are brick positions: row = 32 w + 16 dz + 4 y + x, so warp w
// holds brick z-slices 2w, 2w+1 and needs exactly halo chunks w and w + 1. Per chunk c:
//   S_c = q~ k~_c^T (SS MMA, 128 x 80, fp32 in TMEM)  ->  the two owning warps apply the
//   per-row 3x3x3 mask and the online softmax, the other warps write P = 0  ->
//   O += P_c v_c (TS MMA).
// The halo is gathered by coordinate (inverse map), rotated (axial RoPE) on the way into
// shared memory, and stored in the no-swizzle core-matrix layout. TMEM: S (80 columns at
// column 0, P written over its first 40) + O (<= 96 columns at column 128) in a 256-column
// allocation, so two CTAs share an SM and overlap each other's MMA, softmax and gather.
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

template <int D> struct Smem {
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kCBytes = kChunkPad * D * 2;  // one K or V chunk
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQBytes;               // [2 stages]
  static constexpr int kV = kK + 2 * kCBytes;           // [2 stages]
  static constexpr int kSlots = kV + 2 * kCBytes;           // 128 query + 360 halo slots
  static constexpr int kRope = kSlots + (128 + HZ * HY * HX) * 4;  // [22][D/6] (cos, sin)
  static constexpr int kBar = kRope + (HZ + HY + HX) * (D / 6) * 8;
  static constexpr int kBytes = kBar + 128;
};

enum { B_QFULL = 0, B_KVFULL = 1, B_KVEMPTY = 3, B_SFULL = 5, B_PFULL = 6, B_PVDONE = 7, B_COUNT = 8 };

struct Params {
  pack3d_index ix;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o_loc;
  float* lse_loc;  // optional
  float scale_log2;
  int nbz, nby, nbx;  // bricks per axis
};

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

struct Abort {
  volatile int* flag;
  int32_t* status;
  __device__ bool wait(uint64_t* bar, uint32_t parity) {
    if (tc::mbar_test_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!tc::mbar_test_wait(bar, parity)) {
      if (*flag) return false;
      if (clock64() - t0 > 4000000000LL) {
        *flag = 1;
        set_status(status, PACK3D_ERR_TIMEOUT);
        return false;
      }
    }
    return true;
  }
};

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
  Abort ab{abort_flag, P.ix.status};
  const pack3d_geom& g = P.ix.geom;
  const int64_t N = P.ix.n;

  // tile -> (batch*head, brick origin)
  const int64_t bricks = (int64_t)P.nbz * P.nby * P.nbx;
  const int64_t bh = blockIdx.x / bricks;
  const int64_t br = blockIdx.x % bricks;
  const int z0 = (int)(br / (P.nby * P.nbx)) * BZ;
  const int y0 = (int)((br / P.nbx) % P.nby) * BY;
  const int x0 = (int)(br % P.nbx) * BX;
  const __nv_bfloat16* qb = P.q + bh * N * D;
  const __nv_bfloat16* kb = P.k + bh * N * D;
  const __nv_bfloat16* vb = P.v + bh * N * D;

  if (tid == 0) {
    tc::mbar_init(&bars[B_QFULL], kProd);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_KVFULL + i], kProd);
      tc::mbar_init(&bars[B_KVEMPTY + i], 1);
    }
    tc::mbar_init(&bars[B_SFULL], 1);
    tc::mbar_init(&bars[B_PFULL], 128);
    tc::mbar_init(&bars[B_PVDONE], 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 7) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    // --------------------------------------------------------- softmax + epilogue (row = tid)
    const int dz = lane >> 4, qy = (lane >> 2) & 3, qx = lane & 3;
    const int cz = z0 + 2 * warp + dz, cy = y0 + qy, cx = x0 + qx;
    const bool valid = cz < g.gz && cy < g.gy && cx < g.gx;
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    const uint32_t o_col = 128, s_col = 0;
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
    bool ok = true;
    for (int c = 0; c < kChunks && ok; ++c) {
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_SFULL], c & 1))) { ok = false; break; }
      if (lane == 0) P3D_TRACE(3100 + warp * 16 + c * 2);
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
          if (!__all_sync(0xffffffffu, ab.wait(&bars[B_PVDONE], (c - 1) & 1))) { ok = false; break; }
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
      if (lane == 0) P3D_TRACE(3100 + warp * 16 + c * 2 + 1);
    }
    if (ok) {
      // epilogue after the last PV: o_loc = O / l, lse_loc
      constexpr int last = kChunks - 1;
      if (__all_sync(0xffffffffu, ab.wait(&bars[B_PVDONE], last & 1))) {
        tc::tc_fence_after();
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        const int64_t slot =
            valid ? P.ix.inv[((int64_t)cz * g.gy + cy) * g.gx + cx] : -1;
        uint4* dst = slot >= 0 ? reinterpret_cast<uint4*>(P.o_loc + (bh * N + slot) * D) : nullptr;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint32_t r[16];
          tc::tmem_ld16(tl + o_col + c0, r);
          tc::tmem_wait_ld();
          uint32_t w[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            w[k] = tc::pack_bf16(__uint_as_float(r[2 * k]) * inv_l,
                                 __uint_as_float(r[2 * k + 1]) * inv_l);
          if (dst) {
            dst[c0 / 8] = make_uint4(w[0], w[1], w[2], w[3]);
            dst[c0 / 8 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
        if (lane == 0) P3D_TRACE(3400 + warp);
        if (slot >= 0 && P.lse_loc)
          P.lse_loc[bh * N + slot] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  } else if (warp < 7) {
    // --------------------------------------------------------- producer: q tile, then k/v chunks
    // Slots of the 128 queries and 360 halo keys and the rotation rows of the 22 coordinate
    // values the brick touches are staged in shared memory first; every row piece is then a
    // cp.async (all in flight at once) followed by an in-place rotation for q and k.
    const int ptid = tid - 128;
    constexpr int PR = D / 6;  // rotation pairs per axis
    int32_t* slot_q = reinterpret_cast<int32_t*>(smem + S::kSlots);
    int32_t* slot_h = slot_q + 128;
    float2* rope_s = reinterpret_cast<float2*>(smem + S::kRope);  // [22][PR]
    volatile int* prod_ok = abort_flag + 1;
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
    for (int i = ptid; i < (HZ + HY + HX) * PR; i += kProd) {
      const int idx = i / PR, pp = i % PR;
      const int cv = idx < HZ ? z0 - 1 + idx : (idx < HZ + HY ? y0 - 1 + idx - HZ : x0 - 1 + idx - HZ - HY);
      rope_s[i] = (cv >= 0 && cv < P.ix.rope_rows) ? rope_cs(P.ix.rope, P.ix.rope_pairs, cv, pp)
                                                   : make_float2(0.f, 0.f);
    }
    asm volatile("bar.sync 1, 96;" ::: "memory");
    if (ptid == 0) P3D_TRACE(3001);
    // rotation of one 16-byte piece (8 dims, 4 pairs) in place, for halo position (hz, hy, hx)
    auto rotate_at = [&](uint8_t* ptr, int hz, int hy, int hx, int kc) {
      const int axis = (kc * 8) / DA, p0 = ((kc * 8) % DA) / 2;
      const int idx = axis == 0 ? hz : (axis == 1 ? HZ + hy : HZ + HY + hx);
      const uint4 x = *reinterpret_cast<uint4*>(ptr);
      const float4* cs4 = reinterpret_cast<const float4*>(rope_s + idx * PR + p0);
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
    // q tile: row r <-> brick (2w + dz, y, x) <-> halo (2w + dz + 1, y + 1, x + 1)
    for (int i = ptid; i < 128 * KC; i += kProd) {
      int r, kc;
      tc::PieceOrder<KC>::at(i, r, kc);
      const int slot = slot_q[r];
      tc::cp_async16(smem + S::kQ + kc * 2048 + (r >> 3) * 128 + (r & 7) * 16,
                     qb + (int64_t)(slot >= 0 ? slot : 0) * D + kc * 8, slot >= 0);
    }
    tc::cp_async_commit();
    tc::cp_async_wait_all();
#pragma unroll 4
    for (int i = ptid; i < 128 * KC; i += kProd) {
      int r, kc;
      tc::PieceOrder<KC>::at(i, r, kc);
      const int w = r >> 5, l = r & 31;  // pieces of absent rows are zero and stay zero
      rotate_at(smem + S::kQ + kc * 2048 + (r >> 3) * 128 + (r & 7) * 16, 2 * w + (l >> 4) + 1,
                ((l >> 2) & 3) + 1, (l & 3) + 1, kc);
    }
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars[B_QFULL]);
    if (ptid == 0) P3D_TRACE(3002);
    // halo chunks: key kk of chunk c is halo key 72 c + kk = (2c + kk / 36, (kk / 6) % 6, kk % 6)
    for (int c = 0; c < kChunks; ++c) {
      const int st = c & 1;
      if (c >= 2) {
        if (ptid == 0) *prod_ok = ab.wait(&bars[B_KVEMPTY + st], ((c - 2) >> 1) & 1) ? 1 : 0;
        asm volatile("bar.sync 1, 96;" ::: "memory");
        if (!*prod_ok) break;
      }
      uint8_t* ks = smem + S::kK + st * S::kCBytes;
      uint8_t* vs = smem + S::kV + st * S::kCBytes;
      for (int i = ptid; i < kChunkPad * KC; i += kProd) {
        int kk, kc;
        tc::PieceOrder<KC>::at(i, kk, kc);
        const int slot = kk < kChunkKeys ? slot_h[c * kChunkKeys + kk] : -1;
        const int off = kc * (kChunkPad * 16) + (kk >> 3) * 128 + (kk & 7) * 16;
        const int64_t src = (int64_t)(slot >= 0 ? slot : 0) * D + kc * 8;
        tc::cp_async16(ks + off, kb + src, slot >= 0);
        tc::cp_async16(vs + off, vb + src, slot >= 0);
      }
      tc::cp_async_commit();
      if (ptid == 0) P3D_TRACE(3010 + c * 4);
      tc::cp_async_wait_all();
      if (ptid == 0) P3D_TRACE(3010 + c * 4 + 1);
#pragma unroll 4
      for (int i = ptid; i < kChunkPad * KC; i += kProd) {
        int kk, kc;
        tc::PieceOrder<KC>::at(i, kk, kc);
        // zero-filled pieces (absent or padding keys) rotate to zero; padding keys index a
        // table row inside the 22-row table, so no guard is needed
        rotate_at(ks + kc * (kChunkPad * 16) + (kk >> 3) * 128 + (kk & 7) * 16,
                  2 * c + kk / kSliceKeys, (kk / HX) % HY, kk % HX, kc);
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_KVFULL + st]);
      if (ptid == 0) P3D_TRACE(3010 + c * 4 + 2);
    }
  } else if (warp == 7 && lane == 0) {
    // --------------------------------------------------------- MMA issuer
    const uint32_t id_qk = tc::idesc_bf16_f32(128, kChunkPad, false, false);
    const uint32_t id_pv = tc::idesc_bf16_f32(128, D, false, true);
    const uint32_t qaddr = tc::smem_u32(smem + S::kQ);
    bool ok = ab.wait(&bars[B_QFULL], 0);
    for (int c = 0; c < kChunks && ok; ++c) {
      const int st = c & 1;
      if (!ab.wait(&bars[B_KVFULL + st], (c >> 1) & 1)) break;
      P3D_TRACE(3300 + c * 2);
      // S holds P_{c-1} until PV_{c-1} has completed
      if (c >= 1 && !ab.wait(&bars[B_PVDONE], (c - 1) & 1)) break;
      tc::tc_fence_after();
      const uint32_t kaddr = tc::smem_u32(smem + S::kK + st * S::kCBytes);
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint64_t a = tc::smem_desc(qaddr + ks * 4096, 2048, 128);
        const uint64_t b = tc::smem_desc(kaddr + ks * 2 * (kChunkPad * 16), kChunkPad * 16, 128);
        tc::mma_ss(tbase, a, b, id_qk, ks > 0);
      }
      tc::tc_commit(&bars[B_SFULL]);
      P3D_TRACE(3200 + c * 4);
      if (!ab.wait(&bars[B_PFULL], c & 1)) break;
      P3D_TRACE(3200 + c * 4 + 1);
      tc::tc_fence_after();
      const uint32_t vaddr = tc::smem_u32(smem + S::kV + st * S::kCBytes);
#pragma unroll
      for (int ks = 0; ks < kChunkPad / 16; ++ks) {
        const uint64_t b = tc::smem_desc(vaddr + ks * 256, 128, kChunkPad * 16);
        tc::mma_ts(tbase + 128, tbase + ks * 8, b, id_pv, (c > 0 || ks > 0) ? 1u : 0u);
      }
      tc::tc_commit(&bars[B_PVDONE]);
      tc::tc_commit(&bars[B_KVEMPTY + st]);
      P3D_TRACE(3200 + c * 4 + 2);
    }
  }

  // All roles are done. The MMA issuer's last commit (PV of the final chunk) was awaited by the
  // softmax warps before their epilogue; on an abort, drain any MMA still in flight.
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 7) {
    if (*abort_flag && lane == 0) {
      // a bounded extra wait for the final PV; it arrives once every issued MMA has finished
      tc::mbar_wait(&bars[B_PVDONE], (kChunks - 1) & 1, 100000000LL);
    }
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
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(k_local_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Smem<D>::kBytes) != cudaSuccess)
      return cudaErrorInvalidValue;
    attr = true;
  }
  Params p;
  p.ix = ix;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o_loc = static_cast<__nv_bfloat16*>(o_loc);
  p.lse_loc = lse_loc;
  p.scale_log2 = scale * kLog2e;
  p.nbz = (ix.geom.gz + BZ - 1) / BZ;
  p.nby = (ix.geom.gy + BY - 1) / BY;
  p.nbx = (ix.geom.gx + BX - 1) / BX;
  const int64_t tiles = bh * p.nbz * p.nby * p.nbx;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  k_local_tc<D><<<(unsigned)tiles, kThreads, Smem<D>::kBytes, s>>>(p);
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
