// Local branch of the PACK3D backward on tcgen05 tensor cores: the gradient of q through the
// 3x3x3 softmax (bf16, head_dim 48 or 96), plus the global branch's part of dq~ (computed
// before by k_bwd_dq_tc), then the inverse rotation -> dq.
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 1 (each query
// attends exactly to its 3x3x3 coordinate neighbourhood); paper summary §3.4 (the backward
// follows the forward's streamed access pattern). For query i and neighbour j, with the
// forward's lse_loc, g_i = sigmoid(a_i) and Dl_i = g_i <dO_i, o_loc_i>:
//   P_ij = exp(<q~_i, k~_j> tau - lse_loc_i),  dP_ij = <dO_i, v_j>,
//   dS_ij = P_ij (g_i dP_ij - Dl_i) tau,        dq~_i = sum_j dS_ij k~_j (+ global part),
//   dq_i = R(c_i)^T dq~_i.
//
// Work units, slot boxes and the halo stream are those of the forward local kernel: a 4x8x8
// brick of one (batch, head) = two 128-query tiles (y0..y0+3 and y0+4..y0+7) sharing 6 halo
// z-slices of 10x10 keys; tile t's 64-key window starts at slice row 40 t; warp w of a tile is
// the brick's z-plane w and owns slices w .. w+2. Per tile and slice s:
//   S = q~ k~_s^T and dP = dO v_s^T   (two SS MMAs, 128 x 64, fp32 in TMEM)
//   owners: dS in bf16 over the first 32 columns of S (the 3x3x3 mask; no running max, the
//   forward's lse is known);   dq~ += dS k~_s   (TS MMA, N = d, the other warps' rows disabled
//   through the MMA's output-lane mask).
// TMEM per tile: S 64 + dP 64 + dq~ 96 columns (single-buffered S / dP: the two tiles' chains
// interleave on the tensor core). Warps: elementwise 0-7 (tile = warp / 4; warps 0, 1, 4, 5 also
// stage the next unit's q~ and dO tiles), slot boxes 8 (warp 9 idle), k~ / v producers 10-13,
// MMA 14-15 (one per tile). Units come from the index's device-wide counter (status word 2),
// put back to zero by the last CTA. Every query sits at the same row whatever the packing, so a
// coordinate-carrying repack permutes dq bit for bit.
#include <math.h>

#include "bwd_work.h"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace p3d {

namespace lb {
constexpr int BZ = 4, BY = 8, BX = 8;
constexpr int kTiles = 2;
constexpr int TY = BY / kTiles;
constexpr int HY = BY + 2, HX = BX + 2;
constexpr int kChunks = BZ + 2;        // 6 halo z-slices
constexpr int kSliceKeys = HY * HX;    // 100
constexpr int kNK = 64;                // tile window
constexpr int kNV = (TY + 2) * HX;     // 60 window columns that can hold a neighbour
constexpr int kWin = TY * HX;          // 40: first slice row of tile 1's window
constexpr int kRows = kWin + kNK;      // 104 rows per stage
constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr int W_BOX = 8, W_PROD = 10, W_MMA = 14;
constexpr int kProd = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;
constexpr uint32_t kSCol = 0, kPCol = 64, kDqCol = 128;  // within a tile's 256 columns
constexpr int kBoxX = 16, kBoxY = HY, kBoxZ = kChunks;   // slot box: x from x0 - 4
constexpr int kBoxBytes = kBoxX * kBoxY * kBoxZ * 4;
constexpr int kBoxPitch = 4096;  // box, then the unit index (int64) at kBoxBytes

__host__ __device__ constexpr int slice_row(int hy, int hx) { return hy * HX + hx; }

// Shared memory, no-swizzle core-matrix operand layouts as in the forward local kernel: the
// 16-byte piece (row r, column chunk c) of an A tile (q~ or dO) at c * kQCol + (r / 8) * 128 +
// (r % 8) * 16, that of a k~ or v stage at c * kChunkCol + (row / 8) * 128 + (row % 8) * 16.
template <int D> struct Smem {
  static constexpr int KC = D / 8;
  static constexpr int kQCol = 128 * 16 + 16;
  static constexpr int kQBuf = KC * kQCol;
  static constexpr int kChunkCol = kRows * 16 + 16;
  static constexpr int kStage = KC * kChunkCol;
  static constexpr int kA = 0;                             // [tile][q~, dO]
  static constexpr int kK = kA + 2 * kTiles * kQBuf;       // [kStages] k~ slices
  static constexpr int kV = kK + kStages * kStage;         // [kStages] v slices
  static constexpr int kBox = (kV + kStages * kStage + 127) / 128 * 128;  // [2] slot boxes
  static constexpr int kBar = kBox + 2 * kBoxPitch;
  static constexpr int kBytes = kBar + 1024;
  static_assert(kBox % 128 == 0, "box alignment");
  static_assert(kBoxBytes + 8 <= kBoxPitch, "slot box and unit index");
  static_assert(kBytes <= 232448, "dynamic shared memory of one CTA");
  __device__ static int a_off(int tile, int op) { return kA + (tile * 2 + op) * kQBuf; }
  __device__ static int q_off(int r, int c) { return c * kQCol + (r >> 3) * 128 + (r & 7) * 16; }
};

enum {
  B_QFULL = 0, B_QEMPTY = 2,  // [tile]
  B_KVFULL = 4, B_KVEMPTY = 7, B_BOX = 10, B_BOXFREE = 12,
  B_SFULL = 14,   // [tile][warp]
  B_PFULL = 22,   // [tile][warp]
  B_TSDONE = 30,  // [tile]
  B_EPI = 32,     // [tile][warp]
  B_DRAIN = 40,   // [tile]
  B_COUNT = 42
};
static_assert(B_KVEMPTY - B_KVFULL >= kStages && B_BOX - B_KVEMPTY >= kStages, "ring barriers");
static_assert(8 * B_COUNT + 16 <= 1024, "barrier area");

struct Params {
  pack3d_index ix;
  const __nv_bfloat16* qr;     // rotated q [B, H, N, d]
  const __nv_bfloat16* kr;     // rotated k, one row per query head [B, H, N, d]
  const __nv_bfloat16* v;      // [B, H_kv, N, d]
  const __nv_bfloat16* dO;     // [B, H, N, d]
  const __nv_bfloat16* gate;   // [B, H, N]
  const float* lse_loc;        // [B, H, N]
  const float* Dl;             // [B, H, N]  g <dO, o_loc>
  const float* dqg;            // [B, H, N, d]  the global branch's part of dq~ (or null)
  __nv_bfloat16* dq;
  float scale, scale_log2;
  int nbz, nby, nbx;
  int box_tma;
  int64_t units;
  int kv_group;
  long long wait_budget;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// first and last elementwise warp owning halo slice s (warp w needs slices w .. w + 2)
__device__ __forceinline__ int owner_lo(int s) { return max(0, s - 2); }
__device__ __forceinline__ int owner_hi(int s) { return min(3, s); }

}  // namespace lb

template <int D>
__global__ void __launch_bounds__(lb::kThreads, 1)
    k_bwd_local_dq_tc(const __grid_constant__ CUtensorMap mg, const lb::Params P) {
  using namespace lb;
  using S = Smem<D>;
  constexpr int KC = S::KC;
  constexpr int DA = D / 3;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBar + 8 * B_COUNT + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tc::Abort ab{abort_flag, P.ix.status, P.wait_budget};
  const pack3d_geom& g = P.ix.geom;
  const int64_t N = P.ix.n;
  const int64_t per_field = (int64_t)P.nbz * P.nby * P.nbx;
  auto origin = [&](int64_t u, int64_t& bh, int& z0, int& y0, int& x0) {
    bh = u / per_field;
    const int64_t br = u % per_field;
    z0 = (int)(br / (P.nby * P.nbx)) * BZ;
    y0 = (int)((br / P.nbx) % P.nby) * BY;
    x0 = (int)(br % P.nbx) * BX;
  };
  auto in_grid = [&](int z, int y, int x) {
    return z >= 0 && z < g.gz && y >= 0 && y < g.gy && x >= 0 && x < g.gx;
  };
  auto unit_of = [&](int bb) -> int64_t {
    return *reinterpret_cast<volatile int64_t*>(smem + S::kBox + bb * kBoxPitch + kBoxBytes);
  };

  if (tid == 0) {
    for (int i = 0; i < kTiles; ++i) {
      tc::mbar_init(&bars[B_QFULL + i], 64);  // elementwise warps 0 and 1 of the tile
      tc::mbar_init(&bars[B_QEMPTY + i], 1);
      tc::mbar_init(&bars[B_TSDONE + i], 1);
      tc::mbar_init(&bars[B_DRAIN + i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars[B_KVFULL + i], kProd);
      tc::mbar_init(&bars[B_KVEMPTY + i], kTiles);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_BOX + i], 1);
      tc::mbar_init(&bars[B_BOXFREE + i], 8 + 4);  // elementwise and producer warps
    }
    for (int i = 0; i < 8; ++i) {
      tc::mbar_init(&bars[B_SFULL + i], 1);
      tc::mbar_init(&bars[B_PFULL + i], 32);
      tc::mbar_init(&bars[B_EPI + i], 1);
    }
    abort_flag[0] = 0;
    tc::fence_mbar_init();
  }
  if (warp == W_BOX && lane == 0 && P.box_tma) tc::tma_prefetch_desc(&mg);
  // rows 100..103 of every k~ / v stage are never written by the producers: zero them once
  // (tile 1's MMAs read them; their scores are masked and dS = 0 there)
  for (int i = tid; i < kStages * 2 * KC * (kRows - kSliceKeys); i += kThreads) {
    const int row = kSliceKeys + i % (kRows - kSliceKeys), c = (i / (kRows - kSliceKeys)) % KC;
    const int blk = i / ((kRows - kSliceKeys) * KC);  // stage * 2 + tensor
    *reinterpret_cast<uint4*>(smem + ((blk & 1) ? S::kV : S::kK) + (blk >> 1) * S::kStage +
                              c * S::kChunkCol + (row >> 3) * 128 + (row & 7) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  tc::fence_proxy_async_smem();
  if (warp == W_MMA) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 8) {
    // --------------------------------------------------------- elementwise + epilogue (row = lane)
    const int tile = warp >> 2, w = warp & 3;
    // q~ and dO tiles of unit `un` (slot box nb) into the tile's A buffers: warp w (0 or 1)
    // takes rows 64 w .. 64 w + 63, one row per lane and pass, every 16-byte piece a cp.async
    // straight into the operand layout (rows off the grid or at empty sites are zero-filled);
    // then it publishes its share (QFULL: 64 arrivals per tile)
    auto prepare_a = [&](int64_t un, int nb) {
      int64_t qbh;
      int qz0, qy0, qx0;
      origin(un, qbh, qz0, qy0, qx0);
      const int32_t* qbox = reinterpret_cast<const int32_t*>(smem + S::kBox + nb * kBoxPitch);
      uint8_t* qd = smem + S::a_off(tile, 0);
      uint8_t* gd = smem + S::a_off(tile, 1);
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int r = 64 * w + 32 * pass + lane;
        const int z = r >> 5, y = TY * tile + ((r >> 3) & 3), x = r & 7;
        const int slot = in_grid(qz0 + z, qy0 + y, qx0 + x)
                             ? qbox[((z + 1) * kBoxY + y + 1) * kBoxX + x + 4]
                             : -1;
        const int64_t src = (qbh * N + (slot >= 0 ? slot : 0)) * D;
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          tc::cp_async16(qd + S::q_off(r, c), P.qr + src + c * 8, slot >= 0);
          tc::cp_async16(gd + S::q_off(r, c), P.dO + src + c * 8, slot >= 0);
        }
      }
      tc::cp_async_commit();
      tc::cp_async_wait_all();
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_QFULL + tile]);
    };
    int ti = 0;
    bool ok = true;
    for (; ok; ++ti) {
      const int qy = TY * tile + ((lane >> 3) & 3), qx = lane & 7;  // brick position (w, qy, qx)
      const uint32_t tl = tbase + ((uint32_t)(w * 32) << 16) + tile * kTileCols;
      const int bb = ti & 1;
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_BOX + bb], (ti >> 1) & 1))) break;
      const int64_t u = unit_of(bb);
      if (u < 0) break;
      if (ti == 0 && w < 2) prepare_a(u, 0);  // the first unit's tiles
      int64_t bh;
      int z0, y0, x0;
      origin(u, bh, z0, y0, x0);
      const int32_t* box = reinterpret_cast<const int32_t*>(smem + S::kBox + bb * kBoxPitch);
      const int cz = z0 + w, cy = y0 + qy, cx = x0 + qx;
      const bool valid = cz < g.gz && cy < g.gy && cx < g.gx;
      const int slot = valid ? box[((w + 1) * kBoxY + qy + 1) * kBoxX + qx + 4] : -1;
      // neighbour bits of the warp's three slices w + i (window column c = slice row 40 tile
      // + c): the window's occupied keys as one ballot mask per slice, a row's 3x3 neighbours
      // the pattern 0b111 in three window rows shifted to its position
      uint64_t nb[3];
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        const int hz = w + i;
        uint32_t half[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int c = hh * 32 + lane;
          bool occ = false;
          if (c < kNV) {
            const int hy = TY * tile + c / HX, hx = c % HX;
            occ = in_grid(z0 - 1 + hz, y0 - 1 + hy, x0 - 1 + hx) &&
                  box[(hz * kBoxY + hy) * kBoxX + hx + 3] >= 0;
          }
          half[hh] = __ballot_sync(0xffffffffu, occ);
        }
        const uint64_t occm = (uint64_t)half[0] | ((uint64_t)half[1] << 32);
        const uint64_t row3 = 7ull << qx;
        const uint64_t pat = (row3 | (row3 << HX) | (row3 << (2 * HX))) << (HX * (qy - TY * tile));
        nb[i] = slot >= 0 ? (pat & occm) : 0ull;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars[B_BOXFREE + bb]);  // this warp is done with the box
      // the row's forward values (a row without a token has no neighbour bit, so P = 0)
      const int64_t row = bh * N + (slot >= 0 ? slot : 0);
      const float nl2 = slot >= 0 ? -P.lse_loc[row] * kLog2e : 0.f;
      const float dl = slot >= 0 ? P.Dl[row] : 0.f;
      const float gt = slot >= 0 ? 1.f / (1.f + __expf(-__bfloat162float(P.gate[row]))) : 0.f;
      // this warp's dq~ rows start at zero (the previous unit's epilogue has read them)
      {
        const uint32_t zr[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) tc::tmem_st16(tl + kDqCol + c0, zr);
      }
      uint64_t* sfull = &bars[B_SFULL + tile * 4 + w];
      uint64_t* pfull = &bars[B_PFULL + tile * 4 + w];
#pragma unroll 1  // (rolled: the kernel's code is large; instruction fetch stalls otherwise)
      for (int i = 0; i < 3; ++i) {
        // S and dP of slice w + i (this warp's phase 3 ti + i)
        if (!__all_sync(0xffffffffu, ab.wait(sfull, (uint32_t)(3 * ti + i) & 1))) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint64_t win = i == 0 ? nb[0] : (i == 1 ? nb[1] : nb[2]);  // (no indexed array)
        // two halves of 32 window columns: dS of half h packed over S columns 16 h .. 16 h + 15
        // (columns the first half has already read)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[32], pv[32];
          tc::tmem_ld32(tl + kSCol + 32 * h, sv);
          tc::tmem_ld32(tl + kPCol + 32 * h, pv);
          tc::tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            float ds[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int col = 32 * h + k + e;
              const float p = ((win >> col) & 1ull)
                                  ? ex2(fmaf(__uint_as_float(sv[k + e]), P.scale_log2, nl2))
                                  : 0.f;
              ds[e] = p * (gt * __uint_as_float(pv[k + e]) - dl) * P.scale;
            }
            pk[k >> 1] = tc::pack_bf16(ds[0], ds[1]);
          }
          tc::tmem_st16(tl + kSCol + 16 * h, pk);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(pfull);
      }
      if (!ok) break;
      // epilogue after the TS of the warp's last slice: dq~ (+ global part) -> R(c)^T -> dq
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_EPI + tile * 4 + w], ti & 1))) break;
      tc::tc_fence_after();
      {
        // 16 columns at a time: + the global part, R(c)^T pair by pair, bf16
        const float4* gq = reinterpret_cast<const float4*>(P.dqg + row * D);
        uint4* dst = reinterpret_cast<uint4*>(P.dq + row * D);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint32_t o[16];
          tc::tmem_ld16(tl + kDqCol + c0, o);
          tc::tmem_wait_ld();
          if (slot >= 0) {  // (the loads above are warp-wide; the rest per lane)
            float acc[16];
  #pragma unroll
            for (int k = 0; k < 16; ++k) acc[k] = __uint_as_float(o[k]);
            if (P.dqg) {
  #pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float4 t4 = gq[c0 / 4 + k];
                acc[4 * k] += t4.x;
                acc[4 * k + 1] += t4.y;
                acc[4 * k + 2] += t4.z;
                acc[4 * k + 3] += t4.w;
              }
            }
  #pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
              const int c = c0 / 8 + hc;  // 16-byte piece of the row
              const int axis = (c * 8) / DA, p0 = ((c * 8) % DA) / 2;
              const int cv = axis == 0 ? cz : (axis == 1 ? cy : cx);
              const float4* cs4 = reinterpret_cast<const float4*>(
                  P.ix.rope + 2 * rope_slot(P.ix.rope_rows, P.ix.rope_pairs, axis, cv, p0));
              const float4 ca = __ldg(cs4), cbv = __ldg(cs4 + 1);
              const float cs[8] = {ca.x, ca.y, ca.z, ca.w, cbv.x, cbv.y, cbv.z, cbv.w};
              uint32_t xo[4];
  #pragma unroll
              for (int k = 0; k < 4; ++k) {
                // the transpose of the rotation: (x0 cos + x1 sin, -x0 sin + x1 cos)
                const float x0 = acc[8 * hc + 2 * k], x1 = acc[8 * hc + 2 * k + 1];
                xo[k] = tc::pack_bf16(x0 * cs[2 * k] + x1 * cs[2 * k + 1],
                                      x1 * cs[2 * k] - x0 * cs[2 * k + 1]);
              }
              dst[c] = make_uint4(xo[0], xo[1], xo[2], xo[3]);
            }
          }
          __syncwarp();
        }
      }
      if (w < 2) {
        // the next unit's q~ / dO tiles, once its slot box is in and this unit's last SS of the
        // tile has completed
        const int nbx = (ti + 1) & 1;
        if (!__all_sync(0xffffffffu, ab.wait(&bars[B_BOX + nbx], ((ti + 1) >> 1) & 1))) break;
        const int64_t un = unit_of(nbx);
        if (un >= 0) {
          if (!__all_sync(0xffffffffu, ab.wait(&bars[B_QEMPTY + tile], ti & 1))) break;
          prepare_a(un, nbx);
        }
      }
    }
    tc::cp_async_wait_all();
  } else if (warp == W_BOX) {
    // --------------------------------------------------------- slot boxes (warp 8)
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity));
    };
    uint32_t box_phases[2] = {0u, 0u};
    for (int ti = 0;; ++ti) {
      const int bb = ti & 1;
      int32_t* box = reinterpret_cast<int32_t*>(smem + S::kBox + bb * kBoxPitch);
      volatile int64_t* uslot =
          reinterpret_cast<volatile int64_t*>(smem + S::kBox + bb * kBoxPitch + kBoxBytes);
      if (ti >= 2 && !wwait(&bars[B_BOXFREE + bb], ((ti >> 1) - 1) & 1)) break;
      unsigned int nu = 0;
      if (lane == 0) nu = atomicAdd(reinterpret_cast<unsigned int*>(P.ix.status + 2), 1u);
      const int64_t u = (int64_t)__shfl_sync(0xffffffffu, nu, 0);
      if (u >= P.units) {
        if (lane == 0) {
          *uslot = -1;
          ++box_phases[bb];
          tc::mbar_arrive(&bars[B_BOX + bb]);
        }
        break;
      }
      int64_t bh;
      int z0, y0, x0;
      origin(u, bh, z0, y0, x0);
      if (lane == 0) *uslot = u;
      __syncwarp();
      if (P.box_tma) {
        if (lane == 0) {
          ++box_phases[bb];
          tc::mbar_expect_tx(&bars[B_BOX + bb], kBoxBytes);
          tc::tma_load_3d(box, &mg, x0 - 4, y0 - 1, z0 - 1, &bars[B_BOX + bb]);
        }
      } else {
        for (int i = lane; i < kBoxX * kBoxY * kBoxZ; i += 32) {
          const int bx = i % kBoxX, by = (i / kBoxX) % kBoxY, bz = i / (kBoxX * kBoxY);
          const int z = z0 - 1 + bz, y = y0 - 1 + by, x = x0 - 4 + bx;
          box[i] = in_grid(z, y, x) ? P.ix.inv[((int64_t)z * g.gy + y) * g.gx + x] : 0;
        }
        __syncwarp();
        if (lane == 0) {
          ++box_phases[bb];
          tc::mbar_arrive(&bars[B_BOX + bb]);
        }
      }
    }
    if (lane == 0)
      for (int b2 = 0; b2 < 2; ++b2)
        if (box_phases[b2] &&
            !tc::mbar_wait(&bars[B_BOX + b2], (box_phases[b2] - 1) & 1, 100000000LL))
          set_status(P.ix.status, PACK3D_ERR_TIMEOUT);
  } else if (warp >= W_PROD && warp < W_MMA) {
    // --------------------------------------------------------- k~ / v rows (128 threads)
    // Halo slice s: 100 rows of k~ (the query head's rotated keys) and of v (the KV head's
    // values), one cp.async per 16-byte piece (rows off the grid or at empty sites zero-filled);
    // each thread's copies arrive on the stage's barrier by themselves when they land.
    const int pt = tid - W_PROD * 32;
    volatile int* pflag = abort_flag + 1;  // [2], used alternately
    int nwait = 0;
    auto pwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      volatile int* f = pflag + (nwait++ & 1);
      if (pt == 0) *f = ab.wait(bar, parity) ? 1 : 0;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      return *f != 0;
    };
    // this thread's pieces, the same in every slice: shared-memory offset / 16, halo (hy, hx)
    // and column, packed as off16 | hy << 16 | hx << 20 | col << 24
    constexpr int KPIECES = kSliceKeys * KC;
    constexpr int NP = (KPIECES + kProd - 1) / kProd;
    uint32_t pc[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      const int p = pt + j * kProd;
      const int key = p / KC, c = p % KC;
      const int hy = key / HX, hx = key % HX;
      const int row = slice_row(hy, hx);
      const int off = c * S::kChunkCol + (row >> 3) * 128 + (row & 7) * 16;
      pc[j] = p < KPIECES ? ((uint32_t)(off >> 4) | ((uint32_t)hy << 16) | ((uint32_t)hx << 20) |
                             ((uint32_t)c << 24))
                          : 0xffffffffu;
    }
    int ti = 0;
    uint32_t gs = 0;
    bool ok = true;
    for (; ok; ++ti) {
      const int bb = ti & 1;
      const int32_t* box = reinterpret_cast<const int32_t*>(smem + S::kBox + bb * kBoxPitch);
      if (!pwait(&bars[B_BOX + bb], (ti >> 1) & 1)) break;
      const int64_t u = unit_of(bb);
      if (u < 0) break;
      int64_t bh;
      int z0, y0, x0;
      origin(u, bh, z0, y0, x0);
      const int64_t kbase = bh * N;                       // k~ rows of the query head
      const int64_t vbase = kv_of(bh, P.kv_group) * N;    // v rows of the KV head
      // per piece, fixed for the unit: the box index of its (hy, hx) column in slice 0 (-1 when
      // the column is off the grid in y or x)
      int bidx[NP];
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        const int hy = (pc[j] >> 16) & 0xf, hx = (pc[j] >> 20) & 0xf;
        const int y = y0 - 1 + hy, x = x0 - 1 + hx;
        bidx[j] = (pc[j] != 0xffffffffu && y >= 0 && y < g.gy && x >= 0 && x < g.gx)
                      ? hy * kBoxX + hx + 3
                      : -1;
      }
      const __nv_bfloat16* kgb = P.kr + kbase * D;
      const __nv_bfloat16* vgb = P.v + vbase * D;
      for (int s = 0; s < kChunks; ++s, ++gs) {
        const int st = gs % kStages;
        if (gs >= (uint32_t)kStages && !pwait(&bars[B_KVEMPTY + st], ((gs / kStages) - 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* kd = smem + S::kK + st * S::kStage;
        uint8_t* vd = smem + S::kV + st * S::kStage;
        const bool zin = z0 - 1 + s >= 0 && z0 - 1 + s < g.gz;
        const int32_t* sbox = box + s * kBoxY * kBoxX;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          if (pc[j] == 0xffffffffu) continue;
          const int slot = (zin && bidx[j] >= 0) ? sbox[bidx[j]] : -1;
          const int64_t src = (int64_t)(slot >= 0 ? slot : 0) * D + (int)(pc[j] >> 24) * 8;
          const uint32_t off = (pc[j] & 0xffffu) << 4;
          tc::cp_async16(kd + off, kgb + src, slot >= 0);
          tc::cp_async16(vd + off, vgb + src, slot >= 0);
        }
        tc::cp_async_arrive_noinc(&bars[B_KVFULL + st]);
      }
      if (!ok) break;
      __syncwarp();
      if ((pt & 31) == 0) tc::mbar_arrive(&bars[B_BOXFREE + bb]);
    }
    tc::cp_async_wait_all();
  } else if (warp >= W_MMA) {
    // --------------------------------------------------------- MMA issuers (warps 14, 15)
    // One warp per tile. Per slice s: SS (S and dP) once the previous slice's TS has completed
    // (S / dP are single-buffered), then TS once the slice's owners have written dS. The whole
    // warp runs the schedule with warp-uniform values; one elected lane issues and commits.
    const int tile = warp - W_MMA;
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0) + tile * kTileCols;
    const uint32_t id_ss = tc::idesc_bf16_f32(128, kNK, false, false);
    const uint32_t id_ts = tc::idesc_bf16_f32(128, D, false, true);
    // no-swizzle descriptors: A tiles and k~ / v as K-major (lbo = column-chunk stride, sbo =
    // 8 rows), k~ as the MN-major B of the TS (lbo = 8 key rows, sbo = column-chunk stride);
    // the tile's window starts at slice row 40 tile
    const uint64_t qd = tc::smem_desc(tc::smem_u32(smem + S::a_off(tile, 0)), S::kQCol, 128);
    const uint64_t gd = tc::smem_desc(tc::smem_u32(smem + S::a_off(tile, 1)), S::kQCol, 128);
    const uint64_t kd0 =
        tc::smem_desc(tc::smem_u32(smem + S::kK + (kWin * tile / 8) * 128), S::kChunkCol, 128);
    const uint64_t vd0 =
        tc::smem_desc(tc::smem_u32(smem + S::kV + (kWin * tile / 8) * 128), S::kChunkCol, 128);
    const uint64_t km0 =
        tc::smem_desc(tc::smem_u32(smem + S::kK + (kWin * tile / 8) * 128), 128, S::kChunkCol);
    uint64_t* sfull = &bars[B_SFULL + tile * 4];
    uint64_t* pfull = &bars[B_PFULL + tile * 4];
    uint64_t* tsdone = &bars[B_TSDONE + tile];
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    int ti = 0;
    uint32_t gs = 0;
    bool ok = true;
    for (; ok; ++ti) {
      if (!wwait(&bars[B_BOX + (ti & 1)], (ti >> 1) & 1) || unit_of(ti & 1) < 0) break;
      if (!wwait(&bars[B_QFULL + tile], ti & 1)) break;
      tc::tc_fence_after();
      for (int s = 0; s < kChunks && ok; ++s, ++gs) {
        const int st = gs % kStages;
        const int wlo = owner_lo(s), whi = owner_hi(s);
        if (!wwait(&bars[B_KVFULL + st], (gs / kStages) & 1)) { ok = false; break; }
        if (gs > 0 && !wwait(tsdone, (gs - 1) & 1)) { ok = false; break; }
        // the slice arrived through cp.async (generic proxy); the MMAs read it through the
        // async proxy
        tc::fence_proxy_async_smem();
        tc::tc_fence_after();
        const uint64_t so = (uint64_t)((st * S::kStage) >> 4);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {  // 16 columns = two column chunks
            tc::mma_ss(tb + kSCol, qd + (uint64_t)(ks * ((2 * S::kQCol) >> 4)),
                       kd0 + so + (uint64_t)(ks * ((2 * S::kChunkCol) >> 4)), id_ss, ks > 0);
            tc::mma_ss(tb + kPCol, gd + (uint64_t)(ks * ((2 * S::kQCol) >> 4)),
                       vd0 + so + (uint64_t)(ks * ((2 * S::kChunkCol) >> 4)), id_ss, ks > 0);
          }
          for (int w = wlo; w <= whi; ++w) tc::tc_commit(&sfull[w]);
          if (s == kChunks - 1) tc::tc_commit(&bars[B_QEMPTY + tile]);  // A tiles free again
        }
        __syncwarp();
        for (int w = wlo; w <= whi && ok; ++w)
          ok = wwait(&pfull[w], (uint32_t)(3 * ti + s - w) & 1);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t m0 = (0 < wlo || 0 > whi) ? 0xffffffffu : 0u;
        const uint32_t m1 = (1 < wlo || 1 > whi) ? 0xffffffffu : 0u;
        const uint32_t m2 = (2 < wlo || 2 > whi) ? 0xffffffffu : 0u;
        const uint32_t m3 = (3 < wlo || 3 > whi) ? 0xffffffffu : 0u;
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kNK / 16; ++ks)  // 16 key rows = two row groups
            tc::mma_ts_masked(tb + kDqCol, tb + kSCol + ks * 8, km0 + so + (uint64_t)(ks * (256 >> 4)),
                              id_ts, 1u, m0, m1, m2, m3);
          tc::tc_commit(tsdone);
          tc::tc_commit(&bars[B_KVEMPTY + st]);
          if (s >= 2) tc::tc_commit(&bars[B_EPI + tile * 4 + (s - 2)]);  // warp s-2 done
        }
        __syncwarp();
      }
    }
    if (tc::elect_one()) tc::tc_commit(&bars[B_DRAIN + tile]);
    __syncwarp();
    if (!tc::mbar_wait(&bars[B_DRAIN + tile], 0, 100000000LL))
      set_status(P.ix.status, PACK3D_ERR_TIMEOUT);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
  if (tid == 0) {
    // the last CTA out puts the unit counter (and this count) back to zero for the next call
    unsigned int* ctr = reinterpret_cast<unsigned int*>(P.ix.status + 2);
    __threadfence();
    if (atomicAdd(ctr + 1, 1u) == gridDim.x - 1) {
      atomicExch(ctr, 0u);
      atomicExch(ctr + 1, 0u);
    }
  }
}

// ------------------------------------------------------------------------------ host side

template <int D>
cudaError_t launch_bwd_local_dq_tc(const pack3d_index& ix, const BwdWork& w, const void* v,
                                   const void* dO, const void* gate, const float* lse_loc,
                                   int64_t bh, int kv_group, float scale, void* dq,
                                   cudaStream_t s) {
  using namespace lb;
  static std::atomic<uint64_t> attr_done{0};
  if (smem_attr_once(reinterpret_cast<const void*>(k_bwd_local_dq_tc<D>), Smem<D>::kBytes,
                     attr_done) != cudaSuccess)
    return cudaErrorInvalidValue;
  Params p;
  p.ix = ix;
  p.qr = static_cast<const __nv_bfloat16*>(w.qr);
  p.kr = static_cast<const __nv_bfloat16*>(w.kr);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.lse_loc = lse_loc;
  p.Dl = w.Dl;
  p.dqg = w.dqg;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.wait_budget = wait_budget_cycles();
  p.kv_group = kv_group;
  p.nbz = (ix.geom.gz + BZ - 1) / BZ;
  p.nby = (ix.geom.gy + BY - 1) / BY;
  p.nbx = (ix.geom.gx + BX - 1) / BX;
  p.units = bh * p.nbz * p.nby * p.nbx;
  if (p.units <= 0) return cudaSuccess;
  if (!ix.status || p.units >= 0x7fffffffLL) return cudaErrorInvalidValue;  // unit counter
  CUtensorMap mg;
  memset(&mg, 0, sizeof(mg));
  p.box_tma = encode_grid_i32(&mg, ix.inv, ix.geom.gz, ix.geom.gy, ix.geom.gx, kBoxX, kBoxY, kBoxZ)
                  ? 1
                  : 0;
  const int64_t cap = sm_count();
  const unsigned grid = (unsigned)(p.units < cap ? p.units : cap);
  k_bwd_local_dq_tc<D><<<grid, kThreads, Smem<D>::kBytes, s>>>(mg, p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t bwd_local_dq_tc_dispatch(const pack3d_index& ix, const BwdWork& w, const void* v,
                                     const void* dO, const void* gate, const float* lse_loc,
                                     int64_t bh, int kv_group, float scale, void* dq,
                                     cudaStream_t s) {
  if (ix.geom.head_dim == 96)
    return launch_bwd_local_dq_tc<96>(ix, w, v, dO, gate, lse_loc, bh, kv_group, scale, dq, s);
  return launch_bwd_local_dq_tc<48>(ix, w, v, dO, gate, lse_loc, bh, kv_group, scale, dq, s);
}

}  // namespace p3d
