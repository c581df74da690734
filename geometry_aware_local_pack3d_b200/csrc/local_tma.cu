// Local branch of PACK3D attention on tcgen05 tensor cores (bf16 I/O, head_dim 48 or 96), for
// raw keys (ROT: the producer warps rotate each key row in shared memory once it has landed) or
// for keys rotated once up front by pack3d_summarize_rotated (gathered as they are).
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 1: each query
// attends exactly to every token of its 3x3x3 coordinate neighbourhood, found by coordinate,
// never by adjacency in memory; paper summary §3.5: streamed online softmax, no gathered
// neighbour tensor in memory.
//
// Work unit: one 4x8x8 (z, y, x) brick of one (batch, head), split into two 128-query tiles
// (y0..y0+3 and y0+4..y0+7); one persistent CTA per SM. The two tiles share one stream of
// halo z-slices (6 slices of 10x10 = 100 keys), so a key row is fetched once for 256 queries.
// Units are handed out by a device-wide counter (status word 2 of the index; the last CTA to
// finish puts it back to zero), so SMs that run slower take fewer units. Per unit:
//   * one 3D TMA box load brings the memory slots of the unit's 6x10x10 halo from the inverse
//     map (x start rounded down to a 16-byte boundary: box 16x10x6 int32);
//   * four producer warps fetch, per halo z-slice, the 100 key rows and value rows with one
//     cp.async per 16-byte piece (rows off the grid or at empty sites are zero-filled) into the
//     no-swizzle core-matrix layout, four stages deep. With rotated keys each thread's copies
//     arrive on the stage's barrier by themselves when they land; with raw keys each thread
//     waits for its copies of a slice (the next slice's copies already in flight), rotates its
//     key pieces in place by the key's coordinate (known from the halo position) and then
//     arrives;
//   * one q buffer per tile: softmax warps 0 and 1 of each tile, idle once their slices of a
//     unit are done, load the next unit's q rows (64 rows each, one row per lane), rotate them
//     in registers (axial RoPE by the row's coordinates) and store them into the tile's buffer
//     as soon as the tile's last QK of the unit has completed, while the unit's last slices
//     are still being worked on (a second q buffer would cost the fourth k/v stage).
// Slice key order: halo row hy major, then halo column hx (row 10 hy + hx), so tile t's keys
// (halo rows 4t .. 4t+5) are slice rows 40t .. 40t+59: each tile works on a 64-row window
// starting at slice row 40 t (rows 100..103 of a stage are zero padding).
// Row r = 32 z + 8 y + x of a tile holds brick position (z, 4 t + y, x): warp w is the z-plane
// w of the brick, so it needs exactly slices w .. w+2, and slice s is owned by warps
// max(0, s-2) .. min(3, s). Per tile and slice:
//   S_s = q~ k~_s^T   (SS MMA 128 x 64, fp32, TMEM buffer s % 2)
//   owners: 3x3x3 mask, online softmax over the window's first 60 columns (the only ones that
//   can hold a neighbour of the tile), P = exp2(s - m) as bf16 over the buffer's first 32
//   columns (P = 0 in window columns 60..63);  O += P_s v_s  (TS MMA, N = d) with the rows
//   of the other warps disabled through the MMA's output-lane mask, so non-owners never touch
//   slice s.
// Each tile has its own MMA warp; QK runs two slices ahead of PV, so S_{s+2} is ready when the
// owners finish slice s + 1. Each softmax warp zeroes its O rows when it starts a unit; its
// epilogue runs after the PV of its last slice. Every query sits at the same row and every
// neighbour at the same column whatever the packing, so a coordinate-carrying repack permutes
// the output bit for bit.
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace p3d {

namespace lg {
constexpr int BZ = 4, BY = 8, BX = 8;  // unit; two tiles of 4 x 4 x 8 (z, y, x)
constexpr int kTiles = 2;
constexpr int TY = BY / kTiles;        // 4 y-rows per tile
constexpr int HY = BY + 2, HX = BX + 2;
constexpr int kChunks = BZ + 2;        // 6 halo z-slices
constexpr int kSliceKeys = HY * HX;    // 100
constexpr int kNK = 64;                // tile window (MMA N of QK, K of PV)
constexpr int kNV = (TY + 2) * HX;     // 60 window columns that can hold a neighbour
constexpr int kWin = TY * HX;          // 40: first slice row of tile 1's window
constexpr int kRows = kWin + kNK;      // 104 rows per stage
constexpr int kStages = 4;
// warps: softmax 0-7 (tile = warp / 4; warps 0, 1, 4, 5 also prepare q tiles), slot boxes 8
// (warp 9 idle), k/v producers 10-13, MMA 14-15 (tile = warp - 14)
constexpr int kThreads = 512;
constexpr int W_BOX = 8, W_PROD = 10, W_MMA = 14;
constexpr int kProd = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;  // per tile: S buffers at 0 / 64, O at 128
constexpr uint32_t kOCol = 128;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kBoxX = 16, kBoxY = HY, kBoxZ = kChunks;  // slot box: x from x0 - 4
constexpr int kBoxBytes = kBoxX * kBoxY * kBoxZ * 4;
constexpr int kBoxPitch = 4096;  // box, then the unit index (int64) at kBoxBytes

__device__ __forceinline__ uint32_t s_col(int b) { return b ? 64u : 0u; }

// slice row of halo position (hy, hx): halo row major
__host__ __device__ constexpr int slice_row(int hy, int hx) { return hy * HX + hx; }

// Shared memory. Operands use the no-swizzle core-matrix layout: the 16-byte piece (row r,
// column chunk c) of a q tile sits at c * kQCol + (r / 8) * 128 + (r % 8) * 16 and that of a
// k or v stage at c * kChunkCol + (row / 8) * 128 + (row % 8) * 16. Each column-chunk stride
// carries 16 bytes of padding, so consecutive pieces of one row -- the order in which they are
// read from global memory -- fall on distinct shared-memory banks.
template <int D> struct Smem {
  static constexpr int KC = D / 8;                 // 16-byte pieces of a row
  static constexpr int kQCol = 128 * 16 + 16;      // one 16-byte column of a q tile
  static constexpr int kQBuf = KC * kQCol;         // one q tile
  static constexpr int kChunkCol = kRows * 16 + 16;
  static constexpr int kStage = KC * kChunkCol;
  static constexpr int kQ = 0;                            // [2 tiles] q tiles, one buffer each
  static constexpr int kK = kQ + kTiles * kQBuf;          // [kStages] key chunks
  static constexpr int kV = kK + kStages * kStage;        // [kStages] value chunks
  static constexpr int kBox = (kV + kStages * kStage + 127) / 128 * 128;  // [2] slot boxes (TMA)
  static constexpr int kBar = kBox + 2 * kBoxPitch;
  static constexpr int kBytes = kBar + 1024;
  static_assert(kBox % 128 == 0, "box alignment");
  static_assert(kBoxBytes + 8 <= kBoxPitch, "slot box and unit index");
  static_assert(kBytes <= 232448, "dynamic shared memory of one CTA");
  __device__ static int q_off(int r, int c) { return c * kQCol + (r >> 3) * 128 + (r & 7) * 16; }
};

enum {
  B_QFULL = 0, B_QEMPTY = 4,  // [tile] (slots 2, 3 and 6, 7 unused)
  B_KVFULL = 8, B_KVEMPTY = 12, B_BOX = 16, B_BOXFREE = 18,
  B_SFULL = 20,  // [tile][warp][buffer]
  B_PFULL = 36,  // [tile][warp][buffer]
  B_PVALL = 52,  // [tile]
  B_EPI = 54,    // [tile][warp]
  B_DRAIN = 62,  // [tile]
  B_COUNT = 64
};
static_assert(8 * B_COUNT + 16 <= 1024, "barrier area");

struct Params {
  pack3d_index ix;
  const __nv_bfloat16* q;      // [B, H, N, d]
  const __nv_bfloat16* k;      // keys [B, H_kv, N, d]: raw (ROT) or rotated
  const __nv_bfloat16* v;
  __nv_bfloat16* o_loc;
  float* lse_loc;  // optional
  float scale_log2;
  int nbz, nby, nbx;
  int box_tma;        // slot boxes by TMA (else plain loads)
  int64_t units;      // batch * heads * units per field
  int kv_group;       // query heads per KV head: k_rot and v rows of KV head bh / kv_group
  long long wait_budget;  // SM cycles of each bounded wait
  // RoPE angle per unit coordinate of rotation pair p on axis a: spacing_a * base^(-2p / d_a)
  float theta[3][16];
};

// (cos, sin) of the RoPE angle c * theta of integer coordinate c, computed in registers (the
// q preparation would otherwise load the rotation table from global memory, two 16-byte loads
// per 16-byte piece, on the path between units). The product is reduced to [-pi, pi] by the
// two-constant Cody-Waite method (2 pi = kTwoPiHi + kTwoPiLo, kTwoPiHi the float nearest to
// 2 pi) and the reduced angle goes to the fast sine and cosine. Absolute error about
// 1e-7 * |c * theta| + 1e-6 against the float64 angle: far below the bf16 rounding of q~.
__device__ __forceinline__ float2 rope_angle_cs(int c, float theta) {
  constexpr float kInv2Pi = 0.159154943091895336f;
  constexpr float kTwoPiHi = 6.28318548202514648f;
  constexpr float kTwoPiLo = -1.74845560007448e-07f;
  const float a = (float)c * theta;
  const float n = rintf(a * kInv2Pi);
  const float r = fmaf(-n, kTwoPiLo, fmaf(-n, kTwoPiHi, a));
  float sn, cn;
  __sincosf(r, &sn, &cn);
  return make_float2(cn, sn);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}


// clock64 trace slots of the first four units a CTA processes (tracing builds only)
#define GTR(ti, off)                                       \
  do {                                                     \
    if ((ti) < 4) P3D_TRACE_C((ti) * 400 + (off));         \
  } while (0)

#ifdef P3D_TRACE_ENABLED
// global-timer stamp of each CTA's first 32 unit starts (MMA warp of tile 0), tracing builds
static __device__ unsigned long long g_brick_t[512 * 32];
#define BRICK_T(ti)                                                                       \
  do {                                                                                    \
    if ((ti) < 32 && blockIdx.x < 512) {                                                  \
      unsigned long long t_;                                                              \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                              \
      g_brick_t[blockIdx.x * 32 + (ti)] = t_;                                             \
    }                                                                                     \
  } while (0)
#else
#define BRICK_T(ti) \
  do {              \
  } while (0)
#endif

// first and last softmax warp owning halo slice s (warp w needs slices w .. w + 2)
__device__ __forceinline__ int owner_lo(int s) { return max(0, s - 2); }
__device__ __forceinline__ int owner_hi(int s) { return min(3, s); }
// Parity of the wait of warp w on its S / P barrier of slice s (buffer s % 2) in unit ti:
// per unit the buffer of parity w % 2 serves slices w and w + 2 (two phases), the other
// buffer slice w + 1 (one phase).
__host__ __device__ __forceinline__ uint32_t sp_parity(int w, int s, int ti) {
  const int i = s - w;
  return (i & 1) ? (uint32_t)(ti & 1) : (uint32_t)((i >> 1) & 1);
}

}  // namespace lg

template <int D, bool ROT>
__global__ void __launch_bounds__(lg::kThreads, 1)
    k_local_tma(const __grid_constant__ CUtensorMap mg, const lg::Params P) {
  using namespace lg;
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
  // unit published with slot box bb (-1: no more units), valid once B_BOX[bb] has completed
  auto unit_of = [&](int bb) -> int64_t {
    return *reinterpret_cast<volatile int64_t*>(smem + S::kBox + bb * kBoxPitch + kBoxBytes);
  };

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(&bars[B_QFULL + i], 64);  // softmax warps 0 and 1 of the tile
      tc::mbar_init(&bars[B_QEMPTY + i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars[B_KVFULL + i], kProd);
      tc::mbar_init(&bars[B_KVEMPTY + i], kTiles);  // one commit per tile's MMA warp
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_BOX + i], 1);
      tc::mbar_init(&bars[B_BOXFREE + i], 8 + 4);  // softmax and producer warps
    }
    for (int i = 0; i < 16; ++i) {
      tc::mbar_init(&bars[B_SFULL + i], 1);
      tc::mbar_init(&bars[B_PFULL + i], 32);
    }
    for (int i = 0; i < kTiles; ++i) {
      tc::mbar_init(&bars[B_PVALL + i], 1);
      tc::mbar_init(&bars[B_DRAIN + i], 1);
    }
    for (int i = 0; i < 8; ++i) tc::mbar_init(&bars[B_EPI + i], 1);
    abort_flag[0] = 0;
    tc::fence_mbar_init();
  }
  if (warp == W_BOX && lane == 0 && P.box_tma) tc::tma_prefetch_desc(&mg);
  // rows 100..103 of every k/v stage are never written by the producers: zero them once
  // (tile 1's MMAs read them; their scores are masked, and P = 0 times a zero v row is 0)
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
    // --------------------------------------------------------- softmax + epilogue (row = lane)
    const int tile = warp >> 2, w = warp & 3;
    // q tile of unit `un` (slot box nb) into q buffer qi: warp w (0 or 1) takes rows
    // 64 w .. 64 w + 63, one row per lane and pass -- loaded, rotated in registers by the row's
    // coordinates (axial RoPE) and stored in the operand layout -- then publishes its share
    // (QFULL: 64 arrivals per tile). Row r of a tile holds brick position
    // (r / 32, 4 tile + (r / 8) % 4, r % 8); rows off the grid or at empty sites are zero.
    auto prepare_q = [&](int64_t un, int nb, int qi, int tix) {
      if (lane == 0 && tile == 0) GTR(tix, 200 + w * 2);
      int64_t qbh;
      int qz0, qy0, qx0;
      origin(un, qbh, qz0, qy0, qx0);
      const int32_t* qbox = reinterpret_cast<const int32_t*>(smem + S::kBox + nb * kBoxPitch);
      uint8_t* qd = smem + S::kQ + qi * S::kQBuf;
      const int rmax = P.ix.rope_rows - 1;
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        const int r = 64 * w + 32 * pass + lane;
        const int z = r >> 5, y = TY * tile + ((r >> 3) & 3), x = r & 7;
        const int slot = in_grid(qz0 + z, qy0 + y, qx0 + x)
                             ? qbox[((z + 1) * kBoxY + y + 1) * kBoxX + x + 4]
                             : -1;
        const uint4* src =
            reinterpret_cast<const uint4*>(P.q + (qbh * N + (slot >= 0 ? slot : 0)) * D);
        uint4 row[KC];
#pragma unroll
        for (int c = 0; c < KC; ++c) row[c] = src[c];
        const int cz = min(qz0 + z, rmax), cy = min(qy0 + y, rmax), cx = min(qx0 + x, rmax);
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          const int axis = (c * 8) / DA, p0 = ((c * 8) % DA) / 2;
          const int cv = axis == 0 ? cz : (axis == 1 ? cy : cx);
          // (cos, sin) of the piece's 4 rotation pairs
          float cs[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 e = rope_angle_cs(cv, P.theta[axis][p0 + k]);
            cs[2 * k] = e.x;
            cs[2 * k + 1] = e.y;
          }
          const uint32_t xin[4] = {row[c].x, row[c].y, row[c].z, row[c].w};
          uint32_t xo[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float e0 = __uint_as_float(xin[k] << 16);
            const float e1 = __uint_as_float(xin[k] & 0xffff0000u);
            xo[k] = tc::pack_bf16(e0 * cs[2 * k] - e1 * cs[2 * k + 1],
                                  e0 * cs[2 * k + 1] + e1 * cs[2 * k]);
          }
          if (slot < 0) xo[0] = xo[1] = xo[2] = xo[3] = 0u;
          *reinterpret_cast<uint4*>(qd + S::q_off(r, c)) = make_uint4(xo[0], xo[1], xo[2], xo[3]);
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_QFULL + qi]);
      if (lane == 0 && tile == 0) GTR(tix, 201 + w * 2);
    };
    int ti = 0;
    bool ok = true;
    for (; ok; ++ti) {
      // lane-derived values from opaque copies each unit (keeps the score row in registers)
      int ln = lane;
      uint32_t tl = tbase;
      asm volatile("" : "+r"(ln), "+r"(tl));
      tl += ((uint32_t)(w * 32) << 16) + tile * kTileCols;
      const int qy = TY * tile + ((ln >> 3) & 3), qx = ln & 7;  // brick position (w, qy, qx)
      const int bb = ti & 1;
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_BOX + bb], (ti >> 1) & 1))) break;
      const int64_t u = unit_of(bb);
      if (u < 0) break;
      if (ti == 0 && w < 2) prepare_q(u, 0, tile, 0);  // the first unit's q tile
      int64_t bh;
      int z0, y0, x0;
      origin(u, bh, z0, y0, x0);
      const int32_t* box = reinterpret_cast<const int32_t*>(smem + S::kBox + bb * kBoxPitch);
      const int cz = z0 + w, cy = y0 + qy, cx = x0 + qx;
      const bool valid = cz < g.gz && cy < g.gy && cx < g.gx;
      // neighbour bits of the warp's three slices w + i (i = 1 + dz): bit c of the tile's
      // window holds slice row 40 tile + c. The window's occupied keys (inside the grid, not an
      // empty site) are one mask per slice, two window keys per lane and a ballot each; a row's
      // 3x3 neighbours are the pattern 0b111 in three window rows, shifted to its position.
      uint64_t nb[3];
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        const int hz = w + i;  // halo slice
        uint32_t half[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int c = hh * 32 + ln;  // window column
          bool occ = false;
          if (c < kNV) {
            const int hy = TY * tile + c / HX, hx = c % HX;
            occ = in_grid(z0 - 1 + hz, y0 - 1 + hy, x0 - 1 + hx) &&
                  box[(hz * kBoxY + hy) * kBoxX + hx + 3] >= 0;
          }
          half[hh] = __ballot_sync(0xffffffffu, occ);
        }
        const uint64_t occm = (uint64_t)half[0] | ((uint64_t)half[1] << 32);
        const uint64_t row3 = 7ull << qx;  // halo x = qx .. qx + 2
        const uint64_t pat = (row3 | (row3 << HX) | (row3 << (2 * HX))) << (HX * (qy - TY * tile));
        nb[i] = valid ? (pat & occm) : 0ull;
      }
      // this warp's O rows start at zero (the previous unit's epilogue has read them)
      {
        const uint32_t zr[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) tc::tmem_st16(tl + kOCol + c0, zr);
      }
      if (ln == 0 && tile == 0) GTR(ti, 220 + w);  // preamble done
      uint64_t* sfull = &bars[B_SFULL + (tile * 4 + w) * 2];
      uint64_t* pfull = &bars[B_PFULL + (tile * 4 + w) * 2];
      float m_run = -INFINITY, l_run = 0.f;
#pragma unroll 1  // (rolled: the kernel's code is large; instruction fetch stalls otherwise)
      for (int i = 0; i < 3; ++i) {
        const int s = w + i, b = s & 1;
        const uint32_t gs = (uint32_t)ti * kChunks + s;
        if (!__all_sync(0xffffffffu, ab.wait(&sfull[b], sp_parity(w, s, ti)))) {
          ok = false;
          break;
        }
        if (ln == 0 && tile == 0) GTR(ti, 110 + w * 20 + i * 4);
        tc::tc_fence_after();
        // the slice's first 60 window scores (the rest never hold a neighbour of this tile);
        // entries off the 3x3x3 cube become -inf
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        uint32_t r[kNV];
        tc::tmem_ld32(tl + s_col(b), *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tc::tmem_ld16(tl + s_col(b) + 32, *reinterpret_cast<uint32_t(*)[16]>(&r[32]));
        lg::tmem_ld8(tl + s_col(b) + 48, &r[48]);
        lg::tmem_ld4(tl + s_col(b) + 56, &r[56]);
        tc::tmem_wait_ld();
        const uint64_t win = i == 0 ? nb[0] : (i == 1 ? nb[1] : nb[2]);  // (no indexed array)
#pragma unroll
        for (int k = 0; k < kNV; k += 2) {
          if (!((win >> k) & 1ull)) r[k] = 0xff800000u;
          if (!((win >> (k + 1)) & 1ull)) r[k + 1] = 0xff800000u;
          mx[(k >> 1) & 3] =
              tc::max3f(mx[(k >> 1) & 3], __uint_as_float(r[k]), __uint_as_float(r[k + 1]));
        }
        const float cmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * P.scale_log2;
        const float m_new = fmaxf(m_run, cmax);
        const bool need = m_new > m_run + kRescaleLog2;
        // a row that has met no neighbour yet holds O = 0 and needs no rescaling
        const bool rescale = need && m_run != -INFINITY;
        if (i > 0 && __any_sync(0xffffffffu, rescale)) {
          // O rows hold earlier chunks at the old max: rescale once the previous PV is done
          // (PVALL phase gs - 1 is the only incomplete or just-completed phase here)
          if (!__all_sync(0xffffffffu, ab.wait(&bars[B_PVALL + tile], (gs - 1) & 1))) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const float f = rescale ? ex2(m_run - m_new) : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t o[16];
            tc::tmem_ld16(tl + kOCol + c0, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
            tc::tmem_st16(tl + kOCol + c0, o);
          }
        }
        if (need) {
          l_run *= ex2(m_run - m_new);
          m_run = m_new;
        }
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
        // scaling and row sum two columns per instruction (packed fp32)
        float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        const float2 sl2 = make_float2(P.scale_log2, P.scale_log2), nm2 = make_float2(neg_m, neg_m);
        uint32_t p[kNK / 2];
#pragma unroll
        for (int k = kNV; k < kNK; k += 2) p[k >> 1] = 0u;  // P = 0 where no neighbour can be
#pragma unroll
        for (int k = 0; k < kNV; k += 2) {
          const float2 x =
              tc::fma2(make_float2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), sl2, nm2);
          const float2 e = make_float2(ex2(x.x), ex2(x.y));
          ls[(k >> 1) & 3] = tc::add2(ls[(k >> 1) & 3], e);
          p[k >> 1] = tc::pack_bf16(e.x, e.y);
        }
        l_run += ((ls[0].x + ls[0].y) + (ls[1].x + ls[1].y)) + ((ls[2].x + ls[2].y) + (ls[3].x + ls[3].y));
        tc::tmem_st16(tl + s_col(b), *reinterpret_cast<uint32_t(*)[16]>(&p[0]));
        tc::tmem_st16(tl + s_col(b) + 16, *reinterpret_cast<uint32_t(*)[16]>(&p[16]));
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&pfull[b]);
        if (ln == 0 && tile == 0) GTR(ti, 111 + w * 20 + i * 4);
      }
      if (!ok) break;
      // epilogue after the PV of the warp's last slice: o_loc = O / l, lse_loc
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_EPI + tile * 4 + w], ti & 1))) break;
      tc::tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      uint32_t ow[D / 2];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t o[16];
        tc::tmem_ld16(tl + kOCol + c0, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 8; ++k)
          ow[c0 / 2 + k] =
              tc::pack_bf16(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
      }
      const int slot = valid ? box[((w + 1) * kBoxY + qy + 1) * kBoxX + qx + 4] : -1;
      __syncwarp();
      if (ln == 0) tc::mbar_arrive(&bars[B_BOXFREE + bb]);
      if (ln == 0 && tile == 0) GTR(ti, 190 + w);
      if (slot >= 0) {
        uint4* dst = reinterpret_cast<uint4*>(P.o_loc + (bh * N + slot) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          dst[c] = make_uint4(ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
        if (P.lse_loc)
          P.lse_loc[bh * N + slot] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
      if (w < 2) {
        // the next unit's q tile, into the tile's q buffer once its slot box is in and this
        // unit's last QK of the tile has completed
        const int nb = (ti + 1) & 1;
        if (!__all_sync(0xffffffffu, ab.wait(&bars[B_BOX + nb], ((ti + 1) >> 1) & 1))) break;
        const int64_t un = unit_of(nb);
        if (un >= 0) {
          if (!__all_sync(0xffffffffu, ab.wait(&bars[B_QEMPTY + tile], ti & 1))) break;
          prepare_q(un, nb, tile, ti + 1);
        }
      }
    }
  } else if (warp == W_BOX) {
    // --------------------------------------------------------- slot boxes (warp 8)
    // Per unit: the next unit index from the device-wide counter, posted with the unit's slot
    // box (3D TMA, or plain loads when the grid pitch does not suit TMA); -1 when none is left.
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity));
    };
    uint32_t box_phases[2] = {0u, 0u};  // phases started on B_BOX (lane 0), for the exit
    for (int ti = 0;; ++ti) {
      const int bb = ti & 1;
      int32_t* box = reinterpret_cast<int32_t*>(smem + S::kBox + bb * kBoxPitch);
      volatile int64_t* uslot =
          reinterpret_cast<volatile int64_t*>(smem + S::kBox + bb * kBoxPitch + kBoxBytes);
      if (lane == 0) GTR(ti, 0);
      if (ti >= 2 && !wwait(&bars[B_BOXFREE + bb], ((ti >> 1) - 1) & 1)) break;
      if (lane == 0) GTR(ti, 1);
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
        // the box is read below (this phase of its barrier completes when it has landed)
        if (!wwait(&bars[B_BOX + bb], (ti >> 1) & 1)) break;
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
      // The unit's q rows are read by two softmax warps per tile when the unit before it
      // ends, between two units' MMA chains; start bringing them into L2 now, about one unit
      // ahead (one bulk prefetch per present row of the 4 x 8 x 8 brick).
      for (int i = lane; i < 4 * 8 * 8; i += 32) {
        const int z = i >> 6, y = (i >> 3) & 7, x = i & 7;
        if (!in_grid(z0 + z, y0 + y, x0 + x)) continue;
        const int slot = box[((z + 1) * kBoxY + y + 1) * kBoxX + x + 4];
        if (slot >= 0) tc::prefetch_l2(P.q + (bh * N + slot) * D, D * 2);
      }
    }
    // nothing may still be landing in shared memory when the CTA exits: wait for the latest
    // phase of each box barrier (phases complete in order; bounded waits; lane 0's counts)
    if (lane == 0)
      for (int b2 = 0; b2 < 2; ++b2)
        if (box_phases[b2] &&
            !tc::mbar_wait(&bars[B_BOX + b2], (box_phases[b2] - 1) & 1, 100000000LL))
          set_status(P.ix.status, PACK3D_ERR_TIMEOUT);
  } else if (warp >= W_PROD && warp < W_MMA) {
    // --------------------------------------------------------- k/v rows (128 threads)
    // Halo slice s of keys and values: 100 rows x d, one cp.async per 16-byte piece in
    // row-contiguous order (rows off the grid or at empty sites are zero-filled). Rotated keys:
    // each thread's copies arrive on the stage's barrier by themselves when they land, so the
    // warps run ahead as far as the free stages allow. Raw keys (ROT): slice s's copies are
    // issued, then the thread waits for its copies of slice s - 1, rotates those key pieces in
    // place and arrives for slice s - 1.
    const int pt = tid - W_PROD * 32;
    volatile int* pflag = abort_flag + 1;  // [2], used alternately
    int nwait = 0;
    // one bounded wait by one thread, its verdict shared with all 128 (named barrier 2)
    auto pwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      volatile int* f = pflag + (nwait++ & 1);
      if (pt == 0) *f = ab.wait(bar, parity) ? 1 : 0;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      return *f != 0;
    };
    // this thread's pieces, the same in every slice: shared-memory offset / 16, halo (hy, hx)
    // and column, packed as off16 | hy << 16 | hx << 20 | col << 24 (pieces in halo order,
    // y-major over x; the stage row is slice_row(hy, hx))
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
    const __nv_bfloat16* kg = P.k;
    const __nv_bfloat16* vg = P.v;
    const int pairs = P.ix.rope_pairs;
    // rotation of this thread's key pieces of slice s (stage st) in place: the key's
    // coordinate is its halo position; pieces of rows off the grid stay zero
    auto rotate_slice = [&](int s, int st, int z0, int y0, int x0) {
      uint8_t* kd = smem + S::kK + st * S::kStage;
      const int zc = z0 - 1 + s;
#pragma unroll
      for (int j = 0; j < NP; ++j) {
        if (pc[j] == 0xffffffffu) continue;
        const int hy = (pc[j] >> 16) & 0xf, hx = (pc[j] >> 20) & 0xf, c = pc[j] >> 24;
        const int y = y0 - 1 + hy, x = x0 - 1 + hx;
        if (!in_grid(zc, y, x)) continue;
        const int axis = (c * 8) / DA, p0 = ((c * 8) % DA) / 2;
        const int cv = axis == 0 ? zc : (axis == 1 ? y : x);
        const float4* cs4 = reinterpret_cast<const float4*>(
            P.ix.rope + 2 * rope_slot(P.ix.rope_rows, pairs, axis, cv, p0));
        const float4 ca = __ldg(cs4), cbv = __ldg(cs4 + 1);
        const float cs[8] = {ca.x, ca.y, ca.z, ca.w, cbv.x, cbv.y, cbv.z, cbv.w};
        uint4* ptr = reinterpret_cast<uint4*>(kd + ((pc[j] & 0xffffu) << 4));
        const uint4 xv = *ptr;
        const uint32_t xin[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t xo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float e0 = __uint_as_float(xin[k] << 16);
          const float e1 = __uint_as_float(xin[k] & 0xffff0000u);
          xo[k] = tc::pack_bf16(e0 * cs[2 * k] - e1 * cs[2 * k + 1],
                                e0 * cs[2 * k + 1] + e1 * cs[2 * k]);
        }
        *ptr = make_uint4(xo[0], xo[1], xo[2], xo[3]);
      }
      tc::fence_proxy_async_smem();  // the MMAs read the stage through the async proxy
      tc::mbar_arrive(&bars[B_KVFULL + st]);
    };
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
      const int64_t rbase = kv_of(bh, P.kv_group) * N;  // key and value rows of the KV head
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
      const __nv_bfloat16* kgb = kg + rbase * D;
      const __nv_bfloat16* vgb = vg + rbase * D;
      int prev_st = 0;
      for (int s = 0; s < kChunks; ++s, ++gs) {
        const int st = gs % kStages;
        if (gs >= (uint32_t)kStages && !pwait(&bars[B_KVEMPTY + st], ((gs / kStages) - 1) & 1)) {
          ok = false;
          break;
        }
        if (pt == 0) GTR(ti, 10 + s * 2);
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
        if constexpr (ROT) {
          tc::cp_async_commit();
          if (s > 0) {
            tc::cp_async_wait_group<1>();  // this thread's copies of slice s - 1 have landed
            rotate_slice(s - 1, prev_st, z0, y0, x0);
          }
          prev_st = st;
        } else {
          tc::cp_async_arrive_noinc(&bars[B_KVFULL + st]);
        }
        if (pt == 0) GTR(ti, 11 + s * 2);
      }
      if (!ok) break;
      if constexpr (ROT) {
        tc::cp_async_wait_group<0>();
        rotate_slice(kChunks - 1, prev_st, z0, y0, x0);
      }
      // this warp's reads of the slot box are done
      __syncwarp();
      if ((pt & 31) == 0) tc::mbar_arrive(&bars[B_BOXFREE + bb]);
    }
    tc::cp_async_wait_all();  // nothing may still be landing in shared memory at exit
  } else if (warp >= W_MMA) {
    // --------------------------------------------------------- MMA issuers (warps 14, 15)
    // One warp per tile. Per slice s: PV(s) for its owners (other rows disabled), then -- once
    // PV(s) has completed, which frees S buffer s % 2 -- QK(s + 2). The whole warp runs the
    // schedule with warp-uniform values; one elected lane issues the MMAs and commits.
    const int tile = warp - W_MMA;
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0) + tile * kTileCols;
    const uint32_t id_qk = tc::idesc_bf16_f32(128, kNK, false, false);
    const uint32_t id_pv = tc::idesc_bf16_f32(128, D, false, true);
    // no-swizzle descriptors: q and k K-major (lbo = column-chunk stride, sbo = 8 rows), v
    // MN-major (lbo = 8 key rows, sbo = column-chunk stride); the tile's window starts at
    // slice row 40 tile
    const uint64_t qd0 = tc::smem_desc(tc::smem_u32(smem + S::kQ), S::kQCol, 128);
    const uint64_t kd0 =
        tc::smem_desc(tc::smem_u32(smem + S::kK + (kWin * tile / 8) * 128), S::kChunkCol, 128);
    const uint64_t vd0 =
        tc::smem_desc(tc::smem_u32(smem + S::kV + (kWin * tile / 8) * 128), 128, S::kChunkCol);
    uint64_t* sfull = &bars[B_SFULL + tile * 8];
    uint64_t* pfull = &bars[B_PFULL + tile * 8];
    uint64_t* pvall = &bars[B_PVALL + tile];
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    int ti = 0;
    uint32_t gs = 0;
    bool ok = true;
    // QK(s) of chunk counter gc into S buffer s % 2 (q tile descriptor qd, q barrier qi); the S
    // buffer was freed by the PVALL wait of chunk gc - 2
    auto issue_qk = [&](int s, uint32_t gc, uint64_t qd, int qi) -> bool {
      const int st = gc % kStages;
      if (!wwait(&bars[B_KVFULL + st], (gc / kStages) & 1)) return false;
      // the chunk arrived through cp.async (generic proxy); the MMAs read it through the async
      // proxy
      tc::fence_proxy_async_smem();
      tc::tc_fence_after();
      const uint64_t b0 = kd0 + (uint64_t)((st * S::kStage) >> 4);
      const uint32_t dt = tb + s_col(s & 1);
      if (tc::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)  // 16 columns = two column chunks
          tc::mma_ss(dt, qd + (uint64_t)(ks * ((2 * S::kQCol) >> 4)),
                     b0 + (uint64_t)(ks * ((2 * S::kChunkCol) >> 4)), id_qk, ks > 0);
        for (int w = owner_lo(s); w <= owner_hi(s); ++w) tc::tc_commit(&sfull[2 * w + (s & 1)]);
        if (s == kChunks - 1) tc::tc_commit(&bars[B_QEMPTY + qi]);  // q tile free again
      }
      __syncwarp();
      return true;
    };
    for (; ok; ++ti) {
      if (!wwait(&bars[B_BOX + (ti & 1)], (ti >> 1) & 1) || unit_of(ti & 1) < 0) break;
      const int qi = tile;  // one q buffer per tile
      const uint64_t qd = qd0 + (uint64_t)((qi * S::kQBuf) >> 4);
      if (!wwait(&bars[B_QFULL + qi], ti & 1)) break;
      if (lane == 0 && tile == 0) GTR(ti, 50);
      if (lane == 0 && tile == 0) BRICK_T(ti);
      tc::tc_fence_after();
      ok = issue_qk(0, gs, qd, qi) && issue_qk(1, gs + 1, qd, qi);
      if (lane == 0 && tile == 0) GTR(ti, 51);
      for (int s = 0; s < kChunks && ok; ++s, ++gs) {
        const int st = gs % kStages, b = s & 1;
        const int wlo = owner_lo(s), whi = owner_hi(s);
        for (int w = wlo; w <= whi && ok; ++w) ok = wwait(&pfull[2 * w + b], sp_parity(w, s, ti));
        if (!ok) break;
        if (lane == 0 && tile == 0) GTR(ti, 60 + s * 4);
        tc::tc_fence_after();
        const uint32_t m0 = (0 < wlo || 0 > whi) ? 0xffffffffu : 0u;
        const uint32_t m1 = (1 < wlo || 1 > whi) ? 0xffffffffu : 0u;
        const uint32_t m2 = (2 < wlo || 2 > whi) ? 0xffffffffu : 0u;
        const uint32_t m3 = (3 < wlo || 3 > whi) ? 0xffffffffu : 0u;
        const uint64_t v0 = vd0 + (uint64_t)((st * S::kStage) >> 4);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kNK / 16; ++ks)  // 16 key rows = two row groups
            tc::mma_ts_masked(tb + kOCol, tb + s_col(b) + ks * 8, v0 + (uint64_t)(ks * (256 >> 4)),
                              id_pv, 1u, m0, m1, m2, m3);
          tc::tc_commit(&bars[B_KVEMPTY + st]);
          tc::tc_commit(pvall);
          if (s >= 2) tc::tc_commit(&bars[B_EPI + tile * 4 + (s - 2)]);  // warp s-2 done
        }
        __syncwarp();
        if (lane == 0 && tile == 0) GTR(ti, 61 + s * 4);
        // PV(s) complete: S buffer s % 2 may take QK(s + 2); observed for every chunk, in order
        if (!wwait(pvall, gs & 1)) { ok = false; break; }
        if (lane == 0 && tile == 0) GTR(ti, 62 + s * 4);
        if (s + 2 < kChunks) ok = issue_qk(s + 2, gs + 2, qd, qi);
        if (lane == 0 && tile == 0) GTR(ti, 63 + s * 4);
      }
    }
    // every MMA this warp issued has completed once this commit arrives (bounded wait)
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

template <int D, bool ROT>
cudaError_t launch_local_tma(const pack3d_index& ix, const void* q, const void* k, const void* v,
                             int64_t bh, int kv_group, float scale, void* o_loc, float* lse_loc,
                             cudaStream_t s) {
  using namespace lg;
  static std::atomic<uint64_t> attr_done{0};
  if (smem_attr_once(reinterpret_cast<const void*>(k_local_tma<D, ROT>), Smem<D>::kBytes,
                     attr_done) != cudaSuccess)
    return cudaErrorInvalidValue;
  Params p;
  p.ix = ix;
  p.o_loc = static_cast<__nv_bfloat16*>(o_loc);
  p.lse_loc = lse_loc;
  p.scale_log2 = scale * kLog2e;
  p.wait_budget = wait_budget_cycles();
  p.kv_group = kv_group;
  for (int a = 0; a < 3; ++a)
    for (int pp = 0; pp < 16; ++pp)
      p.theta[a][pp] = pp < ix.rope_pairs
                           ? (float)((double)ix.geom.spacing[a] *
                                     pow((double)ix.geom.rope_base, -2.0 * pp / (2.0 * ix.rope_pairs)))
                           : 0.f;
  p.nbz = (ix.geom.gz + BZ - 1) / BZ;
  p.nby = (ix.geom.gy + BY - 1) / BY;
  p.nbx = (ix.geom.gx + BX - 1) / BX;
  p.units = bh * p.nbz * p.nby * p.nbx;
  if (p.units <= 0) return cudaSuccess;
  if (!ix.status || p.units >= 0x7fffffffLL) return cudaErrorInvalidValue;  // unit counter
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  CUtensorMap mg;
  memset(&mg, 0, sizeof(mg));
  p.box_tma = encode_grid_i32(&mg, ix.inv, ix.geom.gz, ix.geom.gy, ix.geom.gx, kBoxX, kBoxY, kBoxZ)
                  ? 1
                  : 0;
  const int64_t cap = sm_count();
  const unsigned grid = (unsigned)(p.units < cap ? p.units : cap);
  k_local_tma<D, ROT><<<grid, kThreads, Smem<D>::kBytes, s>>>(mg, p);
  count_launch();
  return cudaGetLastError();
}

// k_rotated: k holds R(c) k (pack3d_summarize_rotated); otherwise the kernel rotates the keys.
cudaError_t local_tma_dispatch(const pack3d_index& ix, const void* q, const void* k,
                               const void* v, int64_t bh, int kv_group, float scale,
                               bool k_rotated, void* o_loc, float* lse_loc, cudaStream_t s) {
  if (ix.geom.head_dim == 96)
    return k_rotated
               ? launch_local_tma<96, false>(ix, q, k, v, bh, kv_group, scale, o_loc, lse_loc, s)
               : launch_local_tma<96, true>(ix, q, k, v, bh, kv_group, scale, o_loc, lse_loc, s);
  return k_rotated
             ? launch_local_tma<48, false>(ix, q, k, v, bh, kv_group, scale, o_loc, lse_loc, s)
             : launch_local_tma<48, true>(ix, q, k, v, bh, kv_group, scale, o_loc, lse_loc, s);
}

}  // namespace p3d

#ifdef P3D_TRACE_ENABLED
extern "C" int p3d_trace_read_t(unsigned long long* host) {
  cudaDeviceSynchronize();
  return (int)cudaMemcpyFromSymbol(host, p3d::g_trace, sizeof(unsigned long long) * 4096);
}
extern "C" int p3d_trace_read_b(unsigned long long* host) {
  cudaDeviceSynchronize();
  return (int)cudaMemcpyFromSymbol(host, p3d::lg::g_brick_t, sizeof(unsigned long long) * 512 * 32);
}
extern "C" int p3d_trace_clear_t() {
  static unsigned long long z[4096];
  return (int)cudaMemcpyToSymbol(p3d::g_trace, z, sizeof(z));
}
#endif
