// Global branch of PACK3D attention on tcgen05 tensor cores, with the sigmoid mixer fused into
// the epilogue (bf16 I/O, head_dim 48 or 96).
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 2: every query
// attends to all block summaries; paper summary §3.5: a streamed online softmax, no dense
// token x summary score matrix in memory; §3.3: o = g o_loc + (1 - g) o_glob, g = sigmoid(a).
//
// Work unit: 256 consecutive memory rows of one (batch, head) = two 128-row query tiles that
// share every summary chunk (halves the L2 reads of the summaries). Persistent CTAs walk the
// units round-robin. Warp roles (with PW = 4 query-producer warps, 480 threads; PW = 2 when a
// unit has 32 or more summary chunks, 416 threads, the later roles moving down by two):
//   warps 0-3   softmax + epilogue of tile 0 (thread = row, TMEM lanes 0..127); the epilogue
//               normalises O, writes lse, and parks o_glob in the tile's (by then consumed)
//               q area
//   warps 4-7   softmax + epilogue of tile 1
//   warps 8-11  query producer and mixer: before refilling a q buffer, apply the sigmoid mixer
//               to the unit staged there (coalesced o_loc / gate loads and o stores, overlapped
//               with the next unit's compute); then cp.async of q rows into the K-major
//               shared-memory A operand (double-buffered across units) and axial RoPE in place
//   warp 12     MMA issuer of tile 0 (whole warp, one elected lane issues) and TMEM owner
//   warp 13     MMA issuer of tile 1
//   warp 14     summary loader: each 64-summary chunk of ksum / vsum is one summary tile, i.e.
//               already in the operand layout, fetched by one contiguous bulk copy per tensor
//               into a 4-stage ring
// Per 64-summary chunk j and tile t:  S_t[j%2] = q~_t K_j^T (SS MMA, fp32 in TMEM) -> the
// softmax threads turn it into P = exp2(s - m) in bf16, written over S in TMEM ->
// O_t += P V_j (TS MMA). S is double-buffered per tile; each tile's issuer runs QK two chunks
// ahead of PV, so the next S of a tile is ready when its softmax finishes a chunk, and the two
// tiles' chains run independently on the shared tensor core. The running max uses a lazy
// rescale: O_t is corrected in TMEM only when a row's max grows by more than 2^8.
// The summary order is the same for every query (block ids ascending) and rows never interact,
// so a coordinate-carrying repack permutes the output bit for bit.
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace p3d {

namespace gtc {
constexpr int kRows = 128;        // rows per tile
constexpr int kTiles = 2;         // tiles per unit
constexpr int kChunk = 64;        // summaries per chunk
constexpr int kStages = 4;        // summary ring depth
// Warp roles for PW query-producer warps (4, or 2 when a unit has many summary chunks: the
// producers' per-unit work -- the mixer of one unit and the q tiles of the next -- is then
// spread over a long unit, and fewer producer warps leave the softmax warps more of the SM)
template <int PW> struct Roles {
  static constexpr int kProd = 32 * PW;  // query producer threads
  static constexpr int W_PROD = 8, W_MMA = W_PROD + PW, W_LOAD = W_MMA + kTiles;
  static constexpr int kThreads = 32 * (W_LOAD + 1);
};
constexpr int kManyChunks = 32;  // 2 producer warps from this many 64-summary chunks up
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kRopeSmemBytes = 24576;  // [3 axes][64 coordinates][16 pairs] (cos, sin)

// TMEM columns: tile t uses [256 t, 256 t + 256): S buffers at +0 and +64, O at +128.
__host__ __device__ constexpr uint32_t s_col(int t, int b) { return 256u * t + 64u * b; }
__host__ __device__ constexpr uint32_t o_col(int t) { return 256u * t + 128u; }

template <int D> struct Smem {
  static constexpr int kQTile = kRows * D * 2;       // one q tile
  static constexpr int kCTile = kChunk * D * 2;      // one summary chunk (ksum or vsum)
  static constexpr int kQ = 0;                       // [2 buffers][2 tiles]
  static constexpr int kK = kQ + 2 * kTiles * kQTile;
  static constexpr int kV = kK + kStages * kCTile;
  static constexpr int kCoord = kV + kStages * kCTile;  // 256 packed coordinates
  static constexpr int kGate = kCoord + kRows * kTiles * 4;  // [2 buffers][256] g = sigmoid(a)
  static constexpr int kRope = kGate + 2 * kRows * kTiles * 4;
  static constexpr int kBar = kRope + kRopeSmemBytes;
  static constexpr int kBytes = kBar + 256;
};

// barrier slots
enum {
  B_QFULL = 0,    // [2] q buffer filled
  B_QEMPTY = 2,   // [2] q buffer consumed
  B_KVFULL = 4,   // [kStages]
  B_KVEMPTY = 8,  // [kStages]
  B_SFULL = 12,   // [tile][buf] = 12 + 2 t + b
  B_PFULL = 16,   // [tile][buf]
  B_PVDONE = 20,  // [tile][buf]
  B_OFREE = 24,   // [tile]
  B_DONE = 26,    // [tile]
  B_COUNT = 28
};

struct Params {
  pack3d_index ix;
  const __nv_bfloat16* q;
  const __nv_bfloat16* ksum;   // summary tiles
  const __nv_bfloat16* vsum;
  const __nv_bfloat16* gate;
  const __nv_bfloat16* o_loc;  // may alias o
  __nv_bfloat16* o;
  __nv_bfloat16* o_glob;       // optional
  float* lse_glob;             // optional
  float scale_log2;            // tau * log2(e)
  int exclude_near;
  int64_t units;               // (batch*heads) * units_per_bh
  int units_per_bh;
  int n_chunks;
  int rope_in_smem;
  int kv_group;                // query heads per KV head (summaries are per KV head)
  int has_empty;               // some summary has no member (masked in every row)
  long long wait_budget;       // SM cycles of each bounded wait
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


}  // namespace gtc

template <int D, int PW>
__global__ void __launch_bounds__(gtc::Roles<PW>::kThreads, 1)
    k_global_tc(const gtc::Params P) {
  using namespace gtc;
  using S = Smem<D>;
  constexpr int kProd = Roles<PW>::kProd;
  constexpr int W_PROD = Roles<PW>::W_PROD, W_MMA = Roles<PW>::W_MMA, W_LOAD = Roles<PW>::W_LOAD;
  constexpr int KC = D / 8;  // 16-byte chunks per row
  constexpr int CB = kChunk * 16;  // byte stride between 16-byte columns of a summary chunk
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBar + 8 * B_COUNT + 8);
  volatile int* prod_ok = abort_flag + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) P3D_TRACE(999);
  tc::Abort ab{abort_flag, P.ix.status, P.wait_budget};

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_QFULL + i], kProd);
      tc::mbar_init(&bars[B_QEMPTY + i], kRows * kTiles);
      tc::mbar_init(&bars[B_OFREE + i], 128);
    }
    for (int i = 0; i < 4; ++i) {
      tc::mbar_init(&bars[B_SFULL + i], 1);
      tc::mbar_init(&bars[B_PFULL + i], 128);
      tc::mbar_init(&bars[B_PVDONE + i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars[B_KVFULL + i], 1);
      tc::mbar_init(&bars[B_KVEMPTY + i], kTiles);  // both tiles' PVs of the chunk
    }
    for (int i = 0; i < kTiles; ++i) tc::mbar_init(&bars[B_DONE + i], 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  // the rotation table in shared memory when it fits (read by the query producer)
  if (P.rope_in_smem) {
    const int n = 3 * P.ix.rope_rows * P.ix.rope_pairs * 2;
    float* dst = reinterpret_cast<float*>(smem + S::kRope);
    for (int i = tid; i < n; i += blockDim.x) dst[i] = P.ix.rope[i];
  }
  if (warp == W_MMA) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int64_t N = P.ix.n;
  const int M = (int)P.ix.m;
  const int NC = P.n_chunks;

  if (warp < 8) {
    // ------------------------------------------------------------------ softmax + epilogue
    const int t = warp >> 2;
    const int rin = (warp & 3) * 32 + lane;
    const uint32_t tl = tbase + ((uint32_t)((warp & 3) * 32) << 16);
    const int nby = P.ix.sum_grid[1], nbx = P.ix.sum_grid[2];
    int pc = 0;
    for (int64_t u = blockIdx.x; u < P.units; u += gridDim.x, ++pc) {
      const int64_t bh = u / P.units_per_bh;
      const int64_t row = (u % P.units_per_bh) * (kRows * kTiles) + t * kRows + rin;
      const bool valid = row < N;
      // summaries excluded for this row: those whose box meets the cube [c-1, c+1]^3, kept as
      // summary-grid ranges [z0,z1] x [y0,y1] x [x0,x1] (empty when exclusion is off)
      // the row's gate logit, loaded now and needed only by the epilogue
      const float glogit = valid ? __bfloat162float(P.gate[bh * N + row]) : 0.f;
      const ExclBox xb = excl_box(P.ix, valid ? decode(P.ix.coord[row]) : Coord{0, 0, 0},
                                  P.exclude_near && valid);
      const int z0 = xb.z0, z1 = xb.z1, y0 = xb.y0, y1 = xb.y1, x0 = xb.x0, x1 = xb.x1;
      float m_run = -INFINITY, l_run = 0.f;
      bool ok = true;
      for (int j = 0; j < NC; ++j) {
        const uint32_t gi = (uint32_t)(pc * NC + j);  // chunk counter of this tile
        const int b = gi & 1;
        if (!__all_sync(0xffffffffu, ab.wait(&bars[B_SFULL + 2 * t + b], (gi >> 1) & 1))) {
          ok = false;
          break;
        }
        if (rin == 0 && pc < 3) P3D_TRACE(1000 + pc * 128 + t * 64 + j * 2);
        if (rin == 0 && pc == 1 && j < 10) P3D_TRACE_C(3400 + j * 4 + t * 2);
        if (lane == 0 && pc == 1 && j < 16) P3D_TRACE(3730 + j * 8 + warp);
        tc::tc_fence_after();
        const int m0 = j * kChunk;
        const int ncol = min(kChunk, M - m0);
        // summaries with no member are out of every row's softmax
        uint32_t xm[2] = {0u, 0u};
        if (P.has_empty) {
          xm[0] = P.ix.empty[2 * j];
          xm[1] = (m0 + 32 < M) ? P.ix.empty[2 * j + 1] : 0u;
        }
        bool any_x = (xm[0] | xm[1]) != 0u;
        for (int mz = z0; mz <= z1; ++mz)
          for (int my = y0; my <= y1; ++my)
            for (int mx = x0; mx <= x1; ++mx) {
              const int cidx = (mz * nby + my) * nbx + mx - m0;
              if (cidx >= 0 && cidx < kChunk) {
                const uint32_t bit = 1u << (cidx & 31);
                xm[0] |= (cidx >> 5) == 0 ? bit : 0u;
                xm[1] |= (cidx >> 5) == 1 ? bit : 0u;
                any_x = true;
              }
            }
        const bool masked = any_x || ncol < kChunk;
        // the 64-column chunk in registers; masked entries become -inf in place
        uint32_t r[kChunk];
        const bool fine = rin == 0 && t == 0 && pc == 1 && j >= 2 && j < 6;  // fine trace points
        if (fine) P3D_TRACE(1800 + j * 8);
        tc::tmem_ld64(tl + s_col(t, b), r);
        tc::tmem_wait_ld();
        if (fine) P3D_TRACE(1800 + j * 8 + 1);
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        if (!masked) {
#pragma unroll
          for (int k = 0; k < kChunk; k += 2)
            mx[(k >> 1) & 3] =
                tc::max3f(mx[(k >> 1) & 3], __uint_as_float(r[k]), __uint_as_float(r[k + 1]));
        } else {
#pragma unroll
          for (int k = 0; k < kChunk; ++k) {
            if (((xm[k >> 5] >> (k & 31)) & 1u) || k >= ncol) r[k] = 0xff800000u;  // -inf
            mx[k & 3] = fmaxf(mx[k & 3], __uint_as_float(r[k]));
          }
        }
        // row max in the log2 domain (the scale is positive)
        const float cmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * P.scale_log2;
        const float m_new = fmaxf(m_run, cmax);
        if (fine) P3D_TRACE(1800 + j * 8 + 2);
        const bool need = m_new > m_run + kRescaleLog2;  // false while everything is masked
        if (__any_sync(0xffffffffu, need) && j > 0) {
          // O_t holds sum_{<j} P V with the old max: wait for the previous PV, then rescale
          const uint32_t gp = gi - 1;
          if (!__all_sync(0xffffffffu,
                          ab.wait(&bars[B_PVDONE + 2 * t + (gp & 1)], (gp >> 1) & 1))) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const float f = need ? ex2(m_run - m_new) : 1.f;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t o[16];
            tc::tmem_ld16(tl + o_col(t) + c0, o);
            tc::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
            tc::tmem_st16(tl + o_col(t) + c0, o);
          }
          tc::tmem_wait_st();
        }
        if (need) {
          l_run *= ex2(m_run - m_new);
          m_run = m_new;
        }
        const float neg_m = m_run == -INFINITY ? 0.f : -m_run;
        // P = exp2(s * scale - m) as bf16 over the first half of this S buffer; the scaling
        // and the row sum run two columns per instruction (packed fp32)
        float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
        const float2 sl2 = make_float2(P.scale_log2, P.scale_log2), nm2 = make_float2(neg_m, neg_m);
#pragma unroll
        for (int c0 = 0; c0 < kChunk; c0 += 32) {
          uint32_t p[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 x = tc::fma2(
                make_float2(__uint_as_float(r[c0 + k]), __uint_as_float(r[c0 + k + 1])), sl2, nm2);
            const float2 e = make_float2(ex2(x.x), ex2(x.y));
            ls[(k >> 1) & 3] = tc::add2(ls[(k >> 1) & 3], e);
            p[k >> 1] = tc::pack_bf16(e.x, e.y);
          }
          tc::tmem_st16(tl + s_col(t, b) + (c0 >> 1), p);
        }
        l_run += ((ls[0].x + ls[0].y) + (ls[1].x + ls[1].y)) + ((ls[2].x + ls[2].y) + (ls[3].x + ls[3].y));
        if (fine) P3D_TRACE(1800 + j * 8 + 3);
        tc::tmem_wait_st();
        if (fine) P3D_TRACE(1800 + j * 8 + 4);
        tc::tc_fence_before();
        tc::mbar_arrive(&bars[B_PFULL + 2 * t + b]);
        if (rin == 0 && pc < 3) P3D_TRACE(1000 + pc * 128 + t * 64 + j * 2 + 1);
        if (lane == 0 && pc == 1 && j < 16) P3D_TRACE(3600 + j * 8 + warp);
        if (rin == 0 && pc == 1 && j < 10) P3D_TRACE_C(3400 + j * 4 + t * 2 + 1);
      }
      if (!ok) break;
      // epilogue: o_glob = O / l and lse (the producer warps apply the mixer)
      const uint32_t gl = (uint32_t)(pc * NC + NC - 1);
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_PVDONE + 2 * t + (gl & 1)], (gl >> 1) & 1)))
        break;
      tc::tc_fence_after();
      // O row -> o_glob = O / l, kept packed as bf16 pairs; TMEM is released right after
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      uint32_t gp[(D + 31) / 32 * 16];
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tc::tmem_ld32(tl + o_col(t) + c0, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k)
          gp[c0 / 2 + k] = tc::pack_bf16(__uint_as_float(o[2 * k]) * inv_l,
                                         __uint_as_float(o[2 * k + 1]) * inv_l);
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&bars[B_OFREE + t]);
      if (rin == 0 && pc < 3) P3D_TRACE(1500 + pc * 4 + t * 2);
      // The unit's last QK has completed (its PV is done), so this tile's q area in shared
      // memory is free and holds exactly 128 rows of d bf16: each thread parks its o_glob row
      // there (16-byte chunk c of row r at chunk slot (c + r) mod KC, which spreads a warp's
      // stores over the banks). The producer warps apply the mixer from there, with coalesced
      // accesses, while these warps go on with the next unit.
      uint8_t* stage = smem + S::kQ + (pc & 1) * kTiles * S::kQTile + t * S::kQTile;
      tc::fence_proxy_async_smem();  // the tensor core's reads of this area came first
#pragma unroll
      for (int c = 0; c < KC; ++c)
        *reinterpret_cast<uint4*>(stage + rin * (D * 2) + ((c + rin) % KC) * 16) =
            make_uint4(gp[4 * c], gp[4 * c + 1], gp[4 * c + 2], gp[4 * c + 3]);
      if (valid && P.lse_glob)
        P.lse_glob[bh * N + row] = l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      // the mixer's weight g = sigmoid(a) of the row, once per row
      reinterpret_cast<float*>(smem + S::kGate)[(pc & 1) * kRows * kTiles + t * kRows + rin] =
          1.f / (1.f + __expf(-glogit));
      tc::mbar_arrive(&bars[B_QEMPTY + (pc & 1)]);  // o_glob of this unit is staged
    }
  } else if (warp < W_MMA) {
    // ------------------------------------------------------------------ query producer
    // cp.async the unit's 256 q rows straight into the operand layout (every copy in flight at
    // once), then rotate each 16-byte piece in place with the row's coordinate.
    const int ptid = tid - 32 * W_PROD;
    constexpr int DA = D / 3;
    int32_t* coord_s = reinterpret_cast<int32_t*>(smem + S::kCoord);
    const float* rope = P.rope_in_smem ? reinterpret_cast<const float*>(smem + S::kRope) : P.ix.rope;
    // Mixer of unit k (the k-th unit of this CTA), once the softmax warps have staged its
    // o_glob in q buffer k % 2 (and each row's g = sigmoid(a) beside it): o = g o_loc +
    // (1 - g) o_glob over the unit's 256 rows with consecutive threads on consecutive 16 bytes. o_loc may alias o (in-place
    // mixing): every piece a thread stores is one it loaded itself, and loads come first.
    auto mix = [&](int k) {
      const int64_t uk = blockIdx.x + (int64_t)k * gridDim.x;
      const int64_t bh = uk / P.units_per_bh;
      const int64_t row0 = (uk % P.units_per_bh) * (kRows * kTiles);
      const uint8_t* stage = smem + S::kQ + (k & 1) * kTiles * S::kQTile;
      const float* gsm = reinterpret_cast<const float*>(smem + S::kGate) + (k & 1) * kRows * kTiles;
      constexpr int G = D == 96 ? 12 : 6;  // pieces per thread in flight
      static_assert((kRows * kTiles * KC / kProd) % G == 0, "mixer groups");
#pragma unroll 1
      for (int g0 = 0; g0 < kRows * kTiles * KC / kProd; g0 += G) {
        uint4 lv[G];
#pragma unroll
        for (int i = 0; i < G; ++i) {
          const int pidx = (g0 + i) * kProd + ptid, r = pidx / KC, c = pidx % KC;
          const int64_t grow = row0 + r;
          lv[i] = make_uint4(0u, 0u, 0u, 0u);
          if (grow < N) lv[i] = reinterpret_cast<const uint4*>(P.o_loc + (bh * N + grow) * D)[c];
        }
#pragma unroll
        for (int i = 0; i < G; ++i) {
          const int pidx = (g0 + i) * kProd + ptid, r = pidx / KC, c = pidx % KC;
          const int64_t grow = row0 + r;
          if (grow >= N) continue;
          const int rin = r & (kRows - 1);
          const uint4 gv = *reinterpret_cast<const uint4*>(
              stage + (r >> 7) * S::kQTile + rin * (D * 2) + ((c + rin) % KC) * 16);
          const float g = gsm[r];  // sigmoid(a) of the row, left by the epilogue
          const uint32_t lw[4] = {lv[i].x, lv[i].y, lv[i].z, lv[i].w};
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
          uint32_t outw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float g0f = __uint_as_float(gw[e] << 16), g1f = __uint_as_float(gw[e] & 0xffff0000u);
            const float l0 = __uint_as_float(lw[e] << 16), l1 = __uint_as_float(lw[e] & 0xffff0000u);
            outw[e] = tc::pack_bf16(g * l0 + (1.f - g) * g0f, g * l1 + (1.f - g) * g1f);
          }
          const int64_t off = (bh * N + grow) * D;
          reinterpret_cast<uint4*>(P.o + off)[c] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
          if (P.o_glob) reinterpret_cast<uint4*>(P.o_glob + off)[c] = gv;
        }
      }
    };
    // one thread waits for unit k's staging; the named barrier hands its verdict to all
    auto wait_staged = [&](int k) -> bool {
      if (ptid == 0) *prod_ok = ab.wait(&bars[B_QEMPTY + (k & 1)], (k >> 1) & 1) ? 1 : 0;
      asm volatile("bar.sync 1, %0;" ::"n"(kProd) : "memory");
      return *prod_ok != 0;
    };
    int pc = 0;
    bool pok = true;
    for (int64_t u = blockIdx.x; u < P.units; u += gridDim.x, ++pc) {
      const int b = pc & 1;
      if (ptid == 0) {
        // this unit's o_loc rows (one contiguous run) and gates, read by its mixer two units
        // from now: start bringing them into L2
        const int64_t bhu = u / P.units_per_bh;
        const int64_t r0 = (u % P.units_per_bh) * (kRows * kTiles);
        const int64_t nr = min((int64_t)(kRows * kTiles), N - r0);
        tc::prefetch_l2(P.o_loc + (bhu * N + r0) * D, (uint32_t)(nr * D * 2));
        const __nv_bfloat16* gp0 = P.gate + bhu * N + r0;
        const uint32_t gbytes = (uint32_t)(nr * 2) & ~15u;
        if ((reinterpret_cast<uintptr_t>(gp0) & 15) == 0 && gbytes) tc::prefetch_l2(gp0, gbytes);
      }
      if (pc >= 2) {
        // q buffer b still holds unit pc-2's staged o_glob: mix it, then refill the buffer
        if (!wait_staged(pc - 2)) { pok = false; break; }
        mix(pc - 2);
        asm volatile("bar.sync 1, %0;" ::"n"(kProd) : "memory");
      }
      if (ptid == 0 && pc < 3) P3D_TRACE(2700 + pc * 4);
      const int64_t bh = u / P.units_per_bh;
      const int64_t row0 = (u % P.units_per_bh) * (kRows * kTiles);
      uint8_t* qb = smem + S::kQ + b * kTiles * S::kQTile;
      const __nv_bfloat16* qsrc = P.q + bh * N * D;
      for (int c = ptid; c < kRows * kTiles * KC; c += kProd) {
        int r, kc;
        tc::PieceOrder<KC>::at(c, r, kc);
        const int64_t row = row0 + r;
        const bool ok = row < N;
        tc::cp_async16(qb + (r >> 7) * S::kQTile + kc * 2048 + ((r & 127) >> 3) * 128 +
                           (r & 7) * 16,
                       qsrc + (ok ? row : 0) * D + kc * 8, ok);
      }
      tc::cp_async_commit();
      for (int r = ptid; r < kRows * kTiles; r += kProd)
        coord_s[r] = row0 + r < N ? P.ix.coord[row0 + r] : 0;
      asm volatile("bar.sync 1, %0;" ::"n"(kProd) : "memory");
      tc::cp_async_wait_all();
      if (ptid == 0 && pc < 3) P3D_TRACE(2700 + pc * 4 + 1);
#pragma unroll 4
      for (int c = ptid; c < kRows * kTiles * KC; c += kProd) {
        int r, kc;
        tc::PieceOrder<KC>::at(c, r, kc);
        uint4* ptr = reinterpret_cast<uint4*>(qb + (r >> 7) * S::kQTile + kc * 2048 +
                                              ((r & 127) >> 3) * 128 + (r & 7) * 16);
        const uint4 x = *ptr;
        const Coord cc = decode(coord_s[r]);
        const int axis = (kc * 8) / DA, p0 = ((kc * 8) % DA) / 2;
        const int cv = coord_axis(cc, axis);
        // (cos, sin) of the 4 pairs of this piece: 32 contiguous bytes of the table
        const float4* cs4 = reinterpret_cast<const float4*>(
            rope + 2 * rope_slot(P.ix.rope_rows, P.ix.rope_pairs, axis, cv, p0));
        const float4 ca = cs4[0], cb = cs4[1];
        const float cs[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
        const uint32_t xin[4] = {x.x, x.y, x.z, x.w};
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
      tc::fence_proxy_async_smem();
      asm volatile("bar.sync 1, %0;" ::"n"(kProd) : "memory");  // coord_s is rewritten next unit
      tc::mbar_arrive(&bars[B_QFULL + b]);
      if (ptid == 0 && pc < 3) P3D_TRACE(2700 + pc * 4 + 2);
    }
    // the last one or two units are still staged
    for (int k = pc >= 2 ? pc - 2 : 0; k < pc && pok; ++k) {
      if (!wait_staged(k)) break;
      mix(k);
    }
  } else if (warp < W_LOAD) {
    // ------------------------------------------------------------------ MMA issuers
    // One warp per query tile (warp 12: tile 0, warp 13: tile 1), so each tile's chain
    // softmax(j) -> PV(j) -> QK(j+2) advances on its own and neither waits behind the other's
    // MMAs or barrier probes. Per chunk j: PV_t(j) once the softmax has written P_t(j), then --
    // once PV_t(j) has completed, which frees the S buffer of chunk j -- QK_t(j+2), so S_t(j+1)
    // and S_t(j+2) are ready while the softmax works. The whole warp runs the schedule with
    // warp-uniform values (descriptors formed once and advanced by adding address offsets: the
    // start address is the low 14 bits and every offset keeps it in range); one elected lane
    // issues the MMAs and commits. A summary stage is released once both tiles' PVs of the
    // chunk have completed (KVEMPTY expects one commit from each issuer).
    const int t = warp - W_MMA;
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0);
    const uint32_t id_qk = tc::idesc_bf16_f32(128, kChunk, false, false);
    const uint32_t id_pv = tc::idesc_bf16_f32(128, D, false, true);
    const uint64_t kd0 = tc::smem_desc(tc::smem_u32(smem + S::kK), CB, 128);
    const uint64_t vd0 = tc::smem_desc(tc::smem_u32(smem + S::kV), 128, CB);
    // every lane probes; the verdict is the same on all lanes
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    int pc = 0;
    uint32_t kv_it = 0;
    bool issued = false, ok = true;
    for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++pc) {
      const int qb = pc & 1;
      if (!wwait(&bars[B_QFULL + qb], (pc >> 1) & 1)) break;
      if (lane == 0 && t == 0 && pc < 3) P3D_TRACE(2600 + pc);
      tc::tc_fence_after();
      const uint64_t a0 =
          tc::smem_desc(tc::smem_u32(smem + S::kQ + qb * kTiles * S::kQTile + t * S::kQTile),
                        2048, 128);
      // QK_t(j): S_t[buffer of j] = q~_t K_j^T
      auto issue_qk = [&](int j) -> bool {
        const uint32_t kv = kv_it + j;
        const uint32_t gi = (uint32_t)(pc * NC + j);
        const int b = gi & 1;
        const bool fq = lane == 0 && pc == 1 && j >= 4 && j < 8;
        [[maybe_unused]] const int fs = 3000 + j * 40 + t * 10;
        if (fq) P3D_TRACE_C(fs);
        if (!wwait(&bars[B_KVFULL + kv % kStages], (kv / kStages) & 1)) return false;
        if (fq) P3D_TRACE_C(fs + 1);
        // this S buffer held P of chunk gi - 2 until that PV completed
        if (gi >= 2 && !wwait(&bars[B_PVDONE + 2 * t + b], ((gi >> 1) - 1) & 1)) return false;
        if (fq) P3D_TRACE_C(fs + 2);
        tc::tc_fence_after();
        const uint64_t b0 = kd0 + (uint64_t)(((kv % kStages) * S::kCTile) >> 4);
        const uint32_t dt = tb + s_col(t, b);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks)
            tc::mma_ss(dt, a0 + (uint64_t)(ks * (4096 >> 4)),
                       b0 + (uint64_t)(ks * (2 * CB >> 4)), id_qk, ks > 0);
          tc::tc_commit(&bars[B_SFULL + 2 * t + b]);
        }
        __syncwarp();
        if (fq) P3D_TRACE_C(fs + 4);
        if (lane == 0 && pc < 3) P3D_TRACE(2000 + pc * 128 + t * 64 + j * 2);
        if (lane == 0 && pc < 3 && t == 0) P3D_TRACE(2500 + pc * 32 + j);
        if (lane == 0 && pc == 1 && j == 0 && t == 0) P3D_TRACE_CLK(3900);
        if (lane == 0 && pc == 8 && j == 0 && t == 0) P3D_TRACE_CLK(3902);
        issued = true;
        return true;
      };
      for (int j = 0; j < 2 && j < NC && ok; ++j) ok = issue_qk(j);
      for (int j = 0; j < NC && ok; ++j) {
        const uint32_t kv = kv_it + j;
        const uint32_t gi = (uint32_t)(pc * NC + j);
        const int b = gi & 1;
        const bool fp = lane == 0 && pc == 1 && j >= 2 && j < 6;
        [[maybe_unused]] const int fs = 3000 + (j + 2) * 40 + 20 + t * 10;
        if (fp) P3D_TRACE_C(fs);
        if (!wwait(&bars[B_PFULL + 2 * t + b], (gi >> 1) & 1)) { ok = false; break; }
        if (fp) P3D_TRACE_C(fs + 1);
        // the first PV of a unit overwrites O_t: the previous epilogue must have read it
        if (j == 0 && pc > 0 && !wwait(&bars[B_OFREE + t], (pc - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t v0 = vd0 + (uint64_t)(((kv % kStages) * S::kCTile) >> 4);
        const uint32_t at = tb + s_col(t, b), dt = tb + o_col(t);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kChunk / 16; ++ks)
            tc::mma_ts(dt, at + ks * 8, v0 + (uint64_t)(ks * (256 >> 4)), id_pv,
                       (j > 0 || ks > 0) ? 1u : 0u);
          tc::tc_commit(&bars[B_PVDONE + 2 * t + b]);
          tc::tc_commit(&bars[B_KVEMPTY + kv % kStages]);
        }
        __syncwarp();
        if (fp) P3D_TRACE_C(fs + 4);
        if (lane == 0 && pc < 3) P3D_TRACE(2000 + pc * 128 + t * 64 + j * 2 + 1);
        if (j + 2 < NC) ok = issue_qk(j + 2);
      }
      kv_it += NC;
    }
    // every MMA issued by this warp has completed before TMEM is released
    if (issued) {
      if (tc::elect_one()) tc::tc_commit(&bars[B_DONE + t]);
      __syncwarp();
      tc::mbar_wait(&bars[B_DONE + t], 0, 4000000000LL);
    }
  } else {
    // ------------------------------------------------------------------ summary loader
    if (lane == 0) {
      const int64_t MT = sum_tiles(M);
      uint32_t kv_it = 0;
      for (int64_t u = blockIdx.x; u < P.units && !*abort_flag; u += gridDim.x) {
        const int64_t bhk = kv_of(u / P.units_per_bh, P.kv_group);  // summaries of the KV head
        bool ok = true;
        for (int j = 0; j < NC; ++j, ++kv_it) {
          const int st = kv_it % kStages;
          if (kv_it >= (uint32_t)kStages &&
              !ab.wait(&bars[B_KVEMPTY + st], ((kv_it / kStages) - 1) & 1)) { ok = false; break; }
          tc::mbar_expect_tx(&bars[B_KVFULL + st], 2u * S::kCTile);
          const int64_t tile = (bhk * MT + j) * (int64_t)(kChunk * D);  // element offset
          tc::bulk_g2s(smem + S::kK + st * S::kCTile, P.ksum + tile, S::kCTile,
                       &bars[B_KVFULL + st]);
          tc::bulk_g2s(smem + S::kV + st * S::kCTile, P.vsum + tile, S::kCTile,
                       &bars[B_KVFULL + st]);
        }
        if (!ok) break;
      }
      // the last copies issued to each stage have landed before the CTA may exit
      for (uint32_t k = (kv_it > (uint32_t)kStages ? kv_it - kStages : 0); k < kv_it; ++k)
        tc::mbar_wait(&bars[B_KVFULL + (k % kStages)], (k / kStages) & 1, 4000000000LL);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host side

template <int D, int PW>
cudaError_t launch_global_tc(const pack3d_index& ix, const void* q, const void* gate,
                             const void* ksum, const void* vsum, const void* o_loc, int64_t bh,
                             int kv_group, float scale, int excl, void* o, float* lse_glob,
                             void* o_glob, cudaStream_t s) {
  using namespace gtc;
  static std::atomic<uint64_t> attr_done{0};
  if (smem_attr_once(reinterpret_cast<const void*>(k_global_tc<D, PW>), Smem<D>::kBytes, attr_done) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  Params p;
  p.ix = ix;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.ksum = static_cast<const __nv_bfloat16*>(ksum);
  p.vsum = static_cast<const __nv_bfloat16*>(vsum);
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.o_loc = static_cast<const __nv_bfloat16*>(o_loc);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_glob = static_cast<__nv_bfloat16*>(o_glob);
  p.lse_glob = lse_glob;
  p.scale_log2 = scale * kLog2e;
  p.exclude_near = excl;
  p.wait_budget = wait_budget_cycles();
  p.units_per_bh = (int)((ix.n + kRows * kTiles - 1) / (kRows * kTiles));
  p.units = bh * p.units_per_bh;
  p.n_chunks = (int)((ix.m + kChunk - 1) / kChunk);
  p.rope_in_smem = 3LL * ix.rope_rows * ix.rope_pairs * 8 <= kRopeSmemBytes ? 1 : 0;
  p.kv_group = kv_group;
  p.has_empty = ix.n_empty > 0 ? 1 : 0;
  const int grid = (int)(p.units < sm_count() ? p.units : sm_count());
  k_global_tc<D, PW><<<grid, Roles<PW>::kThreads, Smem<D>::kBytes, s>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t global_tc_dispatch(const pack3d_index& ix, const void* q, const void* gate,
                               const void* ksum, const void* vsum, const void* o_loc, int64_t bh,
                               int kv_group, float scale, int excl, void* o, float* lse_glob,
                               void* o_glob, cudaStream_t s) {
  const bool many = (ix.m + gtc::kChunk - 1) / gtc::kChunk >= gtc::kManyChunks;
#define P3D_GTC(D, PW)                                                                      \
  launch_global_tc<D, PW>(ix, q, gate, ksum, vsum, o_loc, bh, kv_group, scale, excl, o, \
                          lse_glob, o_glob, s)
  if (ix.geom.head_dim == 96) return many ? P3D_GTC(96, 2) : P3D_GTC(96, 4);
  return many ? P3D_GTC(48, 2) : P3D_GTC(48, 4);
#undef P3D_GTC
}

}  // namespace p3d

#ifdef P3D_TRACE_ENABLED
extern "C" int p3d_trace_read_g(unsigned long long* host) {
  cudaDeviceSynchronize();
  return (int)cudaMemcpyFromSymbol(host, p3d::g_trace, sizeof(unsigned long long) * 4096);
}
extern "C" int p3d_trace_clear_g() {
  static unsigned long long z[4096];
  return (int)cudaMemcpyToSymbol(p3d::g_trace, z, sizeof(z));
}
#endif
