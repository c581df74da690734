// Local branch of the PACK3D backward on tcgen05 tensor cores, key side: the gradients of k
// and v through the 3x3x3 softmax (bf16, head_dim 48 or 96), plus each key's share of its
// summary's gradient (un-pooling), then the inverse rotation -> dk, dv.
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 1 and "Rotate
// first, then pool"; paper summary §3.4. The 3x3x3 relation is symmetric, so key j's queries
// are its own coordinate neighbourhood and the gradients gather without scatter or atomics.
// For key j and query i (i in N(j)), with the forward's lse_loc, g_i = sigmoid(a_i) and
// Dl_i = g_i <dO_i, o_loc_i>:
//   P_ij = exp(<q~_i, k~_j> tau - lse_loc_i),  dS_ij = P_ij (g_i <dO_i, v_j> - Dl_i) tau,
//   dv_j = sum_i P_ij g_i dO_i,  dk~_j = sum_i dS_ij q~_i,
// then dv_j += w_j dV_t and dk_j = R(c_j)^T (dk~_j + w_j dK_t) (token RoPE) or
// R(c_j)^T dk~_j + w_j R(centre_t)^T dK_t (summary-centre RoPE), t the summary of j and w_j its
// weight in the summary's mean (1 / (members present in its block x non-empty blocks in the
// summary's group)).
//
// Work unit: one 4x4x8 (z, y, x) brick of keys of one (batch, head) = one 128-key tile; its
// queries stream in 6 halo z-slices of 6 x 10 = 60 (a 64-row window: rows 60..63 are zero).
// Key row r = 32 z + 8 y + x; warp w (the key z-plane w) needs query slices w .. w+2. Per slice s:
//   S^T = k~ q~_s^T and dP^T = v dO_s^T   (two SS MMAs, 128 x 64, fp32 in TMEM, double-buffered)
//   owners: P^T g and dS^T in bf16 over the first 32 columns of S^T and dP^T (per-column lse,
//   g, Dl staged with the slice);   dv += (P^T g) dO_s and dk~ += dS^T q~_s   (TS MMAs, N = d,
//   the other warps' rows disabled through the output-lane mask).
// TMEM: two S^T / dP^T buffers of 128 columns, dk~ and dv 96 columns each. Warps: elementwise
// 0-3 (warps 0 and 1 also stage the next unit's k~ and v tiles), slot boxes 4, q~ / dO
// producers 5-8, MMA 9. Units come from the index's device-wide counter (status word 2), put
// back to zero by the last CTA.
#include <math.h>

#include "bwd_work.h"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"
#include "tmap.h"

namespace p3d {

namespace lk {
constexpr int BZ = 4, BY = 4, BX = 8;  // one 128-key tile
constexpr int HY = BY + 2, HX = BX + 2;
constexpr int kChunks = BZ + 2;        // 6 halo z-slices
constexpr int kSliceKeys = HY * HX;    // 60 queries per slice
constexpr int kNK = 64;                // window (MMA N of the SS MMAs, K of the TS MMAs)
constexpr int kRows = kNK;             // rows per stage (60 .. 63 stay zero)
constexpr int kStages = 4;
constexpr int kThreads = 320;
constexpr int W_BOX = 4, W_PROD = 5, W_MMA = 9;
constexpr int kProd = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDkCol = 256, kDvCol = 352;
constexpr int kBoxX = 16, kBoxY = HY, kBoxZ = kChunks;  // slot box: x from x0 - 4
constexpr int kBoxBytes = kBoxX * kBoxY * kBoxZ * 4;
constexpr int kBoxPitch = 4096;

__device__ __forceinline__ uint32_t s_col(int b) { return 128u * b; }
__device__ __forceinline__ uint32_t p_col(int b) { return 128u * b + 64u; }
__host__ __device__ constexpr int slice_row(int hy, int hx) { return hy * HX + hx; }

template <int D> struct Smem {
  static constexpr int KC = D / 8;
  static constexpr int kQCol = 128 * 16 + 16;          // one 16-byte column of a key tile
  static constexpr int kQBuf = KC * kQCol;
  static constexpr int kChunkCol = kRows * 16 + 16;    // one 16-byte column of a query slice
  static constexpr int kStage = KC * kChunkCol;
  static constexpr int kA = 0;                           // [k~, v] key tiles
  static constexpr int kQ = kA + 2 * kQBuf;              // [kStages] q~ slices
  static constexpr int kG = kQ + kStages * kStage;       // [kStages] dO slices
  static constexpr int kCol = kG + kStages * kStage;     // [kStages][3][64] per-query values
  static constexpr int kBox = (kCol + kStages * 3 * 64 * 4 + 127) / 128 * 128;  // [2] boxes
  static constexpr int kBar = kBox + 2 * kBoxPitch;
  static constexpr int kBytes = kBar + 1024;
  static_assert(kBox % 128 == 0, "box alignment");
  static_assert(kBoxBytes + 8 <= kBoxPitch, "slot box and unit index");
  static_assert(kBytes <= 232448, "dynamic shared memory of one CTA");
  __device__ static int q_off(int r, int c) { return c * kQCol + (r >> 3) * 128 + (r & 7) * 16; }
};

enum {
  B_AFULL = 0, B_AEMPTY = 1,
  B_KVFULL = 2, B_KVEMPTY = 6, B_BOX = 10, B_BOXFREE = 12,
  B_SFULL = 14,  // [warp][buffer]
  B_PFULL = 22,  // [warp][buffer]
  B_TSALL = 30,
  B_EPI = 31,    // [warp]
  B_DRAIN = 35,
  B_COUNT = 36
};
static_assert(B_KVEMPTY - B_KVFULL >= kStages && B_BOX - B_KVEMPTY >= kStages, "ring barriers");
static_assert(8 * B_COUNT + 16 <= 1024, "barrier area");

struct Params {
  pack3d_index ix;
  const __nv_bfloat16* qr;    // rotated q [B, H, N, d]
  const __nv_bfloat16* kr;    // rotated k, one row per query head [B, H, N, d]
  const __nv_bfloat16* v;     // [B, H_kv, N, d]
  const __nv_bfloat16* dO;    // [B, H, N, d]
  const __nv_bfloat16* gate;  // [B, H, N]
  const float* lse_loc;       // [B, H, N]
  const float* Dl;            // [B, H, N]
  const float* dks;           // [nsplit][B, H, M, d] summary key gradients
  const float* dvs;
  int nsplit;
  __nv_bfloat16* dk;          // [B, H, N, d] (one query head per KV head)
  __nv_bfloat16* dv;
  float* dkp;                 // GQA: float32 per-query-head partials instead
  float* dvp;
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
__device__ __forceinline__ int owner_lo(int s) { return max(0, s - 2); }
__device__ __forceinline__ int owner_hi(int s) { return min(3, s); }
// Parity of warp w's wait on its S / P barrier of slice s (buffer s % 2) in unit ti: per unit
// the buffer of parity w % 2 serves slices w and w + 2 (two phases), the other slice w + 1.
__host__ __device__ __forceinline__ uint32_t sp_parity(int w, int s, int ti) {
  const int i = s - w;
  return (i & 1) ? (uint32_t)(ti & 1) : (uint32_t)((i >> 1) & 1);
}

}  // namespace lk

template <int D>
__global__ void __launch_bounds__(lk::kThreads, 1)
    k_bwd_local_dkv_tc(const __grid_constant__ CUtensorMap mg, const lk::Params P) {
  using namespace lk;
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
    tc::mbar_init(&bars[B_AFULL], 64);  // elementwise warps 0 and 1
    tc::mbar_init(&bars[B_AEMPTY], 1);
    for (int i = 0; i < kStages; ++i) {
      // every producer thread's copies landing (asynchronous arrivals), and the 64 threads
      // that store the slice's per-query values
      tc::mbar_init(&bars[B_KVFULL + i], kProd + 64);
      tc::mbar_init(&bars[B_KVEMPTY + i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_BOX + i], 1);
      tc::mbar_init(&bars[B_BOXFREE + i], 4 + 4);  // elementwise and producer warps
    }
    for (int i = 0; i < 8; ++i) {
      tc::mbar_init(&bars[B_SFULL + i], 1);
      tc::mbar_init(&bars[B_PFULL + i], 32);
    }
    tc::mbar_init(&bars[B_TSALL], 1);
    for (int i = 0; i < 4; ++i) tc::mbar_init(&bars[B_EPI + i], 1);
    tc::mbar_init(&bars[B_DRAIN], 1);
    abort_flag[0] = 0;
    tc::fence_mbar_init();
  }
  if (warp == W_BOX && lane == 0 && P.box_tma) tc::tma_prefetch_desc(&mg);
  // rows 60..63 of every q~ / dO stage are never written by the producers: zero them once
  for (int i = tid; i < kStages * 2 * KC * (kRows - kSliceKeys); i += kThreads) {
    const int row = kSliceKeys + i % (kRows - kSliceKeys), c = (i / (kRows - kSliceKeys)) % KC;
    const int blk = i / ((kRows - kSliceKeys) * KC);  // stage * 2 + tensor
    *reinterpret_cast<uint4*>(smem + ((blk & 1) ? S::kG : S::kQ) + (blk >> 1) * S::kStage +
                              c * S::kChunkCol + (row >> 3) * 128 + (row & 7) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  tc::fence_proxy_async_smem();
  if (warp == W_MMA) tc::tmem_alloc(tmem_slot, kTmemCols);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    // --------------------------------------------------------- elementwise + epilogue (row = lane)
    const int w = warp;
    // k~ and v tiles of unit `un` (slot box nb): warp w (0 or 1) takes key rows 64 w ..
    // 64 w + 63, one per lane and pass, each 16-byte piece a cp.async into the operand layout
    // (keys off the grid or at empty sites zero-filled); then it publishes its share
    auto prepare_a = [&](int64_t un, int nb) {
      int64_t kbh;
      int kz0, ky0, kx0;
      origin(un, kbh, kz0, ky0, kx0);
      const int32_t* kbox = reinterpret_cast<const int32_t*>(smem + S::kBox + nb * kBoxPitch);
      const int64_t vrow0 = kv_of(kbh, P.kv_group) * N;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int r = 64 * w + 32 * pass + lane;
        const int z = r >> 5, y = (r >> 3) & 3, x = r & 7;
        const int slot = in_grid(kz0 + z, ky0 + y, kx0 + x)
                             ? kbox[((z + 1) * kBoxY + y + 1) * kBoxX + x + 4]
                             : -1;
        const int sl = slot >= 0 ? slot : 0;
#pragma unroll
        for (int c = 0; c < KC; ++c) {
          tc::cp_async16(smem + S::kA + S::q_off(r, c), P.kr + (kbh * N + sl) * D + c * 8,
                         slot >= 0);
          tc::cp_async16(smem + S::kA + S::kQBuf + S::q_off(r, c), P.v + (vrow0 + sl) * D + c * 8,
                         slot >= 0);
        }
      }
      tc::cp_async_commit();
      tc::cp_async_wait_all();
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_AFULL]);
    };
    const int ky = (lane >> 3) & 3, kx = lane & 7;  // key position (w, ky, kx) in the brick
    const uint32_t tl = tbase + ((uint32_t)(w * 32) << 16);
    int ti = 0;
    bool ok = true;
    for (; ok; ++ti) {
      const int bb = ti & 1;
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_BOX + bb], (ti >> 1) & 1))) break;
      const int64_t u = unit_of(bb);
      if (u < 0) break;
      if (ti == 0 && w < 2) prepare_a(u, 0);
      int64_t bh;
      int z0, y0, x0;
      origin(u, bh, z0, y0, x0);
      const int32_t* box = reinterpret_cast<const int32_t*>(smem + S::kBox + bb * kBoxPitch);
      const int cz = z0 + w, cy = y0 + ky, cx = x0 + kx;
      const bool valid = cz < g.gz && cy < g.gy && cx < g.gx;
      const int slot = valid ? box[((w + 1) * kBoxY + ky + 1) * kBoxX + kx + 4] : -1;
      // query bits of the warp's three slices w + i: the slice's occupied sites (inside the
      // grid, not empty) as one ballot mask, a key's 3x3 queries the pattern 0b111 in three
      // halo rows shifted to its position
      uint64_t nb[3];
#pragma unroll
      for (int i = 0; i < 3; ++i) {
        const int hz = w + i;
        uint32_t half[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int c = hh * 32 + lane;
          bool occ = false;
          if (c < kSliceKeys) {
            const int hy = c / HX, hx = c % HX;
            occ = in_grid(z0 - 1 + hz, y0 - 1 + hy, x0 - 1 + hx) &&
                  box[(hz * kBoxY + hy) * kBoxX + hx + 3] >= 0;
          }
          half[hh] = __ballot_sync(0xffffffffu, occ);
        }
        const uint64_t occm = (uint64_t)half[0] | ((uint64_t)half[1] << 32);
        const uint64_t row3 = 7ull << kx;
        const uint64_t pat = (row3 | (row3 << HX) | (row3 << (2 * HX))) << (HX * ky);
        nb[i] = slot >= 0 ? (pat & occm) : 0ull;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars[B_BOXFREE + bb]);
      // this warp's dk~ and dv rows start at zero (the previous unit's epilogue has read them)
      {
        const uint32_t zr[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 16) {
          tc::tmem_st16(tl + kDkCol + c0, zr);
          tc::tmem_st16(tl + kDvCol + c0, zr);
        }
      }
      uint64_t* sfull = &bars[B_SFULL + w * 2];
      uint64_t* pfull = &bars[B_PFULL + w * 2];
#pragma unroll 1
      for (int i = 0; i < 3; ++i) {
        const int s = w + i, b = s & 1;
        const int st = (int)(((uint32_t)ti * kChunks + s) % kStages);
        if (!__all_sync(0xffffffffu, ab.wait(&sfull[b], sp_parity(w, s, ti)))) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const float* cv = reinterpret_cast<const float*>(smem + S::kCol) + st * 3 * 64;
        const uint64_t win = i == 0 ? nb[0] : (i == 1 ? nb[1] : nb[2]);  // (no indexed array)
        // two halves of 32 query columns: P^T g packed over S^T and dS^T over dP^T, columns
        // 16 h .. 16 h + 15 (columns the first half has already read)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[32], pv[32];
          tc::tmem_ld32(tl + s_col(b) + 32 * h, sv);
          tc::tmem_ld32(tl + p_col(b) + 32 * h, pv);
          tc::tmem_wait_ld();
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const float4 nl = *reinterpret_cast<const float4*>(cv + 32 * h + k);        // -lse log2e
            const float4 dl = *reinterpret_cast<const float4*>(cv + 64 + 32 * h + k);   // Dl
            const float4 gg = *reinterpret_cast<const float4*>(cv + 128 + 32 * h + k);  // g
            const float nla[4] = {nl.x, nl.y, nl.z, nl.w};
            const float dla[4] = {dl.x, dl.y, dl.z, dl.w};
            const float ga[4] = {gg.x, gg.y, gg.z, gg.w};
            float pg[4], ds[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = 32 * h + k + e;
              const float p = ((win >> col) & 1ull)
                                  ? ex2(fmaf(__uint_as_float(sv[k + e]), P.scale_log2, nla[e]))
                                  : 0.f;
              pg[e] = p * ga[e];
              ds[e] = p * (ga[e] * __uint_as_float(pv[k + e]) - dla[e]) * P.scale;
            }
            pk[k >> 1] = tc::pack_bf16(pg[0], pg[1]);
            pk[(k >> 1) + 1] = tc::pack_bf16(pg[2], pg[3]);
            dk[k >> 1] = tc::pack_bf16(ds[0], ds[1]);
            dk[(k >> 1) + 1] = tc::pack_bf16(ds[2], ds[3]);
          }
          tc::tmem_st16(tl + s_col(b) + 16 * h, pk);
          tc::tmem_st16(tl + p_col(b) + 16 * h, dk);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&pfull[b]);
      }
      if (!ok) break;
      // epilogue after the TS MMAs of the warp's last slice: + the summary's share, R^T, store
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_EPI + w], ti & 1))) break;
      tc::tc_fence_after();
      {
        const int64_t row = bh * N + (slot >= 0 ? slot : 0);
        const int t = slot >= 0 ? P.ix.sum_of[slot] : 0;
        const float wt =
            slot >= 0
                ? 1.f / ((float)P.ix.count[P.ix.block_of[slot]] * (float)P.ix.count2[t])
                : 0.f;
        const bool centre = g.summary_rope == PACK3D_ROPE_CENTRE;
        const int64_t part = (int64_t)(P.units / per_field) * P.ix.m * D;  // one split's size
        const float* sk0 = P.dks + (bh * P.ix.m + t) * D;
        const float* sv0 = P.dvs + (bh * P.ix.m + t) * D;
        const float2* rc = reinterpret_cast<const float2*>(P.ix.rope_c) + (int64_t)t * (D / 2);
        // (once per unit: kept rolled, the kernel's code is large)
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 16) {
          uint32_t ok16[16], ov16[16];
          tc::tmem_ld16(tl + kDkCol + c0, ok16);
          tc::tmem_ld16(tl + kDvCol + c0, ov16);
          tc::tmem_wait_ld();
          if (slot >= 0) {  // (the loads above are warp-wide; the rest per lane)
            float ak[16], av[16], sk[16], svv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              ak[k] = __uint_as_float(ok16[k]);
              av[k] = __uint_as_float(ov16[k]);
              sk[k] = svv[k] = 0.f;
            }
            for (int sp = 0; sp < P.nsplit; ++sp) {
#pragma unroll
              for (int k = 0; k < 16; k += 4) {
                const float4 a4 = *reinterpret_cast<const float4*>(sk0 + sp * part + c0 + k);
                const float4 b4 = *reinterpret_cast<const float4*>(sv0 + sp * part + c0 + k);
                sk[k] += a4.x; sk[k + 1] += a4.y; sk[k + 2] += a4.z; sk[k + 3] += a4.w;
                svv[k] += b4.x; svv[k + 1] += b4.y; svv[k + 2] += b4.z; svv[k + 3] += b4.w;
              }
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) av[k] = fmaf(svv[k], wt, av[k]);
            if (!centre) {
#pragma unroll
              for (int k = 0; k < 16; ++k) ak[k] = fmaf(sk[k], wt, ak[k]);
            }
            // R(c_j)^T of the local (and, with token RoPE, the summary's) key gradient
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
              const int c = c0 / 8 + hc;
              const int axis = (c * 8) / DA, p0 = ((c * 8) % DA) / 2;
              const int cvv = axis == 0 ? cz : (axis == 1 ? cy : cx);
              const float4* cs4 = reinterpret_cast<const float4*>(
                  P.ix.rope + 2 * rope_slot(P.ix.rope_rows, P.ix.rope_pairs, axis, cvv, p0));
              const float4 ca = __ldg(cs4), cbv = __ldg(cs4 + 1);
              const float cs[8] = {ca.x, ca.y, ca.z, ca.w, cbv.x, cbv.y, cbv.z, cbv.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int e = 8 * hc + 2 * k;
                const float x0 = ak[e], x1 = ak[e + 1];
                ak[e] = x0 * cs[2 * k] + x1 * cs[2 * k + 1];
                ak[e + 1] = x1 * cs[2 * k] - x0 * cs[2 * k + 1];
              }
            }
            if (centre) {
              // + w R(centre_t)^T dK_t, pair e / 2 of dims (e, e + 1)
#pragma unroll
              for (int k = 0; k < 16; k += 2) {
                const float2 cs = rc[(c0 + k) / 2];
                const float x0 = sk[k], x1 = sk[k + 1];
                ak[k] = fmaf(x0 * cs.x + x1 * cs.y, wt, ak[k]);
                ak[k + 1] = fmaf(x1 * cs.x - x0 * cs.y, wt, ak[k + 1]);
              }
            }
            if (P.dkp) {
              float4* dkp = reinterpret_cast<float4*>(P.dkp + row * D + c0);
              float4* dvp = reinterpret_cast<float4*>(P.dvp + row * D + c0);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                dkp[k] = make_float4(ak[4 * k], ak[4 * k + 1], ak[4 * k + 2], ak[4 * k + 3]);
                dvp[k] = make_float4(av[4 * k], av[4 * k + 1], av[4 * k + 2], av[4 * k + 3]);
              }
            } else {
              uint32_t kw[8], vw[8];
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                kw[k] = tc::pack_bf16(ak[2 * k], ak[2 * k + 1]);
                vw[k] = tc::pack_bf16(av[2 * k], av[2 * k + 1]);
              }
              uint4* dkd = reinterpret_cast<uint4*>(P.dk + row * D + c0);
              uint4* dvd = reinterpret_cast<uint4*>(P.dv + row * D + c0);
              dkd[0] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
              dkd[1] = make_uint4(kw[4], kw[5], kw[6], kw[7]);
              dvd[0] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
              dvd[1] = make_uint4(vw[4], vw[5], vw[6], vw[7]);
            }
          }
          __syncwarp();
        }
      }
      if (w < 2) {
        // the next unit's k~ / v tiles, once its slot box is in and this unit's last SS MMAs
        // have completed
        const int nbx = (ti + 1) & 1;
        if (!__all_sync(0xffffffffu, ab.wait(&bars[B_BOX + nbx], ((ti + 1) >> 1) & 1))) break;
        const int64_t un = unit_of(nbx);
        if (un >= 0) {
          if (!__all_sync(0xffffffffu, ab.wait(&bars[B_AEMPTY], ti & 1))) break;
          prepare_a(un, nbx);
        }
      }
    }
    tc::cp_async_wait_all();
  } else if (warp == W_BOX) {
    // --------------------------------------------------------- slot boxes (warp 4)
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
    // --------------------------------------------------------- q~ / dO rows (128 threads)
    // Halo slice s of queries: 60 rows of q~ and of dO, one cp.async per 16-byte piece (rows
    // off the grid or at empty sites zero-filled), each thread's copies arriving on the
    // stage's barrier by themselves; threads 0..63 also store the window columns' -lse log2e,
    // Dl and g (zero for rows without a token) and arrive for them.
    const int pt = tid - W_PROD * 32;
    volatile int* pflag = abort_flag + 1;  // [2], used alternately
    int nwait = 0;
    auto pwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      volatile int* f = pflag + (nwait++ & 1);
      if (pt == 0) *f = ab.wait(bar, parity) ? 1 : 0;
      asm volatile("bar.sync 2, 128;" ::: "memory");
      return *f != 0;
    };
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
      const int64_t qbase = bh * N;
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
      const __nv_bfloat16* qgb = P.qr + qbase * D;
      const __nv_bfloat16* ggb = P.dO + qbase * D;
      for (int s = 0; s < kChunks; ++s, ++gs) {
        const int st = gs % kStages;
        if (gs >= (uint32_t)kStages && !pwait(&bars[B_KVEMPTY + st], ((gs / kStages) - 1) & 1)) {
          ok = false;
          break;
        }
        uint8_t* qd = smem + S::kQ + st * S::kStage;
        uint8_t* gd = smem + S::kG + st * S::kStage;
        const bool zin = z0 - 1 + s >= 0 && z0 - 1 + s < g.gz;
        const int32_t* sbox = box + s * kBoxY * kBoxX;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
          if (pc[j] == 0xffffffffu) continue;
          const int slot = (zin && bidx[j] >= 0) ? sbox[bidx[j]] : -1;
          const int64_t src = (int64_t)(slot >= 0 ? slot : 0) * D + (int)(pc[j] >> 24) * 8;
          const uint32_t off = (pc[j] & 0xffffu) << 4;
          tc::cp_async16(qd + off, qgb + src, slot >= 0);
          tc::cp_async16(gd + off, ggb + src, slot >= 0);
        }
        tc::cp_async_arrive_noinc(&bars[B_KVFULL + st]);
        if (pt < kNK) {
          // window column pt = slice row pt (halo y-major)
          float nl = 0.f, dl = 0.f, gg = 0.f;
          if (pt < kSliceKeys) {
            const int hy = pt / HX, hx = pt % HX;
            const int y = y0 - 1 + hy, x = x0 - 1 + hx;
            if (zin && y >= 0 && y < g.gy && x >= 0 && x < g.gx) {
              const int slot = box[(s * kBoxY + hy) * kBoxX + hx + 3];
              if (slot >= 0) {
                const int64_t r = qbase + slot;
                nl = -P.lse_loc[r] * kLog2e;
                dl = P.Dl[r];
                gg = 1.f / (1.f + __expf(-__bfloat162float(P.gate[r])));
              }
            }
          }
          float* cv = reinterpret_cast<float*>(smem + S::kCol) + st * 3 * 64;
          cv[pt] = nl;
          cv[64 + pt] = dl;
          cv[128 + pt] = gg;
          tc::mbar_arrive(&bars[B_KVFULL + st]);
        }
      }
      if (!ok) break;
      __syncwarp();
      if ((pt & 31) == 0) tc::mbar_arrive(&bars[B_BOXFREE + bb]);
    }
    tc::cp_async_wait_all();
  } else {
    // --------------------------------------------------------- MMA issuer (warp 9)
    // Per slice s: TS(s) once the owners have written P^T g and dS^T; then -- once TS(s) has
    // completed, which frees buffer s % 2 -- SS(s + 2). The whole warp runs the schedule with
    // warp-uniform values; one elected lane issues the MMAs and commits.
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0);
    const uint32_t id_ss = tc::idesc_bf16_f32(128, kNK, false, false);
    const uint32_t id_ts = tc::idesc_bf16_f32(128, D, false, true);
    // no-swizzle descriptors: key tiles and query slices as K-major operands (lbo = column
    // stride, sbo = 8 rows); query slices as the MN-major B of the TS MMAs (lbo = 8 rows, sbo =
    // column stride)
    const uint64_t kad = tc::smem_desc(tc::smem_u32(smem + S::kA), S::kQCol, 128);
    const uint64_t vad = tc::smem_desc(tc::smem_u32(smem + S::kA + S::kQBuf), S::kQCol, 128);
    const uint64_t qk0 = tc::smem_desc(tc::smem_u32(smem + S::kQ), S::kChunkCol, 128);
    const uint64_t gk0 = tc::smem_desc(tc::smem_u32(smem + S::kG), S::kChunkCol, 128);
    const uint64_t qm0 = tc::smem_desc(tc::smem_u32(smem + S::kQ), 128, S::kChunkCol);
    const uint64_t gm0 = tc::smem_desc(tc::smem_u32(smem + S::kG), 128, S::kChunkCol);
    uint64_t* sfull = &bars[B_SFULL];
    uint64_t* pfull = &bars[B_PFULL];
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    // SS(s) of slice counter gc into buffer s % 2 (freed by the TSALL wait of gc - 2)
    auto issue_ss = [&](int s, uint32_t gc) -> bool {
      const int st = gc % kStages;
      if (!wwait(&bars[B_KVFULL + st], (gc / kStages) & 1)) return false;
      tc::fence_proxy_async_smem();  // the slice arrived through cp.async
      tc::tc_fence_after();
      const uint64_t so = (uint64_t)((st * S::kStage) >> 4);
      const int b = s & 1;
      if (tc::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          tc::mma_ss(tb + s_col(b), kad + (uint64_t)(ks * ((2 * S::kQCol) >> 4)),
                     qk0 + so + (uint64_t)(ks * ((2 * S::kChunkCol) >> 4)), id_ss, ks > 0);
          tc::mma_ss(tb + p_col(b), vad + (uint64_t)(ks * ((2 * S::kQCol) >> 4)),
                     gk0 + so + (uint64_t)(ks * ((2 * S::kChunkCol) >> 4)), id_ss, ks > 0);
        }
        for (int w = owner_lo(s); w <= owner_hi(s); ++w) tc::tc_commit(&sfull[2 * w + b]);
        if (s == kChunks - 1) tc::tc_commit(&bars[B_AEMPTY]);  // key tiles free again
      }
      __syncwarp();
      return true;
    };
    int ti = 0;
    uint32_t gs = 0;
    bool ok = true;
    for (; ok; ++ti) {
      if (!wwait(&bars[B_BOX + (ti & 1)], (ti >> 1) & 1) || unit_of(ti & 1) < 0) break;
      if (!wwait(&bars[B_AFULL], ti & 1)) break;
      tc::tc_fence_after();
      ok = issue_ss(0, gs) && issue_ss(1, gs + 1);
      for (int s = 0; s < kChunks && ok; ++s, ++gs) {
        const int st = gs % kStages, b = s & 1;
        const int wlo = owner_lo(s), whi = owner_hi(s);
        for (int w = wlo; w <= whi && ok; ++w) ok = wwait(&pfull[2 * w + b], sp_parity(w, s, ti));
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t m0 = (0 < wlo || 0 > whi) ? 0xffffffffu : 0u;
        const uint32_t m1 = (1 < wlo || 1 > whi) ? 0xffffffffu : 0u;
        const uint32_t m2 = (2 < wlo || 2 > whi) ? 0xffffffffu : 0u;
        const uint32_t m3 = (3 < wlo || 3 > whi) ? 0xffffffffu : 0u;
        const uint64_t so = (uint64_t)((st * S::kStage) >> 4);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < kNK / 16; ++ks) {  // 16 query rows = two row groups
            // dv += (P^T g) dO_s;  dk~ += dS^T q~_s
            tc::mma_ts_masked(tb + kDvCol, tb + s_col(b) + ks * 8,
                              gm0 + so + (uint64_t)(ks * (256 >> 4)), id_ts, 1u, m0, m1, m2, m3);
            tc::mma_ts_masked(tb + kDkCol, tb + p_col(b) + ks * 8,
                              qm0 + so + (uint64_t)(ks * (256 >> 4)), id_ts, 1u, m0, m1, m2, m3);
          }
          tc::tc_commit(&bars[B_KVEMPTY + st]);
          tc::tc_commit(&bars[B_TSALL]);
          if (s >= 2) tc::tc_commit(&bars[B_EPI + (s - 2)]);  // warp s-2 done
        }
        __syncwarp();
        // TS(s) complete: buffer s % 2 may take SS(s + 2); observed for every slice, in order
        if (!wwait(&bars[B_TSALL], gs & 1)) { ok = false; break; }
        if (s + 2 < kChunks) ok = issue_ss(s + 2, gs + 2);
      }
    }
    if (tc::elect_one()) tc::tc_commit(&bars[B_DRAIN]);
    __syncwarp();
    if (!tc::mbar_wait(&bars[B_DRAIN], 0, 100000000LL))
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
cudaError_t launch_bwd_local_dkv_tc(const pack3d_index& ix, const BwdWork& w, const void* v,
                                    const void* dO, const void* gate, const float* lse_loc,
                                    int64_t bh, int kv_group, float scale, void* dk, void* dv,
                                    cudaStream_t s) {
  using namespace lk;
  static std::atomic<uint64_t> attr_done{0};
  if (smem_attr_once(reinterpret_cast<const void*>(k_bwd_local_dkv_tc<D>), Smem<D>::kBytes,
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
  p.dks = w.dks;
  p.dvs = w.dvs;
  p.nsplit = w.nsplit;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.dkp = w.dkp;
  p.dvp = w.dvp;
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
  k_bwd_local_dkv_tc<D><<<grid, kThreads, Smem<D>::kBytes, s>>>(mg, p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t bwd_local_dkv_tc_dispatch(const pack3d_index& ix, const BwdWork& w, const void* v,
                                      const void* dO, const void* gate, const float* lse_loc,
                                      int64_t bh, int kv_group, float scale, void* dk, void* dv,
                                      cudaStream_t s) {
  if (ix.geom.head_dim == 96)
    return launch_bwd_local_dkv_tc<96>(ix, w, v, dO, gate, lse_loc, bh, kv_group, scale, dk, dv,
                                       s);
  return launch_bwd_local_dkv_tc<48>(ix, w, v, dO, gate, lse_loc, bh, kv_group, scale, dk, dv, s);
}

}  // namespace p3d
