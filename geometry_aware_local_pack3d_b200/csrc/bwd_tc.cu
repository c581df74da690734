// Global branch of the PACK3D backward on tcgen05 tensor cores (bf16, head_dim 48 or 96).
//
// Paper summary §3.4 (the backward follows the forward's streamed access pattern); project
// page Chapter 3 Contract 2 and "Rotate first, then pool". With dO_g = (1 - g) dO and the
// forward's lse_glob, for query i and summary m:
//   P_im = exp(<q~_i, K_m> tau - lse_i),  dP_im = <dO_g,i, V_m>,
//   dS_im = P_im (dP_im - D_i) tau,       D_i = <dO_g,i, o_glob,i>,
//   dq~_i += sum_m dS_im K_m,   dK_m += sum_i dS_im q~_i,   dV_m += sum_i P_im dO_g,i.
// (Summaries excluded for query i by exclude_near have P_im = 0.) The row-wise prologue
// (rotated q and dO_g in bf16, D_i) and the local branch, the un-pooling and the inverse
// rotation stay in the CUDA-core kernels of attn_simt.cu.
//
// k_bwd_dq_tc   query-major, like the forward: a CTA walks 128-query tiles; per 64-summary
//               chunk S = q~ K^T and dP = dO_g V^T (SS MMAs into TMEM), the elementwise warps
//               form dS in bf16 over S, and dq~ += dS K (TS MMA, K read as the MN-major
//               operand). Output: the global part of dq~ in fp32.
// k_bwd_dsum_tc summary-major: a CTA owns 128 summaries of one (batch, head) and one query
//               range; per 64-query tile S^T = K q~^T and dP^T = V dO_g^T (double-buffered in
//               TMEM, issued two tiles ahead), then P^T and dS^T in bf16 over them,
//               dV += P^T dO_g and dK += dS^T q~ (TS MMAs, q~ and dO_g read as MN-major
//               operands). Output: per-range partial dK, dV in fp32.
// Operands use the no-swizzle core-matrix layout; the summary tiles are already in it.
#include <math.h>

#include <type_traits>

#include "bwd_work.h"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace p3d {

namespace btc {
constexpr int kRows = 128;   // queries (dq) or summaries (dsum) per tile: MMA M
constexpr int kChunk = 64;   // summaries per chunk (dq) or queries per tile (dsum): MMA N

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (a.x b.x, a.y b.y) in one instruction, round to nearest
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Asynchronous 4-byte global -> shared copy (through L1); zero-filled when `valid` is false.
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(tc::smem_u32(smem_dst)),
               "l"(gsrc), "r"(valid ? 4 : 0)
               : "memory");
}


struct Params {
  pack3d_index ix;
  const __nv_bfloat16* qtb;   // rotated q, [BH, N, d]
  const __nv_bfloat16* dogb;  // (1 - g) dO, [BH, N, d]
  const __nv_bfloat16* ksum;  // summary tiles
  const __nv_bfloat16* vsum;
  const float* lse;           // lse_glob [BH, N]
  const float* Dg;            // [BH, N]
  float* out0;                // dq: dqg [BH, N, d];  dsum: dks partials
  float* out1;                // dsum: dvs partials
  float scale, scale_log2;
  int exclude_near;
  int64_t bh_count;
  int64_t units, units_per_bh;  // dq: 128-query tiles
  int n_chunks;                 // dq: 64-summary chunks per (batch, head)
  int m_tiles, q_tiles, q_per_split;  // dsum: 128-summary tiles, 64-query tiles
  int nsplit;                         // dsum: query ranges per (batch, head)
  int kv_group;                       // query heads per KV head (summaries per KV head)
  long long wait_budget;              // SM cycles of each bounded wait
};
}  // namespace btc

// ============================================================================= dq~ (global)
namespace bdq {
template <int D> struct Smem {
  static constexpr int kTile = btc::kRows * D * 2;   // one 128-row operand tile
  static constexpr int kCTile = btc::kChunk * D * 2;  // one summary chunk (K or V)
  static constexpr int kStages = 2;
  static constexpr int kQ = 0;                  // q~ tile
  static constexpr int kG = kQ + kTile;         // dO_g tile
  static constexpr int kK = kG + kTile;         // [stages]
  static constexpr int kV = kK + kStages * kCTile;
  static constexpr int kBar = kV + kStages * kCTile;
  static constexpr int kBytes = kBar + 256;
};
enum {
  B_QFULL = 0, B_QEMPTY = 1, B_KVFULL = 2, B_KVEMPTY = 4, B_SFULL = 6, B_PFULL = 7, B_DONE = 8,
  B_OFREE = 9, B_DRAIN = 10, B_COUNT = 11
};
constexpr int kThreads = 256;  // elementwise 0-3, producer 4-5, summary loader 6, MMA 7
constexpr int kProd = 64;
constexpr uint32_t kS = 0, kP = 64, kO = 128;  // TMEM columns: S, dP, dq~
}  // namespace bdq

template <int D>
__global__ void __launch_bounds__(bdq::kThreads, 2) k_bwd_dq_tc(const btc::Params P) {
  using namespace bdq;
  using S = Smem<D>;
  constexpr int KC = D / 8;
  constexpr int CB = btc::kChunk * 16;  // byte stride between 16-byte columns of a chunk
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBar + 8 * B_COUNT + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tc::Abort ab{abort_flag, P.ix.status, P.wait_budget};
  const int64_t N = P.ix.n;
  const int M = (int)P.ix.m;
  const int NC = P.n_chunks;
  if (tid == 0) {
    tc::mbar_init(&bars[B_QFULL], kProd);
    tc::mbar_init(&bars[B_QEMPTY], 1);
    for (int i = 0; i < S::kStages; ++i) {
      tc::mbar_init(&bars[B_KVFULL + i], 1);
      tc::mbar_init(&bars[B_KVEMPTY + i], 1);
    }
    tc::mbar_init(&bars[B_SFULL], 1);
    tc::mbar_init(&bars[B_PFULL], 128);
    tc::mbar_init(&bars[B_DONE], 1);
    tc::mbar_init(&bars[B_OFREE], 128);
    tc::mbar_init(&bars[B_DRAIN], 1);
    abort_flag[0] = 0;
    tc::fence_mbar_init();
  }
  if (warp == 7) tc::tmem_alloc(tmem_slot, 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ elementwise + epilogue
    const int nby = P.ix.sum_grid[1], nbx = P.ix.sum_grid[2];
    uint32_t gc = 0;
    int pc = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++pc) {
      int ln = lane;
      uint32_t tl = tbase;
      asm volatile("" : "+r"(ln), "+r"(tl));
      const int rin = warp * 32 + ln;
      tl += (uint32_t)(warp * 32) << 16;
      const int64_t bh = u / P.units_per_bh;
      const int64_t row = (u % P.units_per_bh) * btc::kRows + rin;
      const bool valid = row < N;
      const int64_t grow = bh * N + row;
      const float lse = valid ? P.lse[grow] : -INFINITY;
      const float Dg = valid ? P.Dg[grow] : 0.f;
      const bool live = lse != -INFINITY;  // every summary excluded: no global gradient
      const float nl = live ? -lse * kLog2e : 0.f;
      const float Ds = Dg * P.scale;
      const ExclBox ex = excl_box(P.ix, decode(valid ? P.ix.coord[row] : 0),
                                  P.exclude_near != 0 && valid);
      for (int j = 0; j < NC; ++j, ++gc) {
        if (!__all_sync(0xffffffffu, ab.wait(&bars[B_SFULL], gc & 1))) { ok = false; break; }
        tc::tc_fence_after();
        const int m0 = j * btc::kChunk;
        // exclusion bits of this chunk (block ids are summary ids)
        uint32_t xm[2] = {0u, 0u};
        for (int mz = ex.z0; mz <= ex.z1; ++mz)
          for (int my = ex.y0; my <= ex.y1; ++my)
            for (int mx = ex.x0; mx <= ex.x1; ++mx) {
              const int cidx = (mz * nby + my) * nbx + mx - m0;
              if (cidx >= 0 && cidx < btc::kChunk) {
                xm[0] |= (cidx >> 5) == 0 ? (1u << (cidx & 31)) : 0u;
                xm[1] |= (cidx >> 5) == 1 ? (1u << (cidx & 31)) : 0u;
              }
            }
        // two halves of 32 columns: read S and dP, write dS (bf16) over S columns already read.
        // Two columns per step with packed fp32: P = 2^(S tau log2(e) - lse log2(e)),
        // dS = P (dP tau - D tau); the columns whose P is zero (no global gradient for the
        // row, past the last summary, or excluded) are one bit mask per half.
        const float2 sl2 = make_float2(P.scale_log2, P.scale_log2);
        const float2 sc2 = make_float2(P.scale, P.scale);
        const float2 nl2 = make_float2(nl, nl), nds2 = make_float2(-Ds, -Ds);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int lim = M - m0 - 32 * h;  // columns of this half with a summary
          uint32_t zm = xm[h] | (live ? 0u : 0xffffffffu);
          if (lim < 32) zm |= lim <= 0 ? 0xffffffffu : (0xffffffffu << lim);
          uint32_t sv[32], dv[32];
          tc::tmem_ld32(tl + kS + 32 * h, sv);
          tc::tmem_ld32(tl + kP + 32 * h, dv);
          tc::tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 x = tc::fma2(make_float2(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])),
                                      sl2, nl2);
            float2 p = make_float2(btc::ex2(x.x), btc::ex2(x.y));
            p.x = ((zm >> k) & 1u) ? 0.f : p.x;
            p.y = ((zm >> (k + 1)) & 1u) ? 0.f : p.y;
            const float2 t = tc::fma2(make_float2(__uint_as_float(dv[k]), __uint_as_float(dv[k + 1])),
                                      sc2, nds2);
            const float2 ds = btc::mul2(p, t);
            pk[k >> 1] = tc::pack_bf16(ds.x, ds.y);
          }
          tc::tmem_st16(tl + kS + 16 * h, pk);
        }
        tc::tmem_wait_st();
        tc::tc_fence_before();
        tc::mbar_arrive(&bars[B_PFULL]);
      }
      if (!ok) break;
      // epilogue: the tile's dq~ after the last chunk's MMA
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_DONE], (gc - 1) & 1))) break;
      tc::tc_fence_after();
      float* dst = P.out0 + grow * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t o[16];
        tc::tmem_ld16(tl + kO + c0, o);
        tc::tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int k = 0; k < 16; k += 4)
            *reinterpret_cast<float4*>(dst + c0 + k) =
                make_float4(__uint_as_float(o[k]), __uint_as_float(o[k + 1]),
                            __uint_as_float(o[k + 2]), __uint_as_float(o[k + 3]));
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&bars[B_OFREE]);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ q~ and dO_g tiles (cp.async)
    const int ptid = tid - 128;
    volatile int* pflag = abort_flag + 1;
    int pc = 0;
    for (int64_t u = blockIdx.x; u < P.units; u += gridDim.x, ++pc) {
      if (pc >= 1) {
        if (ptid == 0) *pflag = ab.wait(&bars[B_QEMPTY], (pc - 1) & 1) ? 1 : 0;
        asm volatile("bar.sync 1, 64;" ::: "memory");
        if (!*pflag) break;
      }
      const int64_t bh = u / P.units_per_bh;
      const int64_t row0 = (u % P.units_per_bh) * btc::kRows;
      for (int i = ptid; i < btc::kRows * KC; i += kProd) {
        int r, kc;
        tc::PieceOrder<KC>::at(i, r, kc);
        const int64_t row = row0 + r;
        const bool ok = row < N;
        const int64_t src = (bh * N + (ok ? row : 0)) * D + kc * 8;
        const int off = kc * 2048 + (r >> 3) * 128 + (r & 7) * 16;
        tc::cp_async16(smem + S::kQ + off, P.qtb + src, ok);
        tc::cp_async16(smem + S::kG + off, P.dogb + src, ok);
      }
      tc::cp_async_commit();
      tc::cp_async_wait_all();
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_QFULL]);
      asm volatile("bar.sync 1, 64;" ::: "memory");  // pflag reuse
    }
    tc::cp_async_wait_all();
  } else if (warp == 6) {
    // ------------------------------------------------------------ summary loader
    if (lane == 0) {
      const int64_t MT = sum_tiles(M);
      uint32_t kv = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x) {
        const int64_t bh = u / P.units_per_bh;
        for (int j = 0; j < NC; ++j, ++kv) {
          const int st = kv % S::kStages;
          if (kv >= (uint32_t)S::kStages &&
              !ab.wait(&bars[B_KVEMPTY + st], ((kv / S::kStages) - 1) & 1)) { ok = false; break; }
          tc::mbar_expect_tx(&bars[B_KVFULL + st], 2u * S::kCTile);
          const int64_t tile = (kv_of(bh, P.kv_group) * MT + j) * (int64_t)(btc::kChunk * D);
          tc::bulk_g2s(smem + S::kK + st * S::kCTile, P.ksum + tile, S::kCTile,
                       &bars[B_KVFULL + st]);
          tc::bulk_g2s(smem + S::kV + st * S::kCTile, P.vsum + tile, S::kCTile,
                       &bars[B_KVFULL + st]);
        }
      }
      for (uint32_t k = (kv > (uint32_t)S::kStages ? kv - S::kStages : 0); k < kv; ++k)
        tc::mbar_wait(&bars[B_KVFULL + (k % S::kStages)], (k / S::kStages) & 1, 4000000000LL);
    }
  } else {
    // ------------------------------------------------------------ MMA issuer (warp 7)
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0);
    const uint32_t id_s = tc::idesc_bf16_f32(128, btc::kChunk, false, false);
    const uint32_t id_q = tc::idesc_bf16_f32(128, D, false, true);
    const uint64_t qd = tc::smem_desc(tc::smem_u32(smem + S::kQ), 2048, 128);
    const uint64_t gd = tc::smem_desc(tc::smem_u32(smem + S::kG), 2048, 128);
    const uint64_t kd0 = tc::smem_desc(tc::smem_u32(smem + S::kK), CB, 128);    // K-major
    const uint64_t vd0 = tc::smem_desc(tc::smem_u32(smem + S::kV), CB, 128);
    const uint64_t km0 = tc::smem_desc(tc::smem_u32(smem + S::kK), 128, CB);    // MN-major
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    uint32_t gc = 0;
    int pc = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < P.units && ok; u += gridDim.x, ++pc) {
      if (!wwait(&bars[B_QFULL], pc & 1)) break;
      tc::tc_fence_after();
      for (int j = 0; j < NC; ++j, ++gc) {
        const int st = gc % S::kStages;
        if (!wwait(&bars[B_KVFULL + st], (gc / S::kStages) & 1)) { ok = false; break; }
        // S and dP hold the previous chunk's dS until its MMA has completed
        if (gc >= 1 && !wwait(&bars[B_DONE], (gc - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        const uint64_t ko = (uint64_t)((st * S::kCTile) >> 4);
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            tc::mma_ss(tb + kS, qd + (uint64_t)(ks * (4096 >> 4)),
                       kd0 + ko + (uint64_t)(ks * (2 * CB >> 4)), id_s, ks > 0);
            tc::mma_ss(tb + kP, gd + (uint64_t)(ks * (4096 >> 4)),
                       vd0 + ko + (uint64_t)(ks * (2 * CB >> 4)), id_s, ks > 0);
          }
          tc::tc_commit(&bars[B_SFULL]);
          if (j == NC - 1) tc::tc_commit(&bars[B_QEMPTY]);  // q~ / dO_g tiles consumed
        }
        __syncwarp();
        if (!wwait(&bars[B_PFULL], gc & 1)) { ok = false; break; }
        if (j == 0 && pc >= 1 && !wwait(&bars[B_OFREE], (pc - 1) & 1)) { ok = false; break; }
        tc::tc_fence_after();
        if (tc::elect_one()) {
#pragma unroll
          for (int ks = 0; ks < btc::kChunk / 16; ++ks)
            tc::mma_ts(tb + kO, tb + kS + ks * 8, km0 + ko + (uint64_t)(ks * (256 >> 4)), id_q,
                       (j > 0 || ks > 0) ? 1u : 0u);
          tc::tc_commit(&bars[B_KVEMPTY + st]);
          tc::tc_commit(&bars[B_DONE]);
        }
        __syncwarp();
      }
    }
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
    tc::tmem_dealloc(tbase, 256);
  }
}

// ======================================================================= dK, dV (summaries)
namespace bds {
constexpr int kStages = 4;
constexpr int kLag = 1;  // a tile's row data is finalized this many tiles after its copies
template <int D> struct Smem {
  static constexpr int kATile = btc::kRows * D * 2;    // K or V summaries, 128 rows
  static constexpr int kBTile = btc::kChunk * D * 2;   // q~ or dO_g, 64 rows
  static constexpr int kK = 0;
  static constexpr int kV = kK + kATile;
  static constexpr int kQ = kV + kATile;               // [stages]
  static constexpr int kG = kQ + kStages * kBTile;     // [stages]
  static constexpr int kRowF = kG + kStages * kBTile;          // [stages][64] (nl, D)
  static constexpr int kRowX = kRowF + kStages * btc::kChunk * 8;  // [stages][64][6] ranges
  // [stages][3][64] raw lse, D and packed coordinate of the tile's queries, as copied
  static constexpr int kRaw = kRowX + kStages * btc::kChunk * 24;
  static constexpr int kBar = kRaw + kStages * 3 * btc::kChunk * 4;
  static constexpr int kBytes = kBar + 256;
};
enum {
  B_QFULL = 0, B_QEMPTY = B_QFULL + kStages, B_AFULL = B_QEMPTY + kStages, B_SFULL = B_AFULL + 1,
  B_PFULL = B_SFULL + 2, B_DONE = B_PFULL + 2, B_DRAIN = B_DONE + 2, B_COUNT = B_DRAIN + 1
};
static_assert(8 * B_COUNT + 16 <= 256, "barrier area");
constexpr int kThreads = 288;  // elementwise 0-3, producer 4-7, MMA 8
constexpr int kProd = 128;
// TMEM columns: dK, dV accumulators; S^T and dP^T double-buffered (buffer b of tile i = i % 2)
constexpr uint32_t kK = 0, kV = 128;
__device__ __forceinline__ uint32_t s_col(int b) { return 256u + 128u * b; }
__device__ __forceinline__ uint32_t p_col(int b) { return 320u + 128u * b; }
// Per query of a tile (staged by the producer): (-lse log2(e), D tau) -- -inf in place of the
// first term when the query has no global gradient, so that P = 0 -- and the block
// coordinate ranges [z0, z1] x [y0, y1] x [x0, x1] of the summaries exclude_near drops.
}  // namespace bds

template <int D>
__global__ void __launch_bounds__(bds::kThreads, 1) k_bwd_dsum_tc(const btc::Params P) {
  using namespace bds;
  using S = Smem<D>;
  constexpr int KC = D / 8;
  constexpr int CB = btc::kChunk * 16;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kBar + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kBar + 8 * B_COUNT + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tc::Abort ab{abort_flag, P.ix.status, P.wait_budget};
  const int64_t N = P.ix.n;
  const int M = (int)P.ix.m;
  // work item: (batch*head, 128-summary tile, query range)
  const int64_t item = blockIdx.x;
  const int split = (int)(item % P.nsplit);
  const int mt = (int)((item / P.nsplit) % P.m_tiles);
  const int64_t bh = item / ((int64_t)P.nsplit * P.m_tiles);
  const int qt0 = split * P.q_per_split;
  const int qt1 = min(P.q_tiles, qt0 + P.q_per_split);
  const int NT = max(qt1 - qt0, 0);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&bars[B_QFULL + i], kProd);
      tc::mbar_init(&bars[B_QEMPTY + i], 1);
    }
    tc::mbar_init(&bars[B_AFULL], kProd);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&bars[B_SFULL + i], 1);
      tc::mbar_init(&bars[B_PFULL + i], 128);
      tc::mbar_init(&bars[B_DONE + i], 1);
    }
    tc::mbar_init(&bars[B_DRAIN], 1);
    abort_flag[0] = 0;
    tc::fence_mbar_init();
  }
  if (warp == 8) tc::tmem_alloc(tmem_slot, 512);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ elementwise + epilogue
    const int rin = warp * 32 + lane;           // summary row of the tile
    const int m = mt * btc::kRows + rin;        // summary id
    const uint32_t tl = tbase + ((uint32_t)(warp * 32) << 16);
    const int nby = P.ix.sum_grid[1], nbx = P.ix.sum_grid[2];
    const int bz = m / (nby * nbx), byy = (m / nbx) % nby, bxx = m % nbx;  // summary coords
    const bool excl = P.exclude_near != 0;
    const float2* rowf = reinterpret_cast<const float2*>(smem + S::kRowF);
    const int* rowx = reinterpret_cast<const int*>(smem + S::kRowX);
    bool ok = true;
    for (int i = 0; i < NT; ++i) {
      const int st = i % kStages, b = i & 1;
      if (!__all_sync(0xffffffffu, ab.wait(&bars[B_SFULL + b], (i >> 1) & 1))) { ok = false; break; }
      tc::tc_fence_after();
      const float2* rf = rowf + st * btc::kChunk;
      const int* rx = rowx + st * btc::kChunk * 6;
      // two halves of 32 query columns: P^T over S^T, dS^T over dP^T (columns already read).
      // Two columns per step with packed fp32: P = 2^(S tau log2(e) - lse log2(e)),
      // dS = P (dP tau - D tau); one 16-byte read brings both columns' row data.
      const float4* rf4 = reinterpret_cast<const float4*>(rf);
      const float2 sl2 = make_float2(P.scale_log2, P.scale_log2);
      const float2 sc2 = make_float2(P.scale, P.scale);
      auto pass = [&](auto excl_c) {
        constexpr bool kExcl = decltype(excl_c)::value;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[32], dv[32];
          tc::tmem_ld32(tl + s_col(b) + 32 * h, sv);
          tc::tmem_ld32(tl + p_col(b) + 32 * h, dv);
          tc::tmem_wait_ld();
          uint32_t pp[16], pd[16];
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const int col = 32 * h + k;
            const float4 r = rf4[col >> 1];  // broadcast: every thread reads the same
            const float2 x = tc::fma2(make_float2(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])),
                                      sl2, make_float2(r.x, r.z));
            float2 p = make_float2(btc::ex2(x.x), btc::ex2(x.y));
            if constexpr (kExcl) {
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int* xr = rx + (col + e) * 6;
                if (bz >= xr[0] && bz <= xr[1] && byy >= xr[2] && byy <= xr[3] && bxx >= xr[4] &&
                    bxx <= xr[5])
                  (e == 0 ? p.x : p.y) = 0.f;
              }
            }
            const float2 t = tc::fma2(make_float2(__uint_as_float(dv[k]), __uint_as_float(dv[k + 1])),
                                      sc2, make_float2(-r.y, -r.w));
            const float2 ds = btc::mul2(p, t);
            pp[k >> 1] = tc::pack_bf16(p.x, p.y);
            pd[k >> 1] = tc::pack_bf16(ds.x, ds.y);
          }
          tc::tmem_st16(tl + s_col(b) + 16 * h, pp);
          tc::tmem_st16(tl + p_col(b) + 16 * h, pd);
        }
      };
      if (excl)
        pass(std::true_type{});
      else
        pass(std::false_type{});
      tc::tmem_wait_st();
      tc::tc_fence_before();
      tc::mbar_arrive(&bars[B_PFULL + b]);
    }
    // epilogue: this range's partial dK, dV of the tile's summaries
    if (ok && NT > 0 &&
        __all_sync(0xffffffffu, ab.wait(&bars[B_DONE + ((NT - 1) & 1)], ((NT - 1) >> 1) & 1))) {
      tc::tc_fence_after();
      const int64_t part = (int64_t)split * P.bh_count * M * D;
      float* dk = P.out0 + part + (bh * M + m) * D;
      float* dv = P.out1 + part + (bh * M + m) * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t a[16], b[16];
        tc::tmem_ld16(tl + kK + c0, a);
        tc::tmem_ld16(tl + kV + c0, b);
        tc::tmem_wait_ld();
        if (m < M) {
#pragma unroll
          for (int k = 0; k < 16; k += 4) {
            *reinterpret_cast<float4*>(dk + c0 + k) =
                make_float4(__uint_as_float(a[k]), __uint_as_float(a[k + 1]),
                            __uint_as_float(a[k + 2]), __uint_as_float(a[k + 3]));
            *reinterpret_cast<float4*>(dv + c0 + k) =
                make_float4(__uint_as_float(b[k]), __uint_as_float(b[k + 1]),
                            __uint_as_float(b[k + 2]), __uint_as_float(b[k + 3]));
          }
        }
      }
    } else if (ok && NT == 0 && m < M) {
      // an empty query range contributes zeros
      const int64_t part = (int64_t)split * P.bh_count * M * D;
      for (int e = 0; e < D; ++e) {
        P.out0[part + (bh * M + m) * D + e] = 0.f;
        P.out1[part + (bh * M + m) * D + e] = 0.f;
      }
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ operands (cp.async)
    const int ptid = tid - 128;
    volatile int* pflag = abort_flag + 1;
    int nwait = 0;
    auto pwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      volatile int* f = pflag + (nwait++ & 1);
      if (ptid == 0) *f = ab.wait(bar, parity) ? 1 : 0;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      return *f != 0;
    };
    // the tile's K and V summaries as 128-row K-major A operands (rows past the summary
    // tiles read as zeros)
    const int64_t MT = sum_tiles(M);
    for (int i = ptid; i < btc::kRows * KC; i += kProd) {
      int r, kc;
      tc::PieceOrder<KC>::at(i, r, kc);
      const int m = mt * btc::kRows + r;
      const bool ok = m < MT * 64;
      const int64_t src = ((kv_of(bh, P.kv_group) * MT + (ok ? m / 64 : 0)) * (D / 8) + kc) * 512 +
                          (ok ? m % 64 : 0) * 8;
      const int off = kc * 2048 + (r >> 3) * 128 + (r & 7) * 16;
      tc::cp_async16(smem + S::kK + off, P.ksum + src, ok);
      tc::cp_async16(smem + S::kV + off, P.vsum + src, ok);
    }
    tc::cp_async_commit();
    tc::cp_async_wait_all();
    tc::fence_proxy_async_smem();
    tc::mbar_arrive(&bars[B_AFULL]);
    // Software pipeline: at step i the copies of tile i are issued (q~ and dO_g rows, and
    // each query's lse, D and coordinate as raw 4-byte copies), and tile i - kLag, whose
    // copies have landed, is finalized: its per-query (-lse log2(e), D) and exclusion ranges
    // are formed in shared memory and the tile is handed to the MMA warp. No producer thread
    // waits on a global load, and kLag + 1 tiles are in flight.
    const float* raw = reinterpret_cast<const float*>(smem + S::kRaw);
    bool pok = true;
    for (int i = 0; i < NT + kLag && pok; ++i) {
      if (i < NT) {
        const int st = i % kStages;
        if (i >= kStages && !pwait(&bars[B_QEMPTY + st], ((i / kStages) - 1) & 1)) {
          pok = false;
          break;
        }
        const int64_t row0 = (int64_t)(qt0 + i) * btc::kChunk;
        for (int k = ptid; k < btc::kChunk * KC; k += kProd) {
          int r, kc;
          tc::PieceOrder<KC>::at(k, r, kc);
          const int64_t row = row0 + r;
          const bool ok = row < N;
          const int64_t src = (bh * N + (ok ? row : 0)) * D + kc * 8;
          const int off = st * S::kBTile + kc * CB + (r >> 3) * 128 + (r & 7) * 16;
          tc::cp_async16(smem + S::kQ + off, P.qtb + src, ok);
          tc::cp_async16(smem + S::kG + off, P.dogb + src, ok);
        }
        if (ptid < btc::kChunk) {
          const int64_t row = row0 + ptid;
          const bool ok = row < N;
          const int64_t g = bh * N + (ok ? row : 0);
          float* rw = reinterpret_cast<float*>(smem + S::kRaw) + st * 3 * btc::kChunk;
          btc::cp_async4(rw + ptid, P.lse + g, ok);
          btc::cp_async4(rw + btc::kChunk + ptid, P.Dg + g, ok);
          if (P.exclude_near)
            btc::cp_async4(rw + 2 * btc::kChunk + ptid, P.ix.coord + (ok ? row : 0), ok);
        }
      }
      tc::cp_async_commit();  // one group per step (empty past the last tile)
      const int f = i - kLag;
      if (f < 0) continue;
      tc::cp_async_wait_group<kLag>();  // tile f's copies have landed
      const int sf = f % kStages;
      if (ptid < btc::kChunk) {
        const int64_t row = (int64_t)(qt0 + f) * btc::kChunk + ptid;
        const float* rw = raw + sf * 3 * btc::kChunk;
        float2 rf = make_float2(-INFINITY, 0.f);
        ExclBox ex{0, -1, 0, -1, 0, -1};
        if (row < N) {
          const float lse = rw[ptid];
          rf = make_float2(lse != -INFINITY ? -lse * kLog2e : -INFINITY,
                           rw[btc::kChunk + ptid] * P.scale);
          if (P.exclude_near)
            ex = excl_box(P.ix, decode(__float_as_int(rw[2 * btc::kChunk + ptid])), true);
        }
        reinterpret_cast<float2*>(smem + S::kRowF)[sf * btc::kChunk + ptid] = rf;
        int* x = reinterpret_cast<int*>(smem + S::kRowX) + (sf * btc::kChunk + ptid) * 6;
        x[0] = ex.z0; x[1] = ex.z1; x[2] = ex.y0; x[3] = ex.y1; x[4] = ex.x0; x[5] = ex.x1;
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[B_QFULL + sf]);
    }
    tc::cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ MMA issuer (warp 8)
    const uint32_t tb = __shfl_sync(0xffffffffu, tbase, 0);
    const uint32_t id_s = tc::idesc_bf16_f32(128, btc::kChunk, false, false);
    const uint32_t id_o = tc::idesc_bf16_f32(128, D, false, true);
    const uint64_t kd = tc::smem_desc(tc::smem_u32(smem + S::kK), 2048, 128);
    const uint64_t vd = tc::smem_desc(tc::smem_u32(smem + S::kV), 2048, 128);
    const uint64_t qk0 = tc::smem_desc(tc::smem_u32(smem + S::kQ), CB, 128);   // K-major
    const uint64_t gk0 = tc::smem_desc(tc::smem_u32(smem + S::kG), CB, 128);
    const uint64_t qm0 = tc::smem_desc(tc::smem_u32(smem + S::kQ), 128, CB);   // MN-major
    const uint64_t gm0 = tc::smem_desc(tc::smem_u32(smem + S::kG), 128, CB);
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, ab.wait(bar, parity, false));
    };
    // SS(i): S^T and dP^T of query tile i into buffer i % 2 (free once TS(i - 2) completed)
    auto issue_ss = [&](int i) -> bool {
      const int st = i % kStages, b = i & 1;
      if (!wwait(&bars[B_QFULL + st], (i / kStages) & 1)) return false;
      if (i >= 2 && !wwait(&bars[B_DONE + b], ((i - 2) >> 1) & 1)) return false;
      tc::tc_fence_after();
      const uint64_t so = (uint64_t)((st * S::kBTile) >> 4);
      if (tc::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          tc::mma_ss(tb + s_col(b), kd + (uint64_t)(ks * (4096 >> 4)),
                     qk0 + so + (uint64_t)(ks * (2 * CB >> 4)), id_s, ks > 0);
          tc::mma_ss(tb + p_col(b), vd + (uint64_t)(ks * (4096 >> 4)),
                     gk0 + so + (uint64_t)(ks * (2 * CB >> 4)), id_s, ks > 0);
        }
        tc::tc_commit(&bars[B_SFULL + b]);
      }
      __syncwarp();
      return true;
    };
    bool ok = wwait(&bars[B_AFULL], 0);
    for (int i = 0; i < 2 && i < NT && ok; ++i) ok = issue_ss(i);
    for (int i = 0; i < NT && ok; ++i) {
      const int st = i % kStages, b = i & 1;
      if (!wwait(&bars[B_PFULL + b], (i >> 1) & 1)) break;
      tc::tc_fence_after();
      const uint64_t so = (uint64_t)((st * S::kBTile) >> 4);
      if (tc::elect_one()) {
#pragma unroll
        for (int ks = 0; ks < btc::kChunk / 16; ++ks) {
          // dV += P^T dO_g;  dK += dS^T q~   (K = the tile's 64 queries)
          tc::mma_ts(tb + kV, tb + s_col(b) + ks * 8, gm0 + so + (uint64_t)(ks * (256 >> 4)),
                     id_o, (i > 0 || ks > 0) ? 1u : 0u);
          tc::mma_ts(tb + kK, tb + p_col(b) + ks * 8, qm0 + so + (uint64_t)(ks * (256 >> 4)),
                     id_o, (i > 0 || ks > 0) ? 1u : 0u);
        }
        tc::tc_commit(&bars[B_QEMPTY + st]);
        tc::tc_commit(&bars[B_DONE + b]);
      }
      __syncwarp();
      if (i + 2 < NT) ok = issue_ss(i + 2);
    }
    if (tc::elect_one()) tc::tc_commit(&bars[B_DRAIN]);
    __syncwarp();
    if (!tc::mbar_wait(&bars[B_DRAIN], 0, 100000000LL))
      set_status(P.ix.status, PACK3D_ERR_TIMEOUT);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    __syncwarp();
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, 512);
  }
}

// Adds the per-query-range partials 1 .. nsplit-1 of the summary gradients, in range order,
// into partial 0 (deterministic), so the un-pooling reads one.
__global__ void __launch_bounds__(256) k_sum_splits(float* __restrict__ dks,
                                                    float* __restrict__ dvs, int64_t elems,
                                                    int nsplit) {
  const int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (e >= elems) return;
  float sk = dks[e], sv = dvs[e];
  for (int sp = 1; sp < nsplit; ++sp) {
    sk += dks[sp * elems + e];
    sv += dvs[sp * elems + e];
  }
  dks[e] = sk;
  dvs[e] = sv;
}

// Query ranges per (batch, head) for the summary-gradient kernel (one CTA per SM): the count
// in [1, kDsumSplitMax] whose CTAs fill the last wave best (fewer ranges on a tie).
inline int dsum_splits(int64_t bh_tiles, int q_tiles, int sms) {
  int best = 1;
  double best_eff = 0.0;
  for (int sp = 1; sp <= kDsumSplitMax && sp <= q_tiles; ++sp) {
    const int64_t items = bh_tiles * sp;
    const int64_t waves = (items + sms - 1) / sms;
    const double eff = (double)items / (double)(waves * sms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = sp;
    }
  }
  return best;
}

// ------------------------------------------------------------------------------ host side
template <int D>
cudaError_t launch_bwd_tc(const pack3d_index& ix, const BwdWork& w, const void* ksum,
                          const void* vsum, const float* lse_glob, int64_t bh, int kv_group,
                          float scale, int excl, cudaStream_t s) {
  static std::atomic<uint64_t> attr_dq{0}, attr_dsum{0};
  if (smem_attr_once(reinterpret_cast<const void*>(k_bwd_dq_tc<D>), bdq::Smem<D>::kBytes,
                     attr_dq) != cudaSuccess ||
      smem_attr_once(reinterpret_cast<const void*>(k_bwd_dsum_tc<D>), bds::Smem<D>::kBytes,
                     attr_dsum) != cudaSuccess)
    return cudaErrorInvalidValue;
  btc::Params p;
  p.ix = ix;
  p.qtb = w.qtb;
  p.dogb = w.dogb;
  p.ksum = static_cast<const __nv_bfloat16*>(ksum);
  p.vsum = static_cast<const __nv_bfloat16*>(vsum);
  p.lse = lse_glob;
  p.Dg = w.Dg;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.exclude_near = excl;
  p.wait_budget = wait_budget_cycles();
  p.kv_group = kv_group;
  p.bh_count = bh;
  // summary gradients: (batch*head) x 128-summary tiles x query ranges
  p.m_tiles = (int)((ix.m + btc::kRows - 1) / btc::kRows);
  p.q_tiles = (int)((ix.n + btc::kChunk - 1) / btc::kChunk);
  p.nsplit = dsum_splits(bh * p.m_tiles, p.q_tiles, sm_count());
  p.q_per_split = (p.q_tiles + p.nsplit - 1) / p.nsplit;
  p.out0 = w.dks;
  p.out1 = w.dvs;
  const int64_t items = bh * p.m_tiles * p.nsplit;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  k_bwd_dsum_tc<D><<<(unsigned)items, bds::kThreads, bds::Smem<D>::kBytes, s>>>(p);
  if (p.nsplit > 1) {
    const int64_t elems = bh * ix.m * D;
    k_sum_splits<<<(unsigned)((elems + 255) / 256), 256, 0, s>>>(w.dks, w.dvs, elems, p.nsplit);
    count_launch();
  }
  // dq~: persistent over 128-query tiles, two CTAs per SM
  p.units_per_bh = (ix.n + btc::kRows - 1) / btc::kRows;
  p.units = bh * p.units_per_bh;
  p.n_chunks = (int)((ix.m + btc::kChunk - 1) / btc::kChunk);
  p.out0 = w.dqg;
  p.out1 = nullptr;
  const int64_t cap = 2 * (int64_t)sm_count();
  const unsigned grid = (unsigned)(p.units < cap ? p.units : cap);
  k_bwd_dq_tc<D><<<grid, bdq::kThreads, bdq::Smem<D>::kBytes, s>>>(p);
  count_launch(2);
  return cudaGetLastError();
}

cudaError_t bwd_tc_dispatch(const pack3d_index& ix, const BwdWork& w, const void* ksum,
                            const void* vsum, const float* lse_glob, int64_t bh, int kv_group,
                            float scale, int excl, cudaStream_t s) {
  if (ix.geom.head_dim == 96)
    return launch_bwd_tc<96>(ix, w, ksum, vsum, lse_glob, bh, kv_group, scale, excl, s);
  return launch_bwd_tc<48>(ix, w, ksum, vsum, lse_glob, bh, kv_group, scale, excl, s);
}

}  // namespace p3d
