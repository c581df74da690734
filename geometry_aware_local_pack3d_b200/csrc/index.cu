// Index build of a packed field: coordinate -> slot inverse map, 27-neighbour table, block
// membership tables and the axial-RoPE rotation table.
//
// Project page "Geometry Matters in Packed 3D Attention", Chapter 3 Contract 1: the
// neighbourhood is defined by coordinate offsets and validity, never by adjacency in the
// packed array; Chapter 4 Proposition 2: coordinate, neighbourhood edges, block membership
// and the canonical within-block slot travel with each token. Paper summary §B.1.
#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace p3d {

// Packed coordinates from either (z, y, x) triples or raster ids; flags out-of-range.
__global__ void k_coords(const int32_t* __restrict__ coords, const int64_t* __restrict__ perm,
                         int64_t n, int gz, int gy, int gx, int32_t* __restrict__ coord_out,
                         int32_t* status) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  int64_t z, y, x;
  if (coords) {
    z = coords[3 * i];
    y = coords[3 * i + 1];
    x = coords[3 * i + 2];
  } else {
    const int64_t r = perm[i];
    if (r < 0 || r >= (int64_t)gz * gy * gx) {
      set_status(status, PACK3D_ERR_COORD_RANGE);
      coord_out[i] = -1;
      return;
    }
    z = r / ((int64_t)gy * gx);
    y = (r / gx) % gy;
    x = r % gx;
  }
  if (z < 0 || z >= gz || y < 0 || y >= gy || x < 0 || x >= gx) {
    set_status(status, PACK3D_ERR_COORD_RANGE);
    coord_out[i] = -1;
    return;
  }
  coord_out[i] = (int32_t)((z << 20) | (y << 10) | x);
}

// inv[raster(c_i)] = i; a second token at the same site is a duplicate.
__global__ void k_inverse(const int32_t* __restrict__ coord, int64_t n, int gy, int gx,
                          int32_t* inv, int32_t* status) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int32_t cc = coord[i];
  if (cc < 0) return;
  const Coord c = decode(cc);
  const int64_t r = ((int64_t)c.z * gy + c.y) * gx + c.x;
  const int32_t old = atomicCAS(inv + r, -1, (int32_t)i);
  if (old != -1) set_status(status, PACK3D_ERR_DUP_COORD);
}

// nbr[i][o] = inv[c_i + delta_o], o = 9(dz+1) + 3(dy+1) + (dx+1).
__global__ void k_neighbours(const int32_t* __restrict__ coord, const int32_t* __restrict__ inv,
                             int64_t n, int gz, int gy, int gx, int32_t* __restrict__ nbr) {
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= n * kNbr) return;
  const int64_t i = t / kNbr;
  const int o = (int)(t % kNbr);
  const int32_t cc = coord[i];
  int32_t out = -1;
  if (cc >= 0) {
    const Coord c = decode(cc);
    const int z = c.z + o / 9 - 1, y = c.y + (o / 3) % 3 - 1, x = c.x + o % 3 - 1;
    if (z >= 0 && z < gz && y >= 0 && y < gy && x >= 0 && x < gx)
      out = inv[((int64_t)z * gy + y) * gx + x];
  }
  nbr[t] = out;
}

// block_of, slot_of and members[block][slot] = i (blocks tile the grid from the origin; the
// block grid is rounded up, so blocks at the far edges may stick out of the grid).
__global__ void k_blocks(const int32_t* __restrict__ coord, int64_t n, pack3d_geom g,
                         int32_t* __restrict__ block_of, int32_t* __restrict__ slot_of,
                         int32_t* __restrict__ members) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int32_t cc = coord[i];
  if (cc < 0) {
    block_of[i] = -1;
    slot_of[i] = -1;
    return;
  }
  const Coord c = decode(cc);
  const int nby = (g.gy + g.by - 1) / g.by, nbx = (g.gx + g.bx - 1) / g.bx;
  const int b = ((c.z / g.bz) * nby + c.y / g.by) * nbx + c.x / g.bx;
  const int s = ((c.z % g.bz) * g.by + c.y % g.by) * g.bx + c.x % g.bx;
  block_of[i] = b;
  slot_of[i] = s;
  members[(int64_t)b * (g.bz * g.by * g.bx) + s] = (int32_t)i;
}

__global__ void k_count(const int32_t* __restrict__ members, int64_t m, int vol,
                        int32_t* __restrict__ count) {
  int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (b >= m) return;
  int c = 0;
  for (int s = 0; s < vol; ++s) c += members[b * vol + s] >= 0;
  count[b] = c;
}

// Second pooling stage: summary t holds the blocks of a pz x py x px group of the block grid,
// raster inside the group (-1 past the block grid); count2[t] = its non-empty blocks, bit t of
// `empty` set when it has none (status[1] counts those summaries).
__global__ void k_groups(const int32_t* __restrict__ count, int nbz, int nby, int nbx, int pz,
                         int py, int px, int ngy, int ngx, int64_t m_sum,
                         int32_t* __restrict__ groups, int32_t* __restrict__ count2,
                         uint32_t* __restrict__ empty, int32_t* status) {
  int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= m_sum) return;
  const int gx = (int)(t % ngx), gy = (int)((t / ngx) % ngy), gz = (int)(t / ((int64_t)ngx * ngy));
  const int gv = pz * py * px;
  int c2 = 0;
  for (int s = 0; s < gv; ++s) {
    const int mz = gz * pz + s / (py * px), my = gy * py + (s / px) % py, mx = gx * px + s % px;
    int32_t m = -1;
    if (mz < nbz && my < nby && mx < nbx) {
      m = (mz * nby + my) * nbx + mx;
      c2 += count[m] > 0;
    }
    groups[t * gv + s] = m;
  }
  count2[t] = c2;
  if (c2 == 0) {
    atomicOr(empty + (t >> 5), 1u << (t & 31));
    atomicAdd(status + 1, 1);
  }
}

// sum_of[i]: the summary (group) of each token's block.
__global__ void k_sum_of(const int32_t* __restrict__ block_of, int64_t n, int nby, int nbx,
                         int pz, int py, int px, int ngy, int ngx, int32_t* __restrict__ sum_of) {
  int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int b = block_of[i];
  if (b < 0) {
    sum_of[i] = -1;
    return;
  }
  const int mx = b % nbx, my = (b / nbx) % nby, mz = b / (nbx * nby);
  sum_of[i] = ((mz / pz) * ngy + my / py) * ngx + mx / px;
}

// rope[a][c][p] = (cos, sin)(s_a * c * base^(-2p/d_a)), evaluated in double and rounded to
// float.
__global__ void k_rope_table(int rows, int pairs, double base, double s0, double s1, double s2,
                             float* __restrict__ rope) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= 3 * rows * pairs) return;
  const int a = t / (rows * pairs), c = (t / pairs) % rows, p = t % pairs;
  const double da = 2.0 * pairs;
  const double theta = pow(base, -2.0 * p / da);
  const double sc = a == 0 ? s0 : (a == 1 ? s1 : s2);
  double s, co;
  sincos(sc * (double)c * theta, &s, &co);
  rope[2 * t] = (float)co;
  rope[2 * t + 1] = (float)s;
}

// rope_c[t][e/2] = (cos, sin) of the angle of dims (e, e+1) at the centre of summary t's box
// (lo + hi) / 2, lo = t's grid position * ext, hi = min(lo + ext, G) - 1, per axis.
__global__ void k_rope_centre(int64_t m_sum, int pairs, double base, pack3d_geom g, int ez,
                              int ey, int ex, int ngy, int ngx, float* __restrict__ rope_c) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int hp = 3 * pairs;  // rotation pairs of a head
  if (t >= m_sum * hp) return;
  const int64_t m = t / hp;
  const int e2 = (int)(t % hp), a = e2 / pairs, p = e2 % pairs;
  const int pos = a == 0 ? (int)(m / ((int64_t)ngx * ngy))
                         : (a == 1 ? (int)((m / ngx) % ngy) : (int)(m % ngx));
  const int ext = a == 0 ? ez : (a == 1 ? ey : ex);
  const int G = a == 0 ? g.gz : (a == 1 ? g.gy : g.gx);
  const int lo = pos * ext, hi = min(lo + ext, G) - 1;
  const double sp = g.spacing[a] > 0.f ? (double)g.spacing[a] : 1.0;
  const double theta = pow(base, -2.0 * p / (2.0 * pairs));
  double s, co;
  sincos(sp * 0.5 * (double)(lo + hi) * theta, &s, &co);
  rope_c[2 * t] = (float)co;
  rope_c[2 * t + 1] = (float)s;
}

}  // namespace p3d

using namespace p3d;

namespace {
struct IndexLayout {
  size_t coord, inv, nbr, block_of, slot_of, members, count, sum_of, groups, count2, empty, rope,
      rope_c, status, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
inline int pool_ext(int32_t p) { return p > 1 ? p : 1; }

// Block, summary and rotation-table sizes of a geometry (valid geometries only).
struct Plan {
  int nb[3], pe[3], ext[3], ng[3];
  int64_t sites, n_blocks, m, vol, gv;
  int rows;
};
Plan plan_of(const pack3d_geom* g) {
  Plan P{};
  const int G[3] = {g->gz, g->gy, g->gx}, b[3] = {g->bz, g->by, g->bx};
  const int32_t p[3] = {g->pz, g->py, g->px};
  P.sites = (int64_t)G[0] * G[1] * G[2];
  P.n_blocks = 1;
  P.m = 1;
  P.vol = (int64_t)b[0] * b[1] * b[2];
  P.gv = 1;
  P.rows = 1;
  for (int a = 0; a < 3; ++a) {
    P.nb[a] = ceil_div(G[a], b[a]);
    P.pe[a] = pool_ext(p[a]);
    P.ext[a] = b[a] * P.pe[a];
    P.ng[a] = ceil_div(P.nb[a], P.pe[a]);
    P.n_blocks *= P.nb[a];
    P.m *= P.ng[a];
    P.gv *= P.pe[a];
    if (G[a] > P.rows) P.rows = G[a];
  }
  return P;
}

bool geom_ok(const pack3d_geom* g) {
  if (!g) return false;
  const int32_t e[3] = {g->gz, g->gy, g->gx}, b[3] = {g->bz, g->by, g->bx};
  const int32_t p[3] = {g->pz, g->py, g->px};
  for (int a = 0; a < 3; ++a) {
    if (e[a] < 1 || e[a] > 1024 || b[a] < 1 || b[a] > e[a]) return false;
    if (p[a] < 0 || p[a] > 1024) return false;
    if (!(g->spacing[a] >= 0.f) || g->spacing[a] > 1e6f) return false;  // also rejects NaN
  }
  if (g->head_dim <= 0 || g->head_dim % 6) return false;
  if (!(g->rope_base > 0.0f)) return false;
  if (g->summary_rope != PACK3D_ROPE_TOKEN && g->summary_rope != PACK3D_ROPE_CENTRE) return false;
  return true;
}

IndexLayout layout(const pack3d_geom* g, int64_t n) {
  IndexLayout L{};
  const Plan P = plan_of(g);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.coord = take(sizeof(int32_t) * n);
  L.inv = take(sizeof(int32_t) * P.sites);
  L.nbr = take(sizeof(int32_t) * n * kNbr);
  L.block_of = take(sizeof(int32_t) * n);
  L.slot_of = take(sizeof(int32_t) * n);
  L.members = take(sizeof(int32_t) * P.n_blocks * P.vol);
  L.count = take(sizeof(int32_t) * P.n_blocks);
  L.sum_of = take(sizeof(int32_t) * n);
  L.groups = take(sizeof(int32_t) * P.m * P.gv);
  L.count2 = take(sizeof(int32_t) * P.m);
  L.empty = take(sizeof(uint32_t) * ((P.m + 31) / 32));
  L.rope = take(sizeof(float) * 2 * 3 * P.rows * (g->head_dim / 6));
  L.rope_c = take(sizeof(float) * P.m * g->head_dim);
  L.status = take(sizeof(int32_t) * 4);
  L.total = off;
  return L;
}
}  // namespace

extern "C" size_t pack3d_index_bytes(const pack3d_geom* g, int64_t n) {
  if (!geom_ok(g) || n <= 0 || n > plan_of(g).sites) return 0;
  return layout(g, n).total;
}

extern "C" pack3d_status pack3d_build_index(const pack3d_geom* g, const int32_t* coords,
                                            const int64_t* perm, int64_t n, void* buf,
                                            size_t buf_bytes, pack3d_index* out,
                                            void* stream) {
  if (!g || !out || !buf || n <= 0) return PACK3D_ERR_INVALID_ARG;
  if ((coords == nullptr) == (perm == nullptr)) return PACK3D_ERR_INVALID_ARG;
  if (!geom_ok(g)) return PACK3D_ERR_INVALID_ARG;
  if (g->head_dim != 48 && g->head_dim != 96) return PACK3D_ERR_UNSUPPORTED;
  const Plan P = plan_of(g);
  if (n > P.sites) return PACK3D_ERR_INVALID_ARG;  // more tokens than lattice sites
  if (P.m > 0x7fffffffLL || P.n_blocks > 0x7fffffffLL) return PACK3D_ERR_UNSUPPORTED;
  if (((uintptr_t)buf) & 255) return PACK3D_ERR_ALIGN;
  if (coords && (((uintptr_t)coords) & 3)) return PACK3D_ERR_ALIGN;
  if (perm && (((uintptr_t)perm) & 7)) return PACK3D_ERR_ALIGN;
  const IndexLayout L = layout(g, n);
  if (buf_bytes < L.total) return PACK3D_ERR_WORKSPACE;

  char* base = static_cast<char*>(buf);
  pack3d_index ix{};
  ix.geom = *g;
  for (int a = 0; a < 3; ++a)
    if (!(ix.geom.spacing[a] > 0.f)) ix.geom.spacing[a] = 1.f;
  ix.geom.pz = P.pe[0];
  ix.geom.py = P.pe[1];
  ix.geom.px = P.pe[2];
  ix.n = n;
  ix.m = P.m;
  ix.n_blocks = P.n_blocks;
  ix.block_volume = (int32_t)P.vol;
  ix.rope_pairs = g->head_dim / 6;
  ix.rope_rows = P.rows;
  ix.group_volume = (int32_t)P.gv;
  for (int a = 0; a < 3; ++a) {
    ix.sum_ext[a] = P.ext[a];
    ix.sum_grid[a] = P.ng[a];
  }
  ix.coord = reinterpret_cast<int32_t*>(base + L.coord);
  ix.inv = reinterpret_cast<int32_t*>(base + L.inv);
  ix.nbr = reinterpret_cast<int32_t*>(base + L.nbr);
  ix.block_of = reinterpret_cast<int32_t*>(base + L.block_of);
  ix.slot_of = reinterpret_cast<int32_t*>(base + L.slot_of);
  ix.members = reinterpret_cast<int32_t*>(base + L.members);
  ix.count = reinterpret_cast<int32_t*>(base + L.count);
  ix.sum_of = reinterpret_cast<int32_t*>(base + L.sum_of);
  ix.groups = reinterpret_cast<int32_t*>(base + L.groups);
  ix.count2 = reinterpret_cast<int32_t*>(base + L.count2);
  ix.empty = reinterpret_cast<uint32_t*>(base + L.empty);
  ix.rope = reinterpret_cast<float*>(base + L.rope);
  ix.rope_c = reinterpret_cast<float*>(base + L.rope_c);
  ix.status = reinterpret_cast<int32_t*>(base + L.status);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int T = 256;
  auto blocks = [&](int64_t work) { return (unsigned)((work + T - 1) / T); };
  if (cudaMemsetAsync(ix.status, 0, sizeof(int32_t) * 4, s) != cudaSuccess ||
      cudaMemsetAsync(ix.inv, 0xff, sizeof(int32_t) * P.sites, s) != cudaSuccess ||
      cudaMemsetAsync(ix.members, 0xff, sizeof(int32_t) * P.n_blocks * P.vol, s) !=
          cudaSuccess ||
      cudaMemsetAsync(ix.empty, 0, sizeof(uint32_t) * ((P.m + 31) / 32), s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  k_coords<<<blocks(n), T, 0, s>>>(coords, perm, n, g->gz, g->gy, g->gx, ix.coord, ix.status);
  k_inverse<<<blocks(n), T, 0, s>>>(ix.coord, n, g->gy, g->gx, ix.inv, ix.status);
  k_neighbours<<<blocks(n * kNbr), T, 0, s>>>(ix.coord, ix.inv, n, g->gz, g->gy, g->gx, ix.nbr);
  k_blocks<<<blocks(n), T, 0, s>>>(ix.coord, n, *g, ix.block_of, ix.slot_of, ix.members);
  k_count<<<blocks(P.n_blocks), T, 0, s>>>(ix.members, P.n_blocks, (int)P.vol, ix.count);
  k_groups<<<blocks(P.m), T, 0, s>>>(ix.count, P.nb[0], P.nb[1], P.nb[2], P.pe[0], P.pe[1],
                                      P.pe[2], P.ng[1], P.ng[2], P.m, ix.groups, ix.count2,
                                      ix.empty, ix.status);
  k_sum_of<<<blocks(n), T, 0, s>>>(ix.block_of, n, P.nb[1], P.nb[2], P.pe[0], P.pe[1], P.pe[2],
                                    P.ng[1], P.ng[2], ix.sum_of);
  k_rope_table<<<blocks(3LL * ix.rope_rows * ix.rope_pairs), T, 0, s>>>(
      ix.rope_rows, ix.rope_pairs, (double)g->rope_base, (double)ix.geom.spacing[0],
      (double)ix.geom.spacing[1], (double)ix.geom.spacing[2], ix.rope);
  k_rope_centre<<<blocks(P.m * 3 * ix.rope_pairs), T, 0, s>>>(
      P.m, ix.rope_pairs, (double)g->rope_base, ix.geom, P.ext[0], P.ext[1], P.ext[2], P.ng[1],
      P.ng[2], ix.rope_c);
  if (cudaGetLastError() != cudaSuccess) return PACK3D_ERR_CUDA;

  int32_t st[2] = {0, 0};
  if (cudaMemcpyAsync(st, ix.status, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  ix.n_empty = st[1];
  *out = ix;
  return st[0] ? static_cast<pack3d_status>(st[0]) : PACK3D_OK;
}

extern "C" pack3d_status pack3d_device_status(const pack3d_index* idx, void* stream) {
  if (!idx || !idx->status) return PACK3D_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t st = 0;
  if (cudaMemcpyAsync(&st, idx->status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  if (st && cudaMemsetAsync(idx->status, 0, sizeof(int32_t), s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PACK3D_ERR_CUDA;
  return static_cast<pack3d_status>(st);
}
