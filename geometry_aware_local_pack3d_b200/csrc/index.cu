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

// block_of, slot_of and members[block][slot] = i.
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
  const int nby = g.gy / g.by, nbx = g.gx / g.bx;
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

// rope[c][p] = (cos, sin)(c * base^(-2p/d_a)), evaluated in double and rounded to float.
__global__ void k_rope_table(int rows, int pairs, double base, float* __restrict__ rope) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= rows * pairs) return;
  const int c = t / pairs, p = t % pairs;
  const double da = 2.0 * pairs;
  const double theta = pow(base, -2.0 * p / da);
  double s, co;
  sincos((double)c * theta, &s, &co);
  rope[2 * t] = (float)co;
  rope[2 * t + 1] = (float)s;
}

}  // namespace p3d

using namespace p3d;

namespace {
struct IndexLayout {
  size_t coord, inv, nbr, block_of, slot_of, members, count, rope, status, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool geom_ok(const pack3d_geom* g) {
  if (!g) return false;
  const int32_t e[3] = {g->gz, g->gy, g->gx}, b[3] = {g->bz, g->by, g->bx};
  for (int a = 0; a < 3; ++a) {
    if (e[a] < 1 || e[a] > 1024 || b[a] < 1 || b[a] > e[a] || e[a] % b[a]) return false;
  }
  if (g->head_dim <= 0 || g->head_dim % 6) return false;
  if (!(g->rope_base > 0.0f)) return false;
  return true;
}

IndexLayout layout(const pack3d_geom* g, int64_t n) {
  IndexLayout L{};
  const int64_t sites = (int64_t)g->gz * g->gy * g->gx;
  const int64_t m = (int64_t)(g->gz / g->bz) * (g->gy / g->by) * (g->gx / g->bx);
  const int64_t vol = (int64_t)g->bz * g->by * g->bx;
  int rows = g->gz;
  if (g->gy > rows) rows = g->gy;
  if (g->gx > rows) rows = g->gx;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  L.coord = take(sizeof(int32_t) * n);
  L.inv = take(sizeof(int32_t) * sites);
  L.nbr = take(sizeof(int32_t) * n * kNbr);
  L.block_of = take(sizeof(int32_t) * n);
  L.slot_of = take(sizeof(int32_t) * n);
  L.members = take(sizeof(int32_t) * m * vol);
  L.count = take(sizeof(int32_t) * m);
  L.rope = take(sizeof(float) * 2 * rows * (g->head_dim / 6));
  L.status = take(sizeof(int32_t) * 4);
  L.total = off;
  return L;
}
}  // namespace

extern "C" size_t pack3d_index_bytes(const pack3d_geom* g, int64_t n) {
  if (!geom_ok(g) || n <= 0) return 0;
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
  if (n != (int64_t)g->gz * g->gy * g->gx) return PACK3D_ERR_UNSUPPORTED;
  if (((uintptr_t)buf) & 255) return PACK3D_ERR_ALIGN;
  if (coords && (((uintptr_t)coords) & 3)) return PACK3D_ERR_ALIGN;
  if (perm && (((uintptr_t)perm) & 7)) return PACK3D_ERR_ALIGN;
  const IndexLayout L = layout(g, n);
  if (buf_bytes < L.total) return PACK3D_ERR_WORKSPACE;

  char* base = static_cast<char*>(buf);
  pack3d_index ix{};
  ix.geom = *g;
  ix.n = n;
  ix.m = (int64_t)(g->gz / g->bz) * (g->gy / g->by) * (g->gx / g->bx);
  ix.block_volume = g->bz * g->by * g->bx;
  ix.rope_pairs = g->head_dim / 6;
  ix.rope_rows = g->gz > g->gy ? (g->gz > g->gx ? g->gz : g->gx) : (g->gy > g->gx ? g->gy : g->gx);
  ix.coord = reinterpret_cast<int32_t*>(base + L.coord);
  ix.inv = reinterpret_cast<int32_t*>(base + L.inv);
  ix.nbr = reinterpret_cast<int32_t*>(base + L.nbr);
  ix.block_of = reinterpret_cast<int32_t*>(base + L.block_of);
  ix.slot_of = reinterpret_cast<int32_t*>(base + L.slot_of);
  ix.members = reinterpret_cast<int32_t*>(base + L.members);
  ix.count = reinterpret_cast<int32_t*>(base + L.count);
  ix.rope = reinterpret_cast<float*>(base + L.rope);
  ix.status = reinterpret_cast<int32_t*>(base + L.status);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t sites = (int64_t)g->gz * g->gy * g->gx;
  const int T = 256;
  auto blocks = [&](int64_t work) { return (unsigned)((work + T - 1) / T); };
  if (cudaMemsetAsync(ix.status, 0, sizeof(int32_t) * 4, s) != cudaSuccess ||
      cudaMemsetAsync(ix.inv, 0xff, sizeof(int32_t) * sites, s) != cudaSuccess ||
      cudaMemsetAsync(ix.members, 0xff, sizeof(int32_t) * ix.m * ix.block_volume, s) !=
          cudaSuccess)
    return PACK3D_ERR_CUDA;
  k_coords<<<blocks(n), T, 0, s>>>(coords, perm, n, g->gz, g->gy, g->gx, ix.coord, ix.status);
  k_inverse<<<blocks(n), T, 0, s>>>(ix.coord, n, g->gy, g->gx, ix.inv, ix.status);
  k_neighbours<<<blocks(n * kNbr), T, 0, s>>>(ix.coord, ix.inv, n, g->gz, g->gy, g->gx, ix.nbr);
  k_blocks<<<blocks(n), T, 0, s>>>(ix.coord, n, *g, ix.block_of, ix.slot_of, ix.members);
  k_count<<<blocks(ix.m), T, 0, s>>>(ix.members, ix.m, ix.block_volume, ix.count);
  k_rope_table<<<blocks((int64_t)ix.rope_rows * ix.rope_pairs), T, 0, s>>>(
      ix.rope_rows, ix.rope_pairs, (double)g->rope_base, ix.rope);
  if (cudaGetLastError() != cudaSuccess) return PACK3D_ERR_CUDA;

  int32_t st = 0;
  if (cudaMemcpyAsync(&st, ix.status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  *out = ix;
  return st ? static_cast<pack3d_status>(st) : PACK3D_OK;
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
