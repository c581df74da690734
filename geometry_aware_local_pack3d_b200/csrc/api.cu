// C ABI of the PACK3D operator: argument checks and dispatch to the kernels.
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "launch.h"

namespace p3d {
thread_local int g_launches = 0;

cudaError_t summarize_dispatch(const pack3d_index& ix, const void* k, const void* v, int dtype,
                               int64_t bh, void* ksum, void* vsum, void* krot, cudaStream_t s);
cudaError_t bwd_simt_dispatch(const pack3d_index& ix, const void* q, const void* k,
                              const void* v, const void* gate, const void* ksum,
                              const void* vsum, const void* o_loc, const void* o_glob,
                              const float* lse_loc, const float* lse_glob, const void* dO,
                              int dtype, int64_t bh, int kv_group, float scale, int excl,
                              void* dq, void* dk, void* dv, void* dgate, void* ws, bool tc,
                              cudaStream_t s);
size_t bwd_workspace_bytes(const pack3d_index& ix, int64_t bh, int dtype, bool tc,
                           int kv_group);
cudaError_t global_simt_dispatch(const pack3d_index& ix, const void* q, const void* gate,
                                 const void* ksum, const void* vsum, const void* o_loc,
                                 int dtype, int64_t bh, int kv_group, float scale, int excl,
                                 void* o, float* lse_glob, void* o_glob, cudaStream_t s);
cudaError_t local_simt_dispatch(const pack3d_index& ix, const void* q, const void* k,
                                const void* v, int dtype, int64_t bh, int kv_group, float scale,
                                void* o_loc, float* lse_loc, cudaStream_t s);
cudaError_t local_tma_dispatch(const pack3d_index& ix, const void* q, const void* k,
                               const void* v, int64_t bh, int kv_group, float scale,
                               bool k_rotated, void* o_loc, float* lse_loc, cudaStream_t s);
pack3d_status check_common(const pack3d_index* idx, int dtype, int batch, int heads);
pack3d_status kv_group_of(int heads, int kv_heads, int* group);
cudaError_t global_tc_dispatch(const pack3d_index& ix, const void* q, const void* gate,
                               const void* ksum, const void* vsum, const void* o_loc, int64_t bh,
                               int kv_group, float scale, int excl, void* o, float* lse_glob,
                               void* o_glob, cudaStream_t s);
}  // namespace p3d

using namespace p3d;

// Checks shared by every operator call (also used by the no-alloc backward).
pack3d_status p3d::check_common(const pack3d_index* idx, int dtype, int batch, int heads) {
  if (!idx || !idx->coord || !idx->nbr || !idx->members || !idx->rope || !idx->sum_of ||
      !idx->groups || !idx->count2 || !idx->empty || !idx->rope_c)
    return PACK3D_ERR_INVALID_ARG;
  if (dtype != PACK3D_F32 && dtype != PACK3D_BF16) return PACK3D_ERR_INVALID_ARG;
  if (batch <= 0 || heads <= 0) return PACK3D_ERR_INVALID_ARG;
  if ((int64_t)batch * heads > 65535) return PACK3D_ERR_UNSUPPORTED;
  if (idx->geom.head_dim != 48 && idx->geom.head_dim != 96) return PACK3D_ERR_UNSUPPORTED;
  return PACK3D_OK;
}

// Query heads per KV head: kv_heads 0 means one KV head per query head; otherwise it must
// divide the query heads.
pack3d_status p3d::kv_group_of(int heads, int kv_heads, int* group) {
  if (kv_heads == 0) kv_heads = heads;
  if (kv_heads < 0 || kv_heads > heads || heads % kv_heads) return PACK3D_ERR_INVALID_ARG;
  *group = heads / kv_heads;
  return PACK3D_OK;
}

namespace {
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

pack3d_status check_rows(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs) {
    if (!p) return PACK3D_ERR_INVALID_ARG;
    if (!aligned16(p)) return PACK3D_ERR_ALIGN;
  }
  return PACK3D_OK;
}

pack3d_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PACK3D_OK : PACK3D_ERR_CUDA; }

// bf16 runs on tcgen05 tensor cores; float32 stays on CUDA cores for the 1e-4 bar (no TF32)
bool tensor_path(int dtype) { return dtype == PACK3D_BF16; }
}  // namespace

extern "C" const char* pack3d_strerror(pack3d_status s) {
  switch (s) {
    case PACK3D_OK: return "ok";
    case PACK3D_ERR_INVALID_ARG: return "invalid argument";
    case PACK3D_ERR_UNSUPPORTED: return "unsupported configuration";
    case PACK3D_ERR_DUP_COORD: return "two tokens carry the same coordinate";
    case PACK3D_ERR_COORD_RANGE: return "coordinate outside the grid";
    case PACK3D_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PACK3D_ERR_TIMEOUT: return "device-side wait timed out";
    case PACK3D_ERR_CUDA: return "CUDA runtime error";
    case PACK3D_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

extern "C" int pack3d_last_launch_count(void) { return g_launches; }

extern "C" long long pack3d_testing_set_wait_budget(long long cycles) {
  return wait_budget_store().exchange(cycles > 0 ? cycles : kDefaultWaitBudget);
}

extern "C" pack3d_status pack3d_summarize(const pack3d_index* idx, const void* k, const void* v,
                                          int dtype, int batch, int heads, void* ksum,
                                          void* vsum, void* stream) {
  reset_launches();
  pack3d_status st = check_common(idx, dtype, batch, heads);
  if (st != PACK3D_OK) return st;
  if ((st = check_rows({k, v, ksum, vsum})) != PACK3D_OK) return st;
  return cuda_status(summarize_dispatch(*idx, k, v, dtype, (int64_t)batch * heads, ksum, vsum,
                                        nullptr, static_cast<cudaStream_t>(stream)));
}

extern "C" pack3d_status pack3d_summarize_rotated(const pack3d_index* idx, const void* k,
                                                  const void* v, int dtype, int batch, int heads,
                                                  void* ksum, void* vsum, void* k_rot,
                                                  void* stream) {
  reset_launches();
  pack3d_status st = check_common(idx, dtype, batch, heads);
  if (st != PACK3D_OK) return st;
  if ((st = check_rows({k, v, ksum, vsum, k_rot})) != PACK3D_OK) return st;
  if (k_rot == k) return PACK3D_ERR_INVALID_ARG;  // other members of a block still read k
  return cuda_status(summarize_dispatch(*idx, k, v, dtype, (int64_t)batch * heads, ksum, vsum,
                                        k_rot, static_cast<cudaStream_t>(stream)));
}

namespace {
// local branch: o_loc (normalised) and lse_loc
pack3d_status run_local(const pack3d_index* idx, const void* q, const void* k, const void* v,
                        int dtype, int64_t bh, int group, float scale, bool k_rotated,
                        void* o_loc, float* lse_loc, cudaStream_t s) {
  if (tensor_path(dtype))
    return cuda_status(
        local_tma_dispatch(*idx, q, k, v, bh, group, scale, k_rotated, o_loc, lse_loc, s));
  return cuda_status(
      local_simt_dispatch(*idx, q, k, v, dtype, bh, group, scale, o_loc, lse_loc, s));
}

// global branch over the summaries + the sigmoid mixer with a given o_loc (o may alias it)
pack3d_status run_global(const pack3d_index* idx, const void* q, const void* gate,
                         const void* ksum, const void* vsum, const void* o_loc, int dtype,
                         int64_t bh, int group, float scale, int excl, void* o, float* lse_glob,
                         void* o_glob, cudaStream_t s) {
  if (tensor_path(dtype))
    return cuda_status(global_tc_dispatch(*idx, q, gate, ksum, vsum, o_loc, bh, group, scale,
                                          excl, o, lse_glob, o_glob, s));
  return cuda_status(global_simt_dispatch(*idx, q, gate, ksum, vsum, o_loc, dtype, bh, group,
                                          scale, excl, o, lse_glob, o_glob, s));
}

pack3d_status check_flags(int dtype, uint32_t flags, uint32_t allowed) {
  if (flags & ~allowed) return PACK3D_ERR_INVALID_ARG;
  if ((flags & PACK3D_K_ROTATED) && !tensor_path(dtype)) return PACK3D_ERR_UNSUPPORTED;
  return PACK3D_OK;
}
}  // namespace

extern "C" pack3d_status pack3d_attn_fwd(const pack3d_index* idx, const void* q, const void* k,
                                         const void* v, const void* gate, const void* ksum,
                                         const void* vsum, int dtype, int batch, int heads,
                                         int kv_heads, float scale, uint32_t flags, void* o,
                                         float* lse_loc, float* lse_glob, void* o_loc,
                                         void* o_glob, void* stream) {
  reset_launches();
  pack3d_status st = check_common(idx, dtype, batch, heads);
  if (st != PACK3D_OK) return st;
  int group = 1;
  if ((st = kv_group_of(heads, kv_heads, &group)) != PACK3D_OK) return st;
  if ((st = check_rows({q, k, v, ksum, vsum, o})) != PACK3D_OK) return st;
  if (!gate) return PACK3D_ERR_INVALID_ARG;
  if ((o_loc && !aligned16(o_loc)) || (o_glob && !aligned16(o_glob))) return PACK3D_ERR_ALIGN;
  if (!(scale > 0.f)) return PACK3D_ERR_INVALID_ARG;
  if ((st = check_flags(dtype, flags, PACK3D_EXCLUDE_NEAR | PACK3D_K_ROTATED)) != PACK3D_OK)
    return st;
  const int64_t bh = (int64_t)batch * heads;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // local branch first (its normalised output goes to o_loc, or to o until it is mixed), then
  // the global branch with the mixer in its epilogue
  void* ol = o_loc ? o_loc : o;
  st = run_local(idx, q, k, v, dtype, bh, group, scale, (flags & PACK3D_K_ROTATED) != 0, ol,
                 lse_loc, s);
  if (st != PACK3D_OK) return st;
  return run_global(idx, q, gate, ksum, vsum, ol, dtype, bh, group, scale,
                    (flags & PACK3D_EXCLUDE_NEAR) ? 1 : 0, o, lse_glob, o_glob, s);
}

extern "C" pack3d_status pack3d_attn_local(const pack3d_index* idx, const void* q, const void* k,
                                           const void* v, int dtype, int batch, int heads,
                                           int kv_heads, float scale, uint32_t flags,
                                           void* o_loc, float* lse_loc, void* stream) {
  reset_launches();
  pack3d_status st = check_common(idx, dtype, batch, heads);
  if (st != PACK3D_OK) return st;
  int group = 1;
  if ((st = kv_group_of(heads, kv_heads, &group)) != PACK3D_OK) return st;
  if ((st = check_rows({q, k, v, o_loc})) != PACK3D_OK) return st;
  if (!(scale > 0.f)) return PACK3D_ERR_INVALID_ARG;
  if ((st = check_flags(dtype, flags, PACK3D_K_ROTATED)) != PACK3D_OK) return st;
  return run_local(idx, q, k, v, dtype, (int64_t)batch * heads, group, scale,
                   (flags & PACK3D_K_ROTATED) != 0, o_loc, lse_loc,
                   static_cast<cudaStream_t>(stream));
}

extern "C" pack3d_status pack3d_attn_global(const pack3d_index* idx, const void* q,
                                            const void* gate, const void* ksum,
                                            const void* vsum, const void* o_loc, int dtype,
                                            int batch, int heads, int kv_heads, float scale,
                                            uint32_t flags, void* o, float* lse_glob,
                                            void* o_glob, void* stream) {
  reset_launches();
  pack3d_status st = check_common(idx, dtype, batch, heads);
  if (st != PACK3D_OK) return st;
  int group = 1;
  if ((st = kv_group_of(heads, kv_heads, &group)) != PACK3D_OK) return st;
  if ((st = check_rows({q, ksum, vsum, o_loc, o})) != PACK3D_OK) return st;
  if (!gate) return PACK3D_ERR_INVALID_ARG;
  if (o_glob && !aligned16(o_glob)) return PACK3D_ERR_ALIGN;
  if (!(scale > 0.f)) return PACK3D_ERR_INVALID_ARG;
  if ((st = check_flags(dtype, flags, PACK3D_EXCLUDE_NEAR)) != PACK3D_OK) return st;
  return run_global(idx, q, gate, ksum, vsum, o_loc, dtype, (int64_t)batch * heads, group,
                    scale, (flags & PACK3D_EXCLUDE_NEAR) ? 1 : 0, o, lse_glob, o_glob,
                    static_cast<cudaStream_t>(stream));
}

extern "C" size_t pack3d_summary_bytes(const pack3d_index* idx, int dtype, int batch,
                                       int heads) {
  if (check_common(idx, dtype, batch, heads) != PACK3D_OK) return 0;
  const size_t elem = dtype == PACK3D_BF16 ? 2 : 4;
  return (size_t)batch * heads * (size_t)sum_tiles(idx->m) * 64 * idx->geom.head_dim * elem;
}

extern "C" size_t pack3d_bwd_workspace_bytes(const pack3d_index* idx, int dtype, int batch,
                                             int heads, int kv_heads) {
  int group = 1;
  if (check_common(idx, dtype, batch, heads) != PACK3D_OK ||
      kv_group_of(heads, kv_heads, &group) != PACK3D_OK)
    return 0;
  return bwd_workspace_bytes(*idx, (int64_t)batch * heads, dtype, tensor_path(dtype), group);
}

extern "C" pack3d_status pack3d_attn_bwd(const pack3d_index* idx, const void* q, const void* k,
                                         const void* v, const void* gate, const void* ksum,
                                         const void* vsum, const void* o_loc,
                                         const void* o_glob, const float* lse_loc,
                                         const float* lse_glob, const void* dO, int dtype,
                                         int batch, int heads, int kv_heads, float scale,
                                         uint32_t flags, void* dq, void* dk, void* dv,
                                         void* dgate, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  reset_launches();
  pack3d_status st = check_common(idx, dtype, batch, heads);
  if (st != PACK3D_OK) return st;
  int group = 1;
  if ((st = kv_group_of(heads, kv_heads, &group)) != PACK3D_OK) return st;
  if ((st = check_rows({q, k, v, ksum, vsum, o_loc, o_glob, dO, dq, dk, dv})) != PACK3D_OK)
    return st;
  if (!gate || !dgate || !lse_loc || !lse_glob || !workspace) return PACK3D_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255) return PACK3D_ERR_ALIGN;
  if (!(scale > 0.f) || (flags & ~PACK3D_EXCLUDE_NEAR)) return PACK3D_ERR_INVALID_ARG;
  const int64_t bh = (int64_t)batch * heads;
  const bool tc = tensor_path(dtype);
  if (workspace_bytes < bwd_workspace_bytes(*idx, bh, dtype, tc, group))
    return PACK3D_ERR_WORKSPACE;
  const int excl = (flags & PACK3D_EXCLUDE_NEAR) ? 1 : 0;
  return cuda_status(bwd_simt_dispatch(*idx, q, k, v, gate, ksum, vsum, o_loc, o_glob, lse_loc,
                                       lse_glob, dO, dtype, bh, group, scale, excl, dq, dk, dv,
                                       dgate, workspace, tc,
                                       static_cast<cudaStream_t>(stream)));
}
