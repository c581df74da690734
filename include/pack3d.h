/*
 * pack3d.h -- C ABI of the PACK3D attention operator (sm_100a).
 *
 * PACK3D ("Geometry Matters in Packed 3D Attention", Khan, Subrahmanya, Manjunath, NeurIPS
 * 2026) attends over a 3D token grid whose tokens sit in memory in an arbitrary order
 * (raster, Morton, block-contiguous, random). Each token keeps its integer grid coordinate
 * c = (z, y, x) and every operation is indexed by that coordinate, never by the memory slot
 * (project page amilworks.github.io/Pack3D, Chapter 1 and Chapter 3 Contracts 1-3). The
 * operator has four parts:
 *   - axial RoPE of q and k at c (head_dim split in three axis thirds z, y, x; base 10000);
 *   - exact softmax attention over the 3x3x3 coordinate neighbourhood (<= 27 tokens);
 *   - a global branch: rotated keys and values mean-pooled over contiguous 3D blocks into
 *     summaries, and a softmax of each query over all summaries (optionally dropping the
 *     summaries whose block meets the query's neighbourhood);
 *   - a tokenwise mixer o = g * o_local + (1 - g) * o_global, g = sigmoid(gate logit).
 *
 * Conventions shared by every call:
 *   - Tensors are dense, row-major [B, H, N, d] with N in MEMORY order (the packing);
 *     gate logits are [B, H, N]; lse outputs are float32 [B, H, N]. Keys and values may have
 *     fewer heads than queries (GQA / MQA: [B, H_kv, N, d], H_kv dividing H; query head h
 *     uses KV head h / (H / H_kv); project page Ch.3 Contract 2 "summaries per KV head",
 *     paper summary §D.1); the calls take both head counts (kv_heads 0 means H_kv = H).
 *   - Validity: a field holds N <= Gz*Gy*Gx tokens at distinct lattice sites; the sites
 *     without a token are empty (project page Ch.3 Contract 1, "coordinate offsets and
 *     validity"; Ch.4 Proposition 2). Neighbourhoods skip empty sites. Blocks tile the grid
 *     from the origin and may stick out of it at the far edges (partial blocks); a summary is
 *     the mean over its members present, and a summary with none takes part in no softmax.
 *   - Summaries (ksum, vsum) hold M summaries per (b, h_kv), ids raster over the summary
 *     grid, in SUMMARY TILES: the summaries of each (b, h_kv) are grouped in tiles of 64 (the
 *     last tile zero-padded); a tile is d/8 columns of 64 summaries x 8 consecutive
 *     elements. Element (b, h_kv, m, e) sits at element offset
 *         (((b*H_kv + h_kv)*T + m/64)*(d/8) + e/8)*512 + (m%64)*8 + e%8,   T = ceil(M/64),
 *     and a buffer takes pack3d_summary_bytes(...) bytes. A tile is exactly the tensor-core
 *     operand layout of a 64-summary chunk, so the forward moves it with one bulk copy.
 *   - dtype: PACK3D_F32 or PACK3D_BF16 for q, k, v, gate, summaries, outputs and gradients.
 *     All accumulation, softmax and logsumexp run in float32.
 *   - Pointers marked "device" must be device (or managed) memory of the current device;
 *     "host" pointers are host memory. The library never allocates device memory and never
 *     takes ownership of a pointer; all buffers belong to the caller.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are asynchronous on
 *     that stream unless stated otherwise. Argument errors are returned synchronously before
 *     any launch; a launch failure returns PACK3D_ERR_CUDA.
 *   - d (head_dim) must be 48 or 96 (a multiple of 6 is required by axial RoPE; other values
 *     return PACK3D_ERR_UNSUPPORTED).
 */
#ifndef PACK3D_H
#define PACK3D_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PACK3D_OK = 0,
  PACK3D_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent arguments */
  PACK3D_ERR_UNSUPPORTED = 2,   /* valid but not supported by this library (d, partial grid) */
  PACK3D_ERR_DUP_COORD = 3,     /* two tokens carry the same coordinate */
  PACK3D_ERR_COORD_RANGE = 4,   /* a coordinate (or raster id) lies outside the grid */
  PACK3D_ERR_ALIGN = 5,         /* a pointer is not 16-byte aligned */
  PACK3D_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up (status word) */
  PACK3D_ERR_CUDA = 7,          /* a CUDA runtime call or kernel launch failed */
  PACK3D_ERR_WORKSPACE = 8      /* caller's buffer smaller than the size query returned */
} pack3d_status;

typedef enum { PACK3D_F32 = 0, PACK3D_BF16 = 1 } pack3d_dtype;

/* attn_fwd / attn_bwd flag: drop, for each query, the summaries whose block box meets the
 * cube [c-1, c+1]^3 around the query's coordinate. */
#define PACK3D_EXCLUDE_NEAR 1u
/* attn_fwd flag: `k` holds the rotated keys R(c_j) k_j written by pack3d_summarize_rotated
 * (the local branch then gathers them without rotating). bf16 on the tensor-core path only;
 * otherwise the call returns UNSUPPORTED. */
#define PACK3D_K_ROTATED 2u

/* pack3d_geom.summary_rope: where the global branch's keys are rotated. */
#define PACK3D_ROPE_TOKEN 0   /* each key at its own coordinate, then pooled (exact; Ch.3
                                 "Rotate first, then pool", paper summary §B.5) */
#define PACK3D_ROPE_CENTRE 1  /* the unrotated keys pooled, the mean rotated once at the centre
                                 of the summary's box (the cheaper variant; Ch.3 "One block, two
                                 ways to summarize it", paper summary §B.7-§B.8) */

/* Geometry of a packed field: grid extents, block (summary) extents, RoPE plan. */
typedef struct {
  int32_t gz, gy, gx;   /* grid extents, each in [1, 1024] */
  int32_t bz, by, bx;   /* block extents, each in [1, grid extent] */
  int32_t head_dim;     /* d: 48 or 96 */
  float rope_base;      /* RoPE base per axis (10000 on the pages) */
  int32_t pz, py, px;   /* second pooling stage (note under Figure 1 of the project page): each
                           summary is the mean of the non-empty block summaries of a
                           pz x py x px group of the block grid; 0 or 1 on every axis: none.
                           Each extent in [0, 1024]. */
  int32_t summary_rope; /* PACK3D_ROPE_TOKEN or PACK3D_ROPE_CENTRE */
  float spacing[3];     /* RoPE angle of axis a is spacing[a] * c_a * theta_p: a fixed
                           anisotropic or normalised coordinate map (paper summary §B.2, §B.9);
                           0 means 1. Neighbourhoods and blocks stay on the integer lattice. */
} pack3d_geom;

/* Index tables of one packed field (one geometry, one packing). Filled by
 * pack3d_build_index; all pointers point into the caller's device buffer `buf`.
 * Coordinates are stored packed as (z << 20) | (y << 10) | x. */
typedef struct {
  pack3d_geom geom;
  int64_t n;              /* tokens present, N <= Gz*Gy*Gx */
  int64_t m;              /* summaries M the global branch attends to (second stage, if any) */
  int64_t n_blocks;       /* first-stage blocks ceil(Gz/bz)*ceil(Gy/by)*ceil(Gx/bx) */
  int32_t block_volume;   /* v = bz*by*bx */
  int32_t rope_pairs;     /* d / 6 rotation pairs per axis */
  int32_t rope_rows;      /* max(Gz, Gy, Gx): coordinates covered by the rotation table */
  int32_t group_volume;   /* first-stage blocks per summary, pz*py*px (1 without a 2nd stage) */
  int32_t sum_ext[3];     /* lattice extents (z, y, x) of a summary's box: block * group */
  int32_t sum_grid[3];    /* summaries per axis, ceil(G / sum_ext); M is their product */
  int32_t n_empty;        /* summaries with no member present */
  int32_t reserved;
  int32_t* coord;         /* device [N]      packed coordinate of the token at each slot */
  int32_t* inv;           /* device [Gz*Gy*Gx] memory slot of each raster site (-1: empty) */
  int32_t* nbr;           /* device [N, 27]  slot of c + delta_o, o = 9(dz+1)+3(dy+1)+(dx+1);
                             -1 outside the grid or at an empty site */
  int32_t* block_of;      /* device [N]      first-stage block id of each token */
  int32_t* slot_of;       /* device [N]      canonical slot inside its block (raster) */
  int32_t* members;       /* device [n_blocks, v] slot of the member at each canonical slot */
  int32_t* count;         /* device [n_blocks] members present */
  int32_t* sum_of;        /* device [N]      summary id of each token */
  int32_t* groups;        /* device [M, group_volume] first-stage block ids of each summary,
                             raster inside the group; -1 past the block grid */
  int32_t* count2;        /* device [M]      non-empty first-stage blocks of each summary */
  uint32_t* empty;        /* device [ceil(M/32)] bit m%32 of word m/32 set: summary m empty */
  float* rope;            /* device [3, rope_rows, rope_pairs, 2] (cos, sin) of
                             spacing[a] * c * theta_p for axis a */
  float* rope_c;          /* device [M, d/2, 2] (cos, sin) of the angles of each summary's box
                             centre, pair e/2 of dims (e, e+1) (summary-centre RoPE) */
  int32_t* status;        /* device [4]      status words written by kernels: [0] first error;
                             [1] empty summaries (index build); [2], [3] the work counter of
                             the bf16 rotated-key local kernel (zero between calls; calls that
                             use one index must therefore be ordered, e.g. on one stream) */
} pack3d_index;

/* Human-readable name of a status code (static string, never NULL). */
const char* pack3d_strerror(pack3d_status s);

/* Bytes of device memory pack3d_build_index needs for `n` tokens of geometry `g`
 * (0 if the geometry is invalid). Host-only; launches nothing. */
size_t pack3d_index_bytes(const pack3d_geom* g, int64_t n);

/* Build the coordinate -> slot inverse map, the 27-neighbour table, the block-membership
 * tables and the RoPE rotation table of a packed field.
 *   Project page Ch.3 Contract 1 (neighbourhoods by coordinate, not adjacency in memory),
 *   Ch.4 Proposition 2 (coordinates, edges, memberships and within-block slots travel with
 *   each token); paper summary §B.1.
 * g        host   geometry.
 * coords   device int32 [n, 3] (z, y, x) of the token at each memory slot, or NULL;
 * perm     device int64 [n] raster id (z*Gy + y)*Gx + x of the token at each slot, or NULL.
 *          Exactly one of coords / perm must be non-NULL.
 * buf      device buffer of at least pack3d_index_bytes(g, n) bytes, 256-byte aligned; it
 *          holds every table and must outlive `out`'s use.
 * out      host   filled with the table pointers and sizes.
 * n          tokens present, 1 <= n <= Gz*Gy*Gx (the other sites are empty).
 * Errors: INVALID_ARG, UNSUPPORTED (d not 48/96), WORKSPACE, ALIGN, and -- after one stream
 * synchronisation at the end of the call, which also reads the number of empty summaries --
 * DUP_COORD or COORD_RANGE detected by the kernels. */
pack3d_status pack3d_build_index(const pack3d_geom* g, const int32_t* coords,
                                 const int64_t* perm, int64_t n, void* buf, size_t buf_bytes,
                                 pack3d_index* out, void* stream);

/* Rotate-then-pool block summaries: ksum[m] = mean over members j of R(c_j) k_j and
 * vsum[m] = mean of v_j, summed in canonical-slot order (project page Ch.3 "Rotate first,
 * then pool"; paper summary §3.2, §B.5); with a second stage, the mean of the non-empty block
 * means of each group, in group order; with PACK3D_ROPE_CENTRE, the unrotated keys are
 * pooled and the mean is rotated at the centre of the summary's box.
 * k, v       device [B, H_kv, N, d] dtype (`heads` is H_kv here: summaries are per KV head);
 * ksum, vsum device summary tiles, dtype, each of pack3d_summary_bytes(idx, dtype, B, H_kv)
 *            bytes (outputs; the padding and empty summaries are zero). */
pack3d_status pack3d_summarize(const pack3d_index* idx, const void* k, const void* v,
                               int dtype, int batch, int heads, void* ksum, void* vsum,
                               void* stream);

/* As pack3d_summarize, and in the same pass writes the rotated keys
 * k_rot[b,h,j] = R(c_j) k[b,h,j] (axial RoPE of each token's coordinate, rounded to dtype).
 * The pages rotate q and k inside attention; doing it for k once here, where every key row is
 * already read, lets the local branch fetch key rows with plain row gathers.
 * k_rot      device [B, H_kv, N, d] dtype (output); must not alias k. */
pack3d_status pack3d_summarize_rotated(const pack3d_index* idx, const void* k, const void* v,
                                       int dtype, int batch, int heads, void* ksum, void* vsum,
                                       void* k_rot, void* stream);

/* PACK3D forward: local branch + global branch over (ksum, vsum) + sigmoid mixer
 * (project page Ch.3 Contracts 1-3; paper summary §3.2, §3.3, §3.5).
 * q          device [B, H, N, d] dtype;  k, v device [B, H_kv, N, d] dtype (kv_heads = H_kv,
 *            dividing H; 0 means H);  gate device [B, H, N] dtype (logits a).
 * ksum, vsum device summary tiles from pack3d_summarize of the same k, v.
 * scale      softmax scale tau (both branches); pass 1/sqrt(d) for the usual choice.
 * flags      0, or PACK3D_EXCLUDE_NEAR and/or PACK3D_K_ROTATED (k is then the k_rot of
 *            pack3d_summarize_rotated).
 * o          device [B, H, N, d] dtype (output).
 * lse_loc, lse_glob  device float32 [B, H, N] or NULL: natural-log logsumexp of each
 *            branch's logits (-inf where every summary is excluded).
 * o_loc, o_glob      device [B, H, N, d] dtype or NULL: the two normalised branch outputs
 *            (what the backward needs). A query whose summaries are all excluded has
 *            o_glob = 0. */
pack3d_status pack3d_attn_fwd(const pack3d_index* idx, const void* q, const void* k,
                              const void* v, const void* gate, const void* ksum,
                              const void* vsum, int dtype, int batch, int heads, int kv_heads,
                              float scale, uint32_t flags, void* o, float* lse_loc,
                              float* lse_glob, void* o_loc, void* o_glob, void* stream);

/* The two halves of pack3d_attn_fwd as separate calls (same kernels, same results).
 * pack3d_attn_local: the local branch alone (project page Ch.3 Contract 1; paper summary
 *   §3.5): o_loc [B, H, N, d] dtype (output, normalised) and lse_loc float32 [B, H, N] or
 *   NULL. flags: 0 or PACK3D_K_ROTATED.
 * pack3d_attn_global: the global branch over (ksum, vsum) and the sigmoid mixer
 *   o = g o_loc + (1 - g) o_glob (Ch.3 Contract 2; paper summary §3.3), given the o_loc of
 *   pack3d_attn_local; `o` may be the same buffer as o_loc (mixed in place). lse_glob and
 *   o_glob as in pack3d_attn_fwd. flags: 0 or PACK3D_EXCLUDE_NEAR.
 * Errors as pack3d_attn_fwd. */
pack3d_status pack3d_attn_local(const pack3d_index* idx, const void* q, const void* k,
                                const void* v, int dtype, int batch, int heads, int kv_heads,
                                float scale, uint32_t flags, void* o_loc, float* lse_loc,
                                void* stream);
pack3d_status pack3d_attn_global(const pack3d_index* idx, const void* q, const void* gate,
                                 const void* ksum, const void* vsum, const void* o_loc,
                                 int dtype, int batch, int heads, int kv_heads, float scale,
                                 uint32_t flags, void* o, float* lse_glob, void* o_glob,
                                 void* stream);

/* Bytes of one summary buffer (ksum or vsum) for B x H_kv heads in summary tiles (pass the
 * KV head count as `heads`). Host-only; 0 if the arguments are invalid. */
size_t pack3d_summary_bytes(const pack3d_index* idx, int dtype, int batch, int heads);

/* Bytes of device workspace pack3d_attn_bwd needs. Host-only; 0 if the arguments are invalid. */
size_t pack3d_bwd_workspace_bytes(const pack3d_index* idx, int dtype, int batch, int heads,
                                  int kv_heads);

/* PACK3D backward: gradients of sum(dO * o) through the mixer, both softmax branches, the
 * mean pooling and the axial RoPE (paper summary §3.4: the backward follows the forward's
 * streamed access pattern).
 * Inputs as in pack3d_attn_fwd plus the forward's saved o_loc, o_glob (dtype), lse_loc,
 * lse_glob (float32) and the upstream gradient dO [B, H, N, d] dtype.
 * Outputs dq [B, H, N, d], dk, dv [B, H_kv, N, d] (a KV head's gradients sum over its query
 * heads) and dgate [B, H, N], all dtype (dgate: gradient w.r.t. the gate logit).
 * workspace: device, >= pack3d_bwd_workspace_bytes bytes, 256-byte aligned; contents on entry
 * are ignored. */
pack3d_status pack3d_attn_bwd(const pack3d_index* idx, const void* q, const void* k,
                              const void* v, const void* gate, const void* ksum,
                              const void* vsum, const void* o_loc, const void* o_glob,
                              const float* lse_loc, const float* lse_glob, const void* dO,
                              int dtype, int batch, int heads, int kv_heads, float scale,
                              uint32_t flags, void* dq, void* dk, void* dv, void* dgate,
                              void* workspace, size_t workspace_bytes, void* stream);

/* Largest backward workspace pack3d_attn_bwd_noalloc can serve from its built-in buffer. */
#define PACK3D_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* pack3d_attn_bwd without a caller workspace. (The paper has no counterpart: this is a service
 * for callers that cannot allocate device memory, e.g. a host framework that owns every device
 * allocation through its own pool and forbids libraries to allocate, or a latency-critical loop
 * that cannot take cudaMalloc's implicit synchronisation.)
 * Same arguments and results as pack3d_attn_bwd, minus workspace/workspace_bytes. The scratch
 * comes from one device array of PACK3D_NOALLOC_SCRATCH_BYTES bytes inside the library, which
 * every device that loads the library keeps until the process exits; nothing is allocated.
 * Returns PACK3D_ERR_WORKSPACE when pack3d_bwd_workspace_bytes(...) exceeds that size.
 * The first call on a device (with that device current) looks the array's address up once
 * (cudaGetSymbolAddress); make that first call before any stream capture on the device.
 * All calls share the array and it keeps the last call's contents (the kernels overwrite all
 * they read); calls that overlap on the GPU race on it, so order them on one stream. */
pack3d_status pack3d_attn_bwd_noalloc(const pack3d_index* idx, const void* q, const void* k,
                                      const void* v, const void* gate, const void* ksum,
                                      const void* vsum, const void* o_loc, const void* o_glob,
                                      const float* lse_loc, const float* lse_glob,
                                      const void* dO, int dtype, int batch, int heads,
                                      int kv_heads, float scale, uint32_t flags, void* dq,
                                      void* dk, void* dv, void* dgate, void* stream);

/* Reads (after synchronising `stream`) and clears the index's device status word: OK, or
 * the first device-detected error (DUP_COORD, COORD_RANGE, TIMEOUT). */
pack3d_status pack3d_device_status(const pack3d_index* idx, void* stream);

/* Kernel launches issued by the last pack3d_summarize / attn_fwd / attn_bwd call made on
 * this host thread (for launch accounting). */
int pack3d_last_launch_count(void);

/* TESTING HOOK (not part of the operator; the paper has no counterpart). Every device-side
 * wait of the tensor-core kernels (a warp waiting for a copy, an MMA or another warp) gives up
 * after a budget of SM clock cycles: it records PACK3D_ERR_TIMEOUT in the index's status word
 * (read it with pack3d_device_status), the kernel drains its in-flight copies and MMAs, frees
 * its tensor memory and returns, so the CUDA context stays usable. This sets the budget used
 * by the launches that follow, process-wide (cycles <= 0 restores the default of 4e9 cycles)
 * and returns the previous value. A tiny budget makes the next launches time out on purpose;
 * it exists so that tests can exercise that path without faulting or hanging a GPU. */
long long pack3d_testing_set_wait_budget(long long cycles);

#ifdef __cplusplus
}
#endif

#endif /* PACK3D_H */
