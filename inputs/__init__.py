"""Seeded synthetic inputs for PACK3D attention: packings of a 3D token grid and token fields.

This module is shared by the tests, the benchmark and the smoke check. It produces *inputs*
only -- memory orders (packings) and random token values -- and holds none of the operator's
arithmetic (no RoPE, no neighbourhoods, no pooling, no softmax).

Conventions (project page "Geometry Matters in Packed 3D Attention", Chapter 1 "Every token
has two indices"; paper summary §3.1 and Table 9):
  * a grid is (Gz, Gy, Gx); the raster id of site (z, y, x) is (z*Gy + y)*Gx + x (x fastest);
  * a packing is ``perm`` with ``perm[slot] = raster id of the token stored at memory slot``;
  * the coordinate of the token at memory slot i is ``coords[i] = unravel(perm[i])``.

Packings named on the pages: raster, Morton (Z-order), block-contiguous ("raster_block":
blocks in raster order, raster order inside each block) and a seeded uniform random order.
A workload may also leave lattice sites empty (`occupancy` < 1: a seeded subset of the sites
holds tokens) and give k, v fewer heads than q (`kv_heads`); `pool2`, `summary_rope` and
`spacing` describe its summary and RoPE plan and are passed through untouched.
"""
from __future__ import annotations

import numpy as np
import torch

PACKINGS = ("raster", "morton", "raster_block", "random")


def grid_volume(grid):
    gz, gy, gx = (int(g) for g in grid)
    return gz * gy * gx


def unravel(raster_ids, grid):
    """Raster ids -> int32 coordinates [N, 3] in (z, y, x) order."""
    gz, gy, gx = (int(g) for g in grid)
    r = np.asarray(raster_ids, dtype=np.int64)
    z = r // (gy * gx)
    y = (r // gx) % gy
    x = r % gx
    return np.stack([z, y, x], axis=-1).astype(np.int32)


def _morton_code(coords):
    """Interleave the bits of (z, y, x): bit 3b = x_b, 3b+1 = y_b, 3b+2 = z_b."""
    c = np.asarray(coords, dtype=np.int64)
    code = np.zeros(len(c), dtype=np.int64)
    for b in range(21):
        code |= ((c[:, 2] >> b) & 1) << (3 * b)
        code |= ((c[:, 1] >> b) & 1) << (3 * b + 1)
        code |= ((c[:, 0] >> b) & 1) << (3 * b + 2)
    return code


def packing(kind, grid, block=(4, 4, 4), seed=1):
    """Return ``perm`` (int64 [N]): perm[slot] = raster id stored at that memory slot."""
    gz, gy, gx = (int(g) for g in grid)
    n = gz * gy * gx
    ids = np.arange(n, dtype=np.int64)
    if kind == "raster":
        return ids
    if kind == "morton":
        return ids[np.argsort(_morton_code(unravel(ids, grid)), kind="stable")]
    if kind == "raster_block":
        bz, by, bx = (int(b) for b in block)
        c = unravel(ids, grid).astype(np.int64)
        nby, nbx = -(-gy // by), -(-gx // bx)  # blocks at the far edges may be partial
        blk = ((c[:, 0] // bz) * nby + c[:, 1] // by) * nbx + c[:, 2] // bx
        inner = ((c[:, 0] % bz) * by + c[:, 1] % by) * bx + c[:, 2] % bx
        key = blk * (bz * by * bx) + inner
        return ids[np.argsort(key, kind="stable")]
    if kind == "random":
        g = torch.Generator().manual_seed(int(seed))
        return torch.randperm(n, generator=g).numpy().astype(np.int64)
    raise ValueError(f"unknown packing {kind!r}; expected one of {PACKINGS}")


def coords_of(perm, grid):
    return unravel(perm, grid)


def occupied(perm, grid, occupancy, seed=3):
    """Keep a seeded fraction of the lattice sites (the field's valid tokens): site r holds a
    token when a uniform draw for r is below `occupancy`; memory order is kept."""
    if occupancy >= 1.0:
        return np.asarray(perm)
    g = torch.Generator().manual_seed(int(seed))
    keep = (torch.rand(grid_volume(grid), generator=g) < occupancy).numpy()
    keep[np.asarray(perm)[0]] = True  # never empty
    perm = np.asarray(perm)
    return perm[keep[perm]]


def field(batch, heads, grid, d, *, qkv_std=1.0, seed=0, gen_dtype=torch.float32):
    """q, k, v [B,H,N,d] and gate logits a [B,H,N] in RASTER order, drawn in that order.

    q, k, v ~ N(0, qkv_std^2) and a ~ N(0, 1) from ``torch.Generator().manual_seed(seed)``,
    generated in float32 (CPU) as q, k, v, a.
    """
    n = grid_volume(grid)
    g = torch.Generator().manual_seed(int(seed))
    shape = (batch, heads, n, d)
    q = torch.randn(shape, generator=g, dtype=gen_dtype) * qkv_std
    k = torch.randn(shape, generator=g, dtype=gen_dtype) * qkv_std
    v = torch.randn(shape, generator=g, dtype=gen_dtype) * qkv_std
    a = torch.randn(shape[:3], generator=g, dtype=gen_dtype)
    return q, k, v, a


def upstream_grad(batch, heads, grid, d, *, seed=2):
    """dO ~ N(0,1) [B,H,N,d] in raster order (seeded, float32)."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn((batch, heads, grid_volume(grid), d), generator=g, dtype=torch.float32)


def pack(x, perm, token_dim=2):
    """Reorder a raster-order tensor into memory order: out[..., slot, ...] = x[..., perm[slot], ...]."""
    idx = torch.as_tensor(np.asarray(perm), dtype=torch.long)
    return x.index_select(token_dim, idx)


def unpack(x, perm, token_dim=2):
    """Inverse of :func:`pack`: bring a memory-order tensor back to raster order."""
    inv = np.empty(len(perm), dtype=np.int64)
    inv[np.asarray(perm)] = np.arange(len(perm), dtype=np.int64)
    return x.index_select(token_dim, torch.as_tensor(inv, dtype=torch.long))


# --- named workloads -------------------------------------------------------------------------
# Sizes follow the pages' workloads: the 8x8x8 / 2x2x2 field of the project page's "two-indices
# lab" (Chapter 1), 65,536- and 262,144-token fields (paper summary §4.3, project page
# Chapter 3 Contract 2) with 4x4x4 blocks, and the 1M-token point of the latency sweep.
WORKLOADS = {
    "tiny_8x8x8_fp32": dict(grid=(8, 8, 8), block=(2, 2, 2), batch=1, heads=1, d=48,
                            dtype="fp32", packing="raster", qkv_std=1.0, exclude_near=False),
    "field65k_bf16": dict(grid=(32, 32, 64), block=(4, 4, 4), batch=2, heads=8, d=96,
                          dtype="bf16", packing="raster_block", qkv_std=96 ** -0.5,
                          exclude_near=False),
    "field65k_repack_bf16": dict(grid=(32, 32, 64), block=(4, 4, 4), batch=2, heads=8, d=96,
                                 dtype="bf16", packing="raster", qkv_std=96 ** -0.5,
                                 exclude_near=True),
    "field262k_bf16": dict(grid=(64, 64, 64), block=(4, 4, 4), batch=1, heads=8, d=96,
                           dtype="bf16", packing="raster_block", qkv_std=1.0,
                           exclude_near=False),
    "field65k_fwdbwd_bf16": dict(grid=(32, 32, 64), block=(4, 4, 4), batch=2, heads=8, d=96,
                                 dtype="bf16", packing="raster_block", qkv_std=96 ** -0.5,
                                 exclude_near=False),
    # the pages' high-token timing point (project page Ch.9: 1M tokens, 4,096 summaries per KV
    # head): 4x4x4 blocks pooled again over 1x2x2 groups, 256 tokens per summary
    "field1m_bf16": dict(grid=(64, 128, 128), block=(4, 4, 4), pool2=(1, 2, 2), batch=1,
                         heads=8, d=96, dtype="bf16", packing="raster_block",
                         qkv_std=96 ** -0.5, exclude_near=False),
}


def make_workload(name_or_cfg, *, packing_kind=None, seed=0, perm_seed=1):
    """Build a full synthetic workload in memory order.

    Returns a dict with grid, block, perm, coords (int32 [N,3]) and q, k, v, a in memory
    order (float32 CPU tensors already rounded through the workload dtype, so that both the
    oracle and the GPU see exactly the same values).
    """
    cfg = dict(WORKLOADS[name_or_cfg]) if isinstance(name_or_cfg, str) else dict(name_or_cfg)
    kind = packing_kind or cfg["packing"]
    grid, block = tuple(cfg["grid"]), tuple(cfg["block"])
    q, k, v, a = field(cfg["batch"], cfg["heads"], grid, cfg["d"], qkv_std=cfg["qkv_std"],
                       seed=seed)
    hkv = cfg.get("kv_heads") or cfg["heads"]
    k, v = k[:, :hkv].contiguous(), v[:, :hkv].contiguous()  # GQA: the KV heads' rows
    if cfg["dtype"] == "bf16":
        q, k, v, a = (t.to(torch.bfloat16).to(torch.float32) for t in (q, k, v, a))
    perm = occupied(packing(kind, grid, block, seed=perm_seed), grid, cfg.get("occupancy", 1.0))
    cfg.setdefault("pool2", (1, 1, 1))
    cfg.setdefault("summary_rope", "token")
    cfg.setdefault("spacing", (1.0, 1.0, 1.0))
    cfg.setdefault("kv_heads", cfg["heads"])
    out = dict(cfg)
    out.update(packing=kind, perm=perm, coords=coords_of(perm, grid),
               q=pack(q, perm), k=pack(k, perm), v=pack(v, perm), a=pack(a, perm))
    return out
