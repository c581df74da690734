"""PACK3D attention -- plain CPU oracle in float64 (numpy).

TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module. It shares no code with the CUDA path: it builds its own index tables,
rotation angles, neighbourhoods, summaries and softmaxes directly from the definitions on the
pages, step by step, with no blocking, fusion or reordering.

Sources (web pages about "Geometry Matters in Packed 3D Attention", Khan, Subrahmanya,
Manjunath, NeurIPS 2026):
  [site]    project page amilworks.github.io/Pack3D -- Chapter 1 (two indices), Chapter 3
            (Contracts 1-3, "A logit that only sees displacement", "Rotate first, then pool"),
            Chapter 4 (Proposition 2), Chapter 10 (repack test).
  [summary] paperlayer.ai summary -- §3.1, §3.2, §3.3, §3.5, §B.1-§B.5, §B.10.

Readings taken where the pages are silent (equations were lost in extraction):
  * axial RoPE: head_dim d split in three equal thirds for axes (z, y, x) in that order; in each
    third (size d_a = d/3) pair p rotates dims (2p, 2p+1) by phi = c_axis * theta_p with
    theta_p = base^(-2p/d_a), base 10000; (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos).
    q and k are rotated, v is not ([site] Ch.3 Contract 3).  -- parity unpinned as to the
    convention itself: every invariant the pages state holds under any consistent choice.
  * neighbourhood: the 3x3x3 coordinate cube around the query, the query included (at most 27
    tokens, fewer at the volume border) ([site] Ch.3 Contract 1); offsets in the order
    o = 9(dz+1) + 3(dy+1) + (dx+1).
  * blocks: contiguous bz x by x bx boxes, block id raster over the block grid, canonical slot
    raster inside the block ([site] Ch.4); summaries are uniform means of the rotated keys and
    of the values of the members present ([summary] §3.2, §B.5).
  * softmax scale tau (default 1/sqrt(d)) for both branches.
  * exclude_near: a summary is dropped for query i when its block box meets the cube
    [c_i - 1, c_i + 1]^3.  A query with every summary dropped gets o_glob = 0, lse = -inf.
  * mixer: g = sigmoid(a), o = g * o_loc + (1 - g) * o_glob ([summary] §3.3).
  * validity ([site] Ch.3 Contract 1 "offsets and validity", Ch.4 Prop. 2; the sparse field
    view of Figure 1): a field may leave lattice sites empty; the tokens present are the valid
    ones. Neighbourhoods skip empty sites, blocks at the grid's far edges may be partial, and a
    summary is the mean over its members present; a summary with no member takes part in no
    softmax.
  * second pooling stage ([site] note under Figure 1: the reported models add a second pooling
    stage; Ch.3 Contract 2 and Ch.9: 1,024 / 4,096 summaries per KV head at 262,144 / 1M
    tokens): the first-stage block summaries are grouped in contiguous pz x py x px boxes of
    the block grid, and a second-stage summary is the uniform mean of the non-empty
    first-stage summaries of its group. The global branch attends to the second-stage
    summaries; a summary's box (for exclude_near and the summary centre) is its group's box.
  * coordinate maps ([summary] §B.2, §B.9: the results hold for fixed anisotropic or
    normalized coordinate maps): RoPE angles use s_axis * c_axis with a fixed per-axis scale s
    (1 by default); neighbourhoods and blocks stay on the integer lattice.
  * summary-centre RoPE ([site] Ch.3 "One block, two ways to summarize it"; [summary] §B.7,
    §B.8): the cheaper variant pools the unrotated keys and rotates the pooled key once at the
    centre of the summary's box (clipped to the grid), a possibly half-integer coordinate.
  * GQA / MQA ([site] Ch.3 Contract 2 "summaries per KV head"; [summary] §D.1): k and v may
    have H_kv heads, H_kv dividing the H query heads; query head h uses KV head h // (H/H_kv),
    both for its local keys and for its summaries, which are computed per KV head.
"""
from __future__ import annotations

import math

import numpy as np

# Offset order o = 9(dz+1) + 3(dy+1) + (dx+1): dz outermost, dx innermost.
OFFSETS = tuple((dz, dy, dx) for dz in (-1, 0, 1) for dy in (-1, 0, 1) for dx in (-1, 0, 1))


class OracleIndexError(ValueError):
    pass


# ---------------------------------------------------------------------------------------------
# Geometry: inverse map, neighbour table, block tables ([site] Ch.3 Contract 1, Ch.4 Prop. 2;
# [summary] §B.1: neighbourhoods and blocks are defined on the lattice, not on memory order).
# ---------------------------------------------------------------------------------------------
def _ceil_div(a, b):
    return -(-int(a) // int(b))


def build_index(coords, grid, block, pool2=(1, 1, 1), nbr_rows=None):
    """Index tables of a packed field, built by looping over tokens.

    coords: int [N, 3] -- (z, y, x) of the token at memory slot i; N may be smaller than the
    number of lattice sites (the sites without a token are empty). Blocks tile the grid from
    the origin; those at the far edges may stick out of it.
    pool2: extents of the second pooling stage's groups over the block grid ((1, 1, 1): none).
    nbr_rows: fill the neighbour table for these memory slots only (the other rows stay -1),
    for fields too large to loop over every token's neighbourhood in Python.
    Returns dict(inv, nbr, block_of, slot_of, members, count, n_blocks, block_volume,
    groups, count2, sum_of, n_summaries, summary_block).
    """
    coords = np.asarray(coords, dtype=np.int64).reshape(-1, 3)
    gz, gy, gx = (int(g) for g in grid)
    bz, by, bx = (int(b) for b in block)
    n = len(coords)
    inv = np.full(gz * gy * gx, -1, dtype=np.int64)
    for i in range(n):
        z, y, x = (int(t) for t in coords[i])
        if not (0 <= z < gz and 0 <= y < gy and 0 <= x < gx):
            raise OracleIndexError(f"coordinate {(z, y, x)} outside the grid")
        r = (z * gy + y) * gx + x
        if inv[r] != -1:
            raise OracleIndexError(f"two tokens at coordinate {(z, y, x)}")
        inv[r] = i

    nbr = np.full((n, 27), -1, dtype=np.int64)
    for i in (range(n) if nbr_rows is None else (int(r) for r in nbr_rows)):
        z, y, x = (int(t) for t in coords[i])
        for o, (dz, dy, dx) in enumerate(OFFSETS):
            zz, yy, xx = z + dz, y + dy, x + dx
            if 0 <= zz < gz and 0 <= yy < gy and 0 <= xx < gx:
                nbr[i, o] = inv[(zz * gy + yy) * gx + xx]  # -1 at an empty site

    nbz, nby, nbx = _ceil_div(gz, bz), _ceil_div(gy, by), _ceil_div(gx, bx)
    n_blocks, vol = nbz * nby * nbx, bz * by * bx
    block_of = np.empty(n, dtype=np.int64)
    slot_of = np.empty(n, dtype=np.int64)
    members = np.full((n_blocks, vol), -1, dtype=np.int64)
    for i in range(n):
        z, y, x = (int(t) for t in coords[i])
        block_of[i] = ((z // bz) * nby + y // by) * nbx + x // bx
        slot_of[i] = ((z % bz) * by + y % by) * bx + x % bx
        members[block_of[i], slot_of[i]] = i
    count = (members >= 0).sum(axis=1)

    # second stage: group (nz, ny, nx) holds blocks (nz*pz + a, ny*py + b, nx*px + c), listed
    # raster inside the group; -1 past the block grid
    pz, py, px = (int(t) for t in pool2)
    ngz, ngy, ngx = _ceil_div(nbz, pz), _ceil_div(nby, py), _ceil_div(nbx, px)
    n_sum = ngz * ngy * ngx
    groups = np.full((n_sum, pz * py * px), -1, dtype=np.int64)
    for m in range(n_blocks):
        mz, my, mx = m // (nby * nbx), (m // nbx) % nby, m % nbx
        gid = ((mz // pz) * ngy + my // py) * ngx + mx // px
        gslot = ((mz % pz) * py + my % py) * px + mx % px
        groups[gid, gslot] = m
    count2 = np.array([sum(1 for m in groups[t] if m >= 0 and count[m] > 0)
                       for t in range(n_sum)], dtype=np.int64)
    group_of_block = np.empty(n_blocks, dtype=np.int64)
    for t in range(n_sum):
        for m in groups[t]:
            if m >= 0:
                group_of_block[m] = t
    sum_of = group_of_block[block_of] if n else np.zeros(0, dtype=np.int64)
    return dict(inv=inv, nbr=nbr, block_of=block_of, slot_of=slot_of, members=members,
                count=count, n_blocks=n_blocks, block_volume=vol, groups=groups, count2=count2,
                sum_of=sum_of, n_summaries=n_sum, pool2=(pz, py, px),
                summary_block=(bz * pz, by * py, bx * px))


def block_boxes(grid, block):
    """Inclusive [lo, hi] box of the lattice sites of every block (clipped to the grid), block
    ids in raster order over the block grid."""
    gz, gy, gx = (int(g) for g in grid)
    bz, by, bx = (int(b) for b in block)
    boxes = []
    for mz in range(_ceil_div(gz, bz)):
        for my in range(_ceil_div(gy, by)):
            for mx in range(_ceil_div(gx, bx)):
                lo = (mz * bz, my * by, mx * bx)
                hi = (min(lo[0] + bz, gz) - 1, min(lo[1] + by, gy) - 1, min(lo[2] + bx, gx) - 1)
                boxes.append((lo, hi))
    return boxes


def summary_boxes(grid, block, pool2=(1, 1, 1)):
    """Box of every summary: a group of pz x py x px blocks covers the sites of one box of
    extents block * pool2 (clipped to the grid), in the same raster order as the groups."""
    return block_boxes(grid, tuple(int(b) * int(p) for b, p in zip(block, pool2)))


def summary_centres(grid, block, pool2=(1, 1, 1)):
    """float [M, 3]: centre of each summary's box, (lo + hi) / 2 per axis."""
    return np.array([[(lo[a] + hi[a]) / 2.0 for a in range(3)]
                     for lo, hi in summary_boxes(grid, block, pool2)], dtype=np.float64)


def excluded_summaries(coords, grid, block, pool2=(1, 1, 1)):
    """bool [N, M]: True where summary m's box meets the query's cube [c-1, c+1]^3."""
    coords = np.asarray(coords, dtype=np.int64)
    boxes = summary_boxes(grid, block, pool2)
    lo = np.array([b[0] for b in boxes])  # [M, 3]
    hi = np.array([b[1] for b in boxes])
    c = coords[:, None, :]
    meets = (lo[None] <= c + 1) & (hi[None] >= c - 1)
    return meets.all(axis=-1)


# ---------------------------------------------------------------------------------------------
# Axial RoPE ([site] Ch.3 Contract 3 and "A logit that only sees displacement"; [summary] §B.2).
# ---------------------------------------------------------------------------------------------
def rope_theta(d, base=10000.0):
    if d % 6:
        raise ValueError("axial RoPE needs head_dim divisible by 6")
    da = d // 3
    return np.array([base ** (-2.0 * p / da) for p in range(da // 2)], dtype=np.float64)


def rope(x, coords, base=10000.0, spacing=None):
    """Rotate x [..., N, d] by the axial rotation R(c_i) of each token's coordinate; with a
    per-axis scale `spacing` the angle of axis a is spacing[a] * c_a * theta_p."""
    x = np.asarray(x, dtype=np.float64)
    coords = np.asarray(coords, dtype=np.float64).reshape(-1, 3)
    if spacing is not None:
        coords = coords * np.asarray(spacing, dtype=np.float64)[None, :]
    d = x.shape[-1]
    da = d // 3
    theta = rope_theta(d, base)
    out = np.empty_like(x)
    for axis in range(3):  # thirds: z, y, x
        phi = coords[:, axis][:, None] * theta[None, :]  # [N, da/2]
        cos, sin = np.cos(phi), np.sin(phi)
        e = slice(axis * da, (axis + 1) * da, 2)
        od = slice(axis * da + 1, (axis + 1) * da, 2)
        x0, x1 = x[..., e], x[..., od]
        out[..., e] = x0 * cos - x1 * sin
        out[..., od] = x0 * sin + x1 * cos
    return out


def rope_inverse(x, coords, base=10000.0, spacing=None):
    """R(c)^T x: rotations are orthogonal, so the transpose is the rotation by -c."""
    return rope(x, -np.asarray(coords, dtype=np.float64), base, spacing)


# ---------------------------------------------------------------------------------------------
# Branches.
# ---------------------------------------------------------------------------------------------
def _softmax_rows(s):
    """Row softmax of s [..., K] with -inf entries; returns (p, lse). All -inf -> p=0, lse=-inf."""
    m = np.max(s, axis=-1, keepdims=True)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    e = np.where(np.isfinite(s), np.exp(s - m_safe), 0.0)
    l = e.sum(axis=-1, keepdims=True)
    p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
    lse = np.where(l[..., 0] > 0, (m_safe + np.log(np.where(l > 0, l, 1.0)))[..., 0], -np.inf)
    return p, lse


def local_branch(qr, kr, v, nbr, tau, rows=None):
    """Exact softmax attention over each query's coordinate neighbourhood ([site] Ch.3 Contract 1).

    qr, kr: rotated q, k [B,H,N,d]; v [B,H,N,d]; nbr [N,27] (-1 = no token).
    Returns o_loc [B,H,R,d], lse_loc [B,H,R] for the requested rows (default all).
    """
    rows = np.arange(qr.shape[2]) if rows is None else np.asarray(rows)
    B, H, _, d = qr.shape
    o = np.zeros((B, H, len(rows), d))
    lse = np.zeros((B, H, len(rows)))
    for r, i in enumerate(rows):
        js = [int(j) for j in nbr[i] if j >= 0]  # offset order
        s = np.einsum("bhd,bhjd->bhj", qr[:, :, i], kr[:, :, js]) * tau
        p, l = _softmax_rows(s)
        o[:, :, r] = np.einsum("bhj,bhjd->bhd", p, v[:, :, js])
        lse[:, :, r] = l
    return o, lse


def summaries(kr, v, members, groups=None):
    """Block summaries: uniform means over each block's members present, summed in
    canonical-slot order; then, with `groups`, the second stage: the uniform mean of the
    non-empty first-stage summaries of each group, in group-slot order. Empty summaries are 0.

    Rotate-then-pool: the keys are already rotated at their own coordinates ([site] Ch.3
    "Rotate first, then pool"; [summary] §B.5). Values are not rotated.
    """
    B, H, _, d = kr.shape
    M, vol = members.shape
    ks = np.zeros((B, H, M, d))
    vs = np.zeros((B, H, M, d))
    cnt = np.zeros(M)
    for s in range(vol):
        idx = members[:, s]
        ok = idx >= 0
        ks[:, :, ok] += kr[:, :, idx[ok]]
        vs[:, :, ok] += v[:, :, idx[ok]]
        cnt += ok
    nz = cnt > 0
    ks[:, :, nz] /= cnt[nz][:, None]
    vs[:, :, nz] /= cnt[nz][:, None]
    if groups is None:
        return ks, vs
    M2, gv = groups.shape
    ks2 = np.zeros((B, H, M2, d))
    vs2 = np.zeros((B, H, M2, d))
    cnt2 = np.zeros(M2)
    for t in range(gv):
        m = groups[:, t]
        ok = m >= 0
        ok[ok] = nz[m[ok]]  # empty first-stage summaries are skipped
        ks2[:, :, ok] += ks[:, :, m[ok]]
        vs2[:, :, ok] += vs[:, :, m[ok]]
        cnt2 += ok
    nz2 = cnt2 > 0
    ks2[:, :, nz2] /= cnt2[nz2][:, None]
    vs2[:, :, nz2] /= cnt2[nz2][:, None]
    return ks2, vs2


def global_branch(qr, ksum, vsum, tau, excluded=None, rows=None):
    """Softmax of every query over all summaries ([site] Ch.3 Contract 2; [summary] §3.5).

    excluded: optional bool [N, M] (True = summary dropped for that query); a summary with no
    member present is passed as dropped for every query.
    """
    rows = np.arange(qr.shape[2]) if rows is None else np.asarray(rows)
    B, H, _, d = qr.shape
    o = np.zeros((B, H, len(rows), d))
    lse = np.zeros((B, H, len(rows)))
    for c0 in range(0, len(rows), 4096):  # rows are independent; chunking only bounds memory
        rr = rows[c0:c0 + 4096]
        s = np.einsum("bhrd,bhmd->bhrm", qr[:, :, rr], ksum) * tau
        if excluded is not None:
            s = np.where(excluded[rr][None, None], -np.inf, s)
        p, l = _softmax_rows(s)
        o[:, :, c0:c0 + len(rr)] = np.einsum("bhrm,bhmd->bhrd", p, vsum)
        lse[:, :, c0:c0 + len(rr)] = l
    return o, lse


def sigmoid(a):
    a = np.asarray(a, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-a))


def mixer(o_loc, o_glob, a):
    """o = g * o_loc + (1 - g) * o_glob with g = sigmoid(a) per token and head ([summary] §3.3)."""
    g = sigmoid(a)[..., None]
    return g * o_loc + (1.0 - g) * o_glob


# ---------------------------------------------------------------------------------------------
# Whole operator.
# ---------------------------------------------------------------------------------------------
def _heads(q, k):
    """GQA group size: query head h uses KV head h // G."""
    H, Hkv = q.shape[1], k.shape[1]
    if H % Hkv:
        raise ValueError("the KV heads must divide the query heads")
    return H // Hkv


def _dropped(idx, coords, grid, block, exclude_near):
    """bool [N, M] or None: summaries outside each query's softmax (exclude_near, and every
    summary with no member present)."""
    empty = idx["count2"] == 0
    ex = excluded_summaries(coords, grid, block, idx["pool2"]) if exclude_near else None
    if empty.any():
        e = np.broadcast_to(empty[None, :], (len(np.asarray(coords).reshape(-1, 3)), len(empty)))
        ex = e.copy() if ex is None else (ex | e)
    return ex


def forward(q, k, v, a, coords, grid, block, *, exclude_near=False, tau=None, base=10000.0,
            rope_coords=None, index=None, rows=None, pool2=(1, 1, 1), spacing=None,
            summary_rope="token"):
    """PACK3D forward in float64.

    q [B,H,N,d], k, v [B,H_kv,N,d] (H_kv divides H), a [B,H,N], coords int [N,3] (memory
    order). ``rope_coords`` overrides the coordinates used by RoPE only (for the translation
    and negative-control checks). ``rows`` restricts the outputs to some query rows (summaries
    are always computed in full). ``pool2``: second pooling stage; ``spacing``: per-axis
    coordinate scale of RoPE; ``summary_rope``: "token" (rotate each key, then pool) or
    "centre" (pool the unrotated keys, rotate once at the summary's centre).
    """
    q, k, v, a = (np.asarray(t, dtype=np.float64) for t in (q, k, v, a))
    d = q.shape[-1]
    G = _heads(q, k)
    tau = 1.0 / math.sqrt(d) if tau is None else float(tau)
    idx = index if index is not None else build_index(coords, grid, block, pool2)
    groups = idx["groups"] if tuple(idx["pool2"]) != (1, 1, 1) else None
    rc = coords if rope_coords is None else rope_coords
    qr, kr = rope(q, rc, base, spacing), rope(k, rc, base, spacing)
    # each query head uses its KV head's keys and values
    kr_h, v_h = np.repeat(kr, G, axis=1), np.repeat(v, G, axis=1)
    o_loc, lse_loc = local_branch(qr, kr_h, v_h, idx["nbr"], tau, rows)
    if summary_rope == "token":
        ks, vs = summaries(kr, v, idx["members"], groups)
    elif summary_rope == "centre":
        ku, vs = summaries(k, v, idx["members"], groups)
        centres = summary_centres(grid, block, idx["pool2"])
        ks = rope(ku, centres, base, spacing)
    else:
        raise ValueError(f"summary_rope must be 'token' or 'centre', got {summary_rope!r}")
    ex = _dropped(idx, coords, grid, block, exclude_near)
    o_glob, lse_glob = global_branch(qr, np.repeat(ks, G, axis=1), np.repeat(vs, G, axis=1),
                                     tau, ex, rows)
    rsel = slice(None) if rows is None else np.asarray(rows)
    o = mixer(o_loc, o_glob, a[:, :, rsel])
    return dict(o=o, o_loc=o_loc, lse_loc=lse_loc, o_glob=o_glob, lse_glob=lse_glob,
                ksum=ks, vsum=vs, index=idx, tau=tau)


def _unpool_weights(idx):
    """Weight of each token in its summary: 1 / (members present in its block x non-empty
    blocks in its group) -- the derivative of the (two-stage) mean."""
    blk, grp = idx["block_of"], idx["sum_of"]
    c2 = idx["count2"][grp] if tuple(idx["pool2"]) != (1, 1, 1) else np.ones(len(blk))
    return 1.0 / (idx["count"][blk] * c2)


def backward(q, k, v, a, dO, coords, grid, block, *, exclude_near=False, tau=None,
             base=10000.0, index=None, pool2=(1, 1, 1), spacing=None, summary_rope="token"):
    """Gradients of sum(dO * o) w.r.t. q, k, v and the gate logits a, in float64.

    Follows the chain of the forward: mixer -> the two softmax branches -> mean pooling ->
    axial RoPE (R(c)^T = R(-c)). With GQA the KV heads' gradients sum over their query heads.
    """
    q, k, v, a, dO = (np.asarray(t, dtype=np.float64) for t in (q, k, v, a, dO))
    d = q.shape[-1]
    G = _heads(q, k)
    tau = 1.0 / math.sqrt(d) if tau is None else float(tau)
    idx = index if index is not None else build_index(coords, grid, block, pool2)
    nbr = idx["nbr"]
    qr = rope(q, coords, base, spacing)
    kr = np.repeat(rope(k, coords, base, spacing), G, axis=1)
    v_h = np.repeat(v, G, axis=1)
    fw = forward(q, k, v, a, coords, grid, block, exclude_near=exclude_near, tau=tau,
                 base=base, index=idx, spacing=spacing, summary_rope=summary_rope)
    o_loc, lse_loc, o_glob, lse_glob = fw["o_loc"], fw["lse_loc"], fw["o_glob"], fw["lse_glob"]
    ks, vs = np.repeat(fw["ksum"], G, axis=1), np.repeat(fw["vsum"], G, axis=1)
    g = sigmoid(a)

    # mixer
    dg = np.sum(dO * (o_loc - o_glob), axis=-1)
    da = dg * g * (1.0 - g)
    dOl = g[..., None] * dO
    dOg = (1.0 - g)[..., None] * dO

    B, H, N, _ = q.shape
    dqr = np.zeros_like(qr)
    dkr = np.zeros_like(kr)
    dv = np.zeros_like(v_h)
    dk_direct = np.zeros_like(kr)  # summary-centre RoPE: global part, already unrotated

    # local branch: P_ij = exp(s_ij - lse_i), dS_ij = P_ij (dP_ij - D_i) tau
    Dl = np.sum(dOl * o_loc, axis=-1)
    for i in range(N):
        js = [int(j) for j in nbr[i] if j >= 0]
        s = np.einsum("bhd,bhjd->bhj", qr[:, :, i], kr[:, :, js]) * tau
        p = np.exp(s - lse_loc[:, :, i][..., None])
        dp = np.einsum("bhd,bhjd->bhj", dOl[:, :, i], v_h[:, :, js])
        ds = p * (dp - Dl[:, :, i][..., None]) * tau
        dqr[:, :, i] += np.einsum("bhj,bhjd->bhd", ds, kr[:, :, js])
        for t, j in enumerate(js):
            dkr[:, :, j] += ds[:, :, t][..., None] * qr[:, :, i]
            dv[:, :, j] += p[:, :, t][..., None] * dOl[:, :, i]

    # global branch
    Dg = np.sum(dOg * o_glob, axis=-1)
    s = np.einsum("bhnd,bhmd->bhnm", qr, ks) * tau
    ex = _dropped(idx, coords, grid, block, exclude_near)
    if ex is not None:
        s = np.where(ex[None, None], -np.inf, s)
    lse_safe = np.where(np.isfinite(lse_glob), lse_glob, 0.0)
    p = np.where(np.isfinite(s) & np.isfinite(lse_glob)[..., None],
                 np.exp(np.where(np.isfinite(s), s, 0.0) - lse_safe[..., None]), 0.0)
    dp = np.einsum("bhnd,bhmd->bhnm", dOg, vs)
    ds = p * (dp - Dg[..., None]) * tau
    dqr += np.einsum("bhnm,bhmd->bhnd", ds, ks)
    dks = np.einsum("bhnm,bhnd->bhmd", ds, qr)
    dvs = np.einsum("bhnm,bhnd->bhmd", p, dOg)

    # un-pool: each member receives its weight in the (two-stage) mean of its summary's
    # gradient; with summary-centre RoPE the key gradient first goes back through the
    # summary's rotation R(centre)^T
    w = _unpool_weights(idx)
    grp = idx["sum_of"]
    if summary_rope == "centre":
        dku = rope_inverse(dks, summary_centres(grid, block, idx["pool2"]), base, spacing)
        dk_direct += dku[:, :, grp] * w[None, None, :, None]
    else:
        dkr += dks[:, :, grp] * w[None, None, :, None]
    dv += dvs[:, :, grp] * w[None, None, :, None]

    dq = rope_inverse(dqr, coords, base, spacing)
    dk = rope_inverse(dkr, coords, base, spacing) + dk_direct
    # KV heads: sum over the query heads of each group
    dk = dk.reshape(B, H // G, G, N, d).sum(axis=2)
    dv = dv.reshape(B, H // G, G, N, d).sum(axis=2)
    return dict(dq=dq, dk=dk, dv=dv, da=da, dksum=dks, dvsum=dvs, fwd=fw)


def backward_rows(q, k, v, a, dO, coords, grid, block, *, qrows, krows, exclude_near=False,
                  tau=None, base=10000.0, index=None, fwd=None):
    """Gradients for selected query rows (dq, da) and key rows (dk, dv), one (b,h) set at a time.

    Same definitions as :func:`backward`; it needs the full forward of the global branch (for
    D_g of every query) but evaluates the local terms only around the requested rows.
    """
    q, k, v, a, dO = (np.asarray(t, dtype=np.float64) for t in (q, k, v, a, dO))
    d = q.shape[-1]
    tau = 1.0 / math.sqrt(d) if tau is None else float(tau)
    idx = index if index is not None else build_index(coords, grid, block)
    nbr, block_of = idx["nbr"], idx["sum_of"]
    wt = _unpool_weights(idx)
    qr, kr = rope(q, coords, base), rope(k, coords, base)
    fw = fwd if fwd is not None else forward(q, k, v, a, coords, grid, block,
                                             exclude_near=exclude_near, tau=tau, base=base,
                                             index=idx)
    o_loc, lse_loc, o_glob, lse_glob = fw["o_loc"], fw["lse_loc"], fw["o_glob"], fw["lse_glob"]
    ks, vs = fw["ksum"], fw["vsum"]
    g = sigmoid(a)
    dOl = g[..., None] * dO
    dOg = (1.0 - g)[..., None] * dO
    Dl = np.sum(dOl * o_loc, axis=-1)
    Dg = np.sum(dOg * o_glob, axis=-1)
    ex = _dropped(idx, coords, grid, block, exclude_near)

    def p_glob(rows):
        s = np.einsum("bhrd,bhmd->bhrm", qr[:, :, rows], ks) * tau
        if ex is not None:
            s = np.where(ex[rows][None, None], -np.inf, s)
        ls = lse_glob[:, :, rows]
        lsafe = np.where(np.isfinite(ls), ls, 0.0)
        return np.where(np.isfinite(s) & np.isfinite(ls)[..., None],
                        np.exp(np.where(np.isfinite(s), s, 0.0) - lsafe[..., None]), 0.0)

    def local_terms(i):
        js = [int(j) for j in nbr[i] if j >= 0]
        s = np.einsum("bhd,bhjd->bhj", qr[:, :, i], kr[:, :, js]) * tau
        p = np.exp(s - lse_loc[:, :, i][..., None])
        dp = np.einsum("bhd,bhjd->bhj", dOl[:, :, i], v[:, :, js])
        return js, p, p * (dp - Dl[:, :, i][..., None]) * tau

    qrows = np.asarray(qrows)
    krows = np.asarray(krows)
    B, H = q.shape[:2]
    dq = np.zeros((B, H, len(qrows), d))
    for r, i in enumerate(qrows):
        js, _, ds = local_terms(i)
        acc = np.einsum("bhj,bhjd->bhd", ds, kr[:, :, js])
        pg = p_glob(np.array([i]))[:, :, 0]
        dpg = np.einsum("bhd,bhmd->bhm", dOg[:, :, i], vs)
        dsg = pg * (dpg - Dg[:, :, i][..., None]) * tau
        acc += np.einsum("bhm,bhmd->bhd", dsg, ks)
        dq[:, :, r] = acc
    dq = rope_inverse(dq, np.asarray(coords)[qrows], base)
    da = (np.sum(dO * (o_loc - o_glob), axis=-1) * g * (1.0 - g))[:, :, qrows]

    # global summary gradients for the blocks of the requested keys (all queries contribute)
    need = sorted(set(int(block_of[j]) for j in krows))
    dks = {}
    dvs = {}
    S = np.einsum("bhnd,bhmd->bhnm", qr, ks[:, :, need]) * tau
    if ex is not None:
        S = np.where(ex[:, need][None, None], -np.inf, S)
    lsafe = np.where(np.isfinite(lse_glob), lse_glob, 0.0)
    P = np.where(np.isfinite(S) & np.isfinite(lse_glob)[..., None],
                 np.exp(np.where(np.isfinite(S), S, 0.0) - lsafe[..., None]), 0.0)
    dP = np.einsum("bhnd,bhmd->bhnm", dOg, vs[:, :, need])
    dS = P * (dP - Dg[..., None]) * tau
    for t, m in enumerate(need):
        dks[m] = np.einsum("bhn,bhnd->bhd", dS[:, :, :, t], qr)
        dvs[m] = np.einsum("bhn,bhnd->bhd", P[:, :, :, t], dOg)

    dk = np.zeros((B, H, len(krows), d))
    dv = np.zeros((B, H, len(krows), d))
    for r, j in enumerate(krows):
        # queries i with j in N(i) are exactly the tokens of j's own neighbourhood
        for i in [int(t) for t in nbr[j] if t >= 0]:
            js, p, ds = local_terms(i)
            t = js.index(int(j))
            dk[:, :, r] += ds[:, :, t][..., None] * qr[:, :, i]
            dv[:, :, r] += p[:, :, t][..., None] * dOl[:, :, i]
        m = int(block_of[j])
        dk[:, :, r] += dks[m] * wt[j]
        dv[:, :, r] += dvs[m] * wt[j]
    dk = rope_inverse(dk, np.asarray(coords)[krows], base)
    return dict(dq=dq, da=da, dk=dk, dv=dv)
