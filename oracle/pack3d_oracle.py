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
def build_index(coords, grid, block):
    """Index tables of a packed field, built by looping over tokens.

    coords: int [N, 3] -- (z, y, x) of the token at memory slot i.
    Returns dict(inv, nbr, block_of, slot_of, members, count, n_blocks, block_volume).
    """
    coords = np.asarray(coords, dtype=np.int64)
    gz, gy, gx = (int(g) for g in grid)
    bz, by, bx = (int(b) for b in block)
    if gz % bz or gy % by or gx % bx:
        raise OracleIndexError("grid not divisible by block")
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
    for i in range(n):
        z, y, x = (int(t) for t in coords[i])
        for o, (dz, dy, dx) in enumerate(OFFSETS):
            zz, yy, xx = z + dz, y + dy, x + dx
            if 0 <= zz < gz and 0 <= yy < gy and 0 <= xx < gx:
                nbr[i, o] = inv[(zz * gy + yy) * gx + xx]

    nbz, nby, nbx = gz // bz, gy // by, gx // bx
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
    return dict(inv=inv, nbr=nbr, block_of=block_of, slot_of=slot_of, members=members,
                count=count, n_blocks=n_blocks, block_volume=vol)


def block_boxes(grid, block):
    """Inclusive [lo, hi] box of every block, block ids in raster order over the block grid."""
    gz, gy, gx = (int(g) for g in grid)
    bz, by, bx = (int(b) for b in block)
    boxes = []
    for mz in range(gz // bz):
        for my in range(gy // by):
            for mx in range(gx // bx):
                lo = (mz * bz, my * by, mx * bx)
                hi = (lo[0] + bz - 1, lo[1] + by - 1, lo[2] + bx - 1)
                boxes.append((lo, hi))
    return boxes


def excluded_summaries(coords, grid, block):
    """bool [N, M]: True where block m's box meets the query's cube [c-1, c+1]^3."""
    coords = np.asarray(coords, dtype=np.int64)
    boxes = block_boxes(grid, block)
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


def rope(x, coords, base=10000.0):
    """Rotate x [..., N, d] by the axial rotation R(c_i) of each token's coordinate."""
    x = np.asarray(x, dtype=np.float64)
    coords = np.asarray(coords, dtype=np.float64)
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


def rope_inverse(x, coords, base=10000.0):
    """R(c)^T x: rotations are orthogonal, so the transpose is the rotation by -c."""
    return rope(x, -np.asarray(coords, dtype=np.float64), base)


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


def summaries(kr, v, members):
    """Uniform means over each block's members, summed in canonical-slot order.

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
    return ks, vs


def global_branch(qr, ksum, vsum, tau, excluded=None, rows=None):
    """Softmax of every query over all summaries ([site] Ch.3 Contract 2; [summary] §3.5).

    excluded: optional bool [N, M] (True = summary dropped for that query).
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
def forward(q, k, v, a, coords, grid, block, *, exclude_near=False, tau=None, base=10000.0,
            rope_coords=None, index=None, rows=None):
    """PACK3D forward in float64.

    q, k, v [B,H,N,d], a [B,H,N], coords int [N,3] (memory order). ``rope_coords`` overrides the
    coordinates used by RoPE only (for the translation and negative-control checks).
    ``rows`` restricts the outputs to some query rows (summaries are always computed in full).
    """
    q, k, v, a = (np.asarray(t, dtype=np.float64) for t in (q, k, v, a))
    d = q.shape[-1]
    tau = 1.0 / math.sqrt(d) if tau is None else float(tau)
    idx = index if index is not None else build_index(coords, grid, block)
    rc = coords if rope_coords is None else rope_coords
    qr, kr = rope(q, rc, base), rope(k, rc, base)
    o_loc, lse_loc = local_branch(qr, kr, v, idx["nbr"], tau, rows)
    ks, vs = summaries(kr, v, idx["members"])
    ex = excluded_summaries(coords, grid, block) if exclude_near else None
    o_glob, lse_glob = global_branch(qr, ks, vs, tau, ex, rows)
    rsel = slice(None) if rows is None else np.asarray(rows)
    o = mixer(o_loc, o_glob, a[:, :, rsel])
    return dict(o=o, o_loc=o_loc, lse_loc=lse_loc, o_glob=o_glob, lse_glob=lse_glob,
                ksum=ks, vsum=vs, index=idx, tau=tau)


def backward(q, k, v, a, dO, coords, grid, block, *, exclude_near=False, tau=None,
             base=10000.0, index=None):
    """Gradients of sum(dO * o) w.r.t. q, k, v and the gate logits a, in float64.

    Follows the chain of the forward: mixer -> the two softmax branches -> mean pooling ->
    axial RoPE (R(c)^T = R(-c)).
    """
    q, k, v, a, dO = (np.asarray(t, dtype=np.float64) for t in (q, k, v, a, dO))
    d = q.shape[-1]
    tau = 1.0 / math.sqrt(d) if tau is None else float(tau)
    idx = index if index is not None else build_index(coords, grid, block)
    nbr, members, count = idx["nbr"], idx["members"], idx["count"]
    qr, kr = rope(q, coords, base), rope(k, coords, base)
    fw = forward(q, k, v, a, coords, grid, block, exclude_near=exclude_near, tau=tau,
                 base=base, index=idx)
    o_loc, lse_loc, o_glob, lse_glob = fw["o_loc"], fw["lse_loc"], fw["o_glob"], fw["lse_glob"]
    ks, vs = fw["ksum"], fw["vsum"]
    g = sigmoid(a)

    # mixer
    dg = np.sum(dO * (o_loc - o_glob), axis=-1)
    da = dg * g * (1.0 - g)
    dOl = g[..., None] * dO
    dOg = (1.0 - g)[..., None] * dO

    B, H, N, _ = q.shape
    dqr = np.zeros_like(qr)
    dkr = np.zeros_like(kr)
    dv = np.zeros_like(v)

    # local branch: P_ij = exp(s_ij - lse_i), dS_ij = P_ij (dP_ij - D_i) tau
    Dl = np.sum(dOl * o_loc, axis=-1)
    for i in range(N):
        js = [int(j) for j in nbr[i] if j >= 0]
        s = np.einsum("bhd,bhjd->bhj", qr[:, :, i], kr[:, :, js]) * tau
        p = np.exp(s - lse_loc[:, :, i][..., None])
        dp = np.einsum("bhd,bhjd->bhj", dOl[:, :, i], v[:, :, js])
        ds = p * (dp - Dl[:, :, i][..., None]) * tau
        dqr[:, :, i] += np.einsum("bhj,bhjd->bhd", ds, kr[:, :, js])
        for t, j in enumerate(js):
            dkr[:, :, j] += ds[:, :, t][..., None] * qr[:, :, i]
            dv[:, :, j] += p[:, :, t][..., None] * dOl[:, :, i]

    # global branch
    Dg = np.sum(dOg * o_glob, axis=-1)
    s = np.einsum("bhnd,bhmd->bhnm", qr, ks) * tau
    if exclude_near:
        s = np.where(excluded_summaries(coords, grid, block)[None, None], -np.inf, s)
    lse_safe = np.where(np.isfinite(lse_glob), lse_glob, 0.0)
    p = np.where(np.isfinite(s) & np.isfinite(lse_glob)[..., None],
                 np.exp(np.where(np.isfinite(s), s, 0.0) - lse_safe[..., None]), 0.0)
    dp = np.einsum("bhnd,bhmd->bhnm", dOg, vs)
    ds = p * (dp - Dg[..., None]) * tau
    dqr += np.einsum("bhnm,bhmd->bhnd", ds, ks)
    dks = np.einsum("bhnm,bhnd->bhmd", ds, qr)
    dvs = np.einsum("bhnm,bhnd->bhmd", p, dOg)

    # un-pool: each member receives 1/|S_m| of its summary's gradient
    M, vol = members.shape
    for m in range(M):
        for s_ in range(vol):
            j = members[m, s_]
            if j >= 0:
                dkr[:, :, j] += dks[:, :, m] / count[m]
                dv[:, :, j] += dvs[:, :, m] / count[m]

    dq = rope_inverse(dqr, coords, base)
    dk = rope_inverse(dkr, coords, base)
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
    nbr, members, count, block_of = idx["nbr"], idx["members"], idx["count"], idx["block_of"]
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
    ex = excluded_summaries(coords, grid, block) if exclude_near else None

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
        dk[:, :, r] += dks[m] / count[m]
        dv[:, :, r] += dvs[m] / count[m]
    dk = rope_inverse(dk, np.asarray(coords)[krows], base)
    return dict(dq=dq, da=da, dk=dk, dv=dv)
