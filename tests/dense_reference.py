"""A second, deliberately different formulation of PACK3D attention in torch float64.

Used only to pin the CPU oracle (tests). Where the oracle loops over neighbour tables and block
member lists, this file works with dense matrices built straight from coordinates:
  * axial RoPE as a complex multiplication of each (2p, 2p+1) pair by exp(i * c_axis * theta_p);
  * the local branch as dense attention under a Chebyshev-distance <= 1 mask;
  * pooling as a dense [M, N] averaging matrix built from floor(c / block) (and, for a second
    pooling stage, floor(c / (block * pool2)) with per-block and per-group token counts);
  * exclude_near from the summary ids of the (clipped) cube c + {-1, 0, 1}^3.
It is differentiable, so torch.autograd gives gradients independent of the oracle's formulas.
"""
import itertools
import math

import torch


def theta(d, base=10000.0):
    da = d // 3
    return torch.tensor([base ** (-(2.0 * p) / da) for p in range(da // 2)], dtype=torch.float64)


def rope_complex(x, coords, base=10000.0):
    """x [..., N, d] float64; coords [N, 3] (float or int)."""
    d = x.shape[-1]
    da = d // 3
    th = theta(d, base)
    c = torch.as_tensor(coords, dtype=torch.float64)
    parts = []
    for axis in range(3):
        seg = x[..., axis * da:(axis + 1) * da]
        z = torch.view_as_complex(seg.reshape(*seg.shape[:-1], da // 2, 2).contiguous())
        rot = torch.polar(torch.ones_like(c[:, axis:axis + 1] * th), c[:, axis:axis + 1] * th)
        parts.append(torch.view_as_real(z * rot).reshape(seg.shape))
    return torch.cat(parts, dim=-1)


def chebyshev_mask(coords):
    c = torch.as_tensor(coords, dtype=torch.int64)
    return (c[:, None, :] - c[None, :, :]).abs().amax(-1) <= 1


def pooling_matrix(coords, grid, block):
    """A [M, N] with A[m, i] = 1/|S_m| when token i lies in block m."""
    c = torch.as_tensor(coords, dtype=torch.int64)
    g = torch.tensor(grid)
    b = torch.tensor(block)
    nb = g // b
    bc = c // b
    bid = (bc[:, 0] * nb[1] + bc[:, 1]) * nb[2] + bc[:, 2]
    M = int(nb.prod())
    A = torch.zeros(M, len(c), dtype=torch.float64)
    A[bid, torch.arange(len(c))] = 1.0
    cnt = A.sum(1, keepdim=True)
    return A / cnt.clamp_min(1.0)


def near_block_mask(coords, grid, block):
    """E [N, M]: True for the blocks holding any site of the clipped cube around each token."""
    c = torch.as_tensor(coords, dtype=torch.int64)
    g = torch.tensor(grid)
    b = torch.tensor(block)
    nb = g // b
    M = int(nb.prod())
    E = torch.zeros(len(c), M, dtype=torch.bool)
    for off in itertools.product((-1, 0, 1), repeat=3):
        p = c + torch.tensor(off)
        ok = ((p >= 0) & (p < g)).all(-1)
        bc = p // b
        bid = (bc[:, 0] * nb[1] + bc[:, 1]) * nb[2] + bc[:, 2]
        rows = torch.arange(len(c))[ok]
        E[rows, bid[ok]] = True
    return E


def masked_attention(qr, kr, v, allowed, tau):
    s = (qr @ kr.transpose(-1, -2)) * tau
    s = s.masked_fill(~allowed, float("-inf"))
    m = s.amax(-1, keepdim=True)
    m = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
    e = torch.exp(s - m)
    l = e.sum(-1, keepdim=True)
    p = e / torch.where(l > 0, l, torch.ones_like(l))
    lse = torch.where(l[..., 0] > 0, (m + torch.log(torch.where(l > 0, l, torch.ones_like(l))))[..., 0],
                      torch.full_like(l[..., 0], float("-inf")))
    return p @ v, lse


def summary_pooling(coords, grid, block, pool2=(1, 1, 1)):
    """Two-stage averaging matrix A [M, N] built from coordinates alone, plus the centres of the
    summaries' boxes [M, 3] and the summary extents E = block * pool2.

    A token's block is floor(c / block); its summary is floor(c / E) (a group of pool2 blocks),
    numbered raster over ceil(grid / E). Its weight is 1 / (tokens in its block) /
    (non-empty blocks in its summary's group). Rows of empty summaries are zero.
    """
    c = torch.as_tensor(coords, dtype=torch.int64).reshape(-1, 3)
    g = torch.tensor(grid)
    b = torch.tensor(block)
    E = b * torch.tensor(pool2)
    ns = (g + E - 1) // E
    sc = c // E
    sid = (sc[:, 0] * ns[1] + sc[:, 1]) * ns[2] + sc[:, 2]
    bc = c // b
    nbk = (g + b - 1) // b
    bid = (bc[:, 0] * nbk[1] + bc[:, 1]) * nbk[2] + bc[:, 2]
    _, binv, bcnt = torch.unique(bid, return_inverse=True, return_counts=True)
    per_block = bcnt[binv].to(torch.float64)  # tokens present in each token's block
    blocks_in = {}
    for s_, b_ in zip(sid.tolist(), bid.tolist()):
        blocks_in.setdefault(s_, set()).add(b_)
    groups = torch.tensor([len(blocks_in[s_]) for s_ in sid.tolist()], dtype=torch.float64)
    M = int(ns.prod())
    A = torch.zeros(M, len(c), dtype=torch.float64)
    A[sid, torch.arange(len(c))] = 1.0 / (per_block * groups)
    lo = torch.stack(torch.meshgrid(*[torch.arange(int(n)) for n in ns], indexing="ij"),
                     -1).reshape(-1, 3) * E
    hi = torch.minimum(lo + E, g) - 1
    return A, (lo + hi).to(torch.float64) / 2.0, E


def near_summary_mask(coords, grid, E):
    """[N, M]: True for the summaries whose box (extents E) holds a site of the clipped cube."""
    c = torch.as_tensor(coords, dtype=torch.int64).reshape(-1, 3)
    g = torch.tensor(grid)
    E = torch.as_tensor(E)
    ns = (g + E - 1) // E
    M = int(ns.prod())
    X = torch.zeros(len(c), M, dtype=torch.bool)
    for off in itertools.product((-1, 0, 1), repeat=3):
        p = c + torch.tensor(off)
        ok = ((p >= 0) & (p < g)).all(-1)
        sc = p // E
        sid = (sc[:, 0] * ns[1] + sc[:, 1]) * ns[2] + sc[:, 2]
        X[torch.arange(len(c))[ok], sid[ok]] = True
    return X


def pack3d_dense(q, k, v, a, coords, grid, block, exclude_near=False, tau=None, base=10000.0,
                 rope_coords=None, pool2=(1, 1, 1), spacing=None, summary_rope="token"):
    """Dense formulation. k, v may carry fewer (KV) heads than q: query head h uses KV head
    h // (H / H_kv), expanded here by repeat_interleave (autograd then sums the gradients of
    each KV head over its query heads)."""
    d = q.shape[-1]
    tau = 1.0 / math.sqrt(d) if tau is None else tau
    rc = coords if rope_coords is None else rope_coords
    rc = torch.as_tensor(rc, dtype=torch.float64)
    sp = torch.ones(3, dtype=torch.float64) if spacing is None else torch.as_tensor(
        spacing, dtype=torch.float64)
    G = q.shape[1] // k.shape[1]
    qr, kr = rope_complex(q, rc * sp, base), rope_complex(k, rc * sp, base)
    kr_h, v_h = kr.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    o_loc, lse_loc = masked_attention(qr, kr_h, v_h, chebyshev_mask(coords), tau)
    A, centres, E = summary_pooling(coords, grid, block, pool2)
    if summary_rope == "centre":
        ks = rope_complex(A @ k, centres * sp, base)
    else:
        ks = A @ kr
    vs = A @ v
    allowed = (A.sum(1) > 0)[None, :].expand(q.shape[-2], A.shape[0]).clone()  # empty: out
    if exclude_near:
        allowed &= ~near_summary_mask(coords, grid, E)
    o_glob, lse_glob = masked_attention(qr, ks.repeat_interleave(G, dim=1),
                                        vs.repeat_interleave(G, dim=1), allowed, tau)
    g = torch.sigmoid(a)[..., None]
    return dict(o=g * o_loc + (1 - g) * o_glob, o_loc=o_loc, o_glob=o_glob, lse_loc=lse_loc,
                lse_glob=lse_glob, ksum=ks, vsum=vs)
