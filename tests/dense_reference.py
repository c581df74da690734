"""A second, deliberately different formulation of PACK3D attention in torch float64.

Used only to pin the CPU oracle (tests). Where the oracle loops over neighbour tables and block
member lists, this file works with dense matrices built straight from coordinates:
  * axial RoPE as a complex multiplication of each (2p, 2p+1) pair by exp(i * c_axis * theta_p);
  * the local branch as dense attention under a Chebyshev-distance <= 1 mask;
  * pooling as a dense [M, N] averaging matrix built from floor(c / block);
  * exclude_near from the block ids of the (clipped) cube c + {-1, 0, 1}^3.
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


def pack3d_dense(q, k, v, a, coords, grid, block, exclude_near=False, tau=None, base=10000.0,
                 rope_coords=None):
    d = q.shape[-1]
    tau = 1.0 / math.sqrt(d) if tau is None else tau
    rc = coords if rope_coords is None else rope_coords
    qr, kr = rope_complex(q, rc, base), rope_complex(k, rc, base)
    o_loc, lse_loc = masked_attention(qr, kr, v, chebyshev_mask(coords), tau)
    A = pooling_matrix(coords, grid, block)
    ks, vs = A @ kr, A @ v
    allowed = torch.ones(q.shape[-2], A.shape[0], dtype=torch.bool)
    if exclude_near:
        allowed = ~near_block_mask(coords, grid, block)
    o_glob, lse_glob = masked_attention(qr, ks, vs, allowed, tau)
    g = torch.sigmoid(a)[..., None]
    return dict(o=g * o_loc + (1 - g) * o_glob, o_loc=o_loc, o_glob=o_glob, lse_loc=lse_loc,
                lse_glob=lse_glob, ksum=ks, vsum=vs)
