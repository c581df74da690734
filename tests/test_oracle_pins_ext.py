"""Pins of the oracle's extended geometry, each against something other than the oracle itself.

Sparse fields (validity = which lattice sites hold a token) and partial edge blocks, the
second pooling stage, per-axis coordinate maps in RoPE, summary-centre RoPE and GQA/MQA:
brute-force neighbourhoods, the independent dense formulation of tests/dense_reference.py
(averaging matrices and summary boxes built from coordinates alone, complex-multiply RoPE,
torch.autograd), an error bound derived from the rotation geometry, identities that reduce one
case to another, central differences and the pages' printed summary counts. CPU only.
"""
import itertools

import numpy as np
import pytest
import torch

import inputs
from oracle import pack3d_oracle as orc
from tests import dense_reference as dref

T = lambda x: torch.as_tensor(np.asarray(x), dtype=torch.float64)  # noqa: E731


def sparse_field(grid, keep, seed):
    """Coordinates of a random subset (fraction `keep`) of the grid's sites, randomly packed."""
    rng = np.random.default_rng(seed)
    n = int(np.prod(grid))
    sites = np.sort(rng.choice(n, size=max(1, int(round(keep * n))), replace=False))
    perm = sites[rng.permutation(len(sites))]
    return inputs.unravel(perm, grid).astype(np.int64)


def rand(B, H, n, d, seed, Hkv=None):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, n, d, generator=g, dtype=torch.float64)
    k, v = (torch.randn(B, Hkv or H, n, d, generator=g, dtype=torch.float64) for _ in range(2))
    a = torch.randn(B, H, n, generator=g, dtype=torch.float64)
    return q, k, v, a


def close(x, y, tol=1e-10):
    x, y = np.asarray(x, dtype=np.float64), np.asarray(y, dtype=np.float64)
    assert x.shape == y.shape
    assert np.allclose(x, y, rtol=0, atol=tol), float(np.abs(x - y).max())


# ------------------------------------------------------------------------ sparse / partial
def test_sparse_neighbours_brute_force():
    grid = (5, 6, 7)
    c = sparse_field(grid, 0.55, seed=1)
    idx = orc.build_index(c, grid, (2, 4, 3))
    for i in range(len(c)):
        brute = {j for j in range(len(c)) if np.abs(c[j] - c[i]).max() <= 1}
        got = [int(j) for j in idx["nbr"][i] if j >= 0]
        assert set(got) == brute and len(got) == len(brute)
        for o, off in enumerate(itertools.product((-1, 0, 1), repeat=3)):
            j = idx["nbr"][i, o]
            if j >= 0:
                assert tuple(c[j] - c[i]) == off


@pytest.mark.parametrize("pool2", [(1, 1, 1), (2, 1, 2), (1, 2, 3)])
def test_partial_and_two_stage_pooling_equals_dense_averaging(pool2):
    grid, block = (5, 7, 6), (2, 3, 4)  # no extent divides: partial edge blocks everywhere
    c = sparse_field(grid, 0.6, seed=2)
    q, k, v, _ = rand(1, 2, len(c), 12, seed=3)
    idx = orc.build_index(c, grid, block, pool2)
    groups = idx["groups"] if pool2 != (1, 1, 1) else None
    ks, vs = orc.summaries(k.numpy(), v.numpy(), idx["members"], groups)
    A, _, _ = dref.summary_pooling(c, grid, block, pool2)
    assert A.shape[0] == idx["n_summaries"]
    close(ks, (A @ k).numpy(), 1e-12)
    close(vs, (A @ v).numpy(), 1e-12)
    # empty summaries: zero rows exactly where no member is present
    assert np.array_equal(idx["count2"] == 0, (A.sum(1) == 0).numpy())


def test_two_stage_pooling_of_full_blocks_is_one_stage_pooling_over_the_union():
    grid, block, pool2 = (8, 8, 12), (2, 2, 2), (2, 2, 3)
    c = inputs.coords_of(inputs.packing("random", grid, seed=4), grid)
    _, k, v, _ = rand(1, 1, len(c), 6, seed=5)
    two = orc.build_index(c, grid, block, pool2)
    one = orc.build_index(c, grid, (4, 4, 6))
    k2, v2 = orc.summaries(k.numpy(), v.numpy(), two["members"], two["groups"])
    k1, v1 = orc.summaries(k.numpy(), v.numpy(), one["members"])
    close(k2, k1, 1e-12)
    close(v2, v1, 1e-12)
    assert np.array_equal(two["sum_of"], one["block_of"])


@pytest.mark.parametrize("exclude_near", [False, True])
@pytest.mark.parametrize("pool2", [(1, 1, 1), (1, 2, 2)])
def test_sparse_partial_forward_equals_dense_formulation(exclude_near, pool2):
    grid, block = (5, 6, 7), (2, 2, 3)
    c = sparse_field(grid, 0.5, seed=6)
    q, k, v, a = rand(2, 2, len(c), 12, seed=7)
    got = orc.forward(q, k, v, a, c, grid, block, exclude_near=exclude_near, pool2=pool2)
    want = dref.pack3d_dense(q, k, v, a, c, grid, block, exclude_near=exclude_near,
                             pool2=pool2)
    for key in ("o", "o_loc", "o_glob", "lse_loc", "lse_glob"):
        close(got[key], want[key].numpy(), 1e-10)


def test_empty_summaries_drop_out_of_the_softmax():
    # a field with a hole the size of several blocks: the global branch equals a softmax over
    # the non-empty summaries alone
    grid, block = (6, 6, 6), (2, 2, 2)
    allc = inputs.unravel(np.arange(216), grid).astype(np.int64)
    c = allc[~((allc[:, 0] < 4) & (allc[:, 1] < 4) & (allc[:, 2] < 2))]
    q, k, v, a = rand(1, 1, len(c), 12, seed=8)
    idx = orc.build_index(c, grid, block)
    assert (idx["count2"] == 0).sum() == 4
    got = orc.forward(q, k, v, a, c, grid, block, index=idx)
    keep = idx["count2"] > 0
    qr = orc.rope(q.numpy(), c)
    o, lse = orc.global_branch(qr, got["ksum"][:, :, keep], got["vsum"][:, :, keep], got["tau"])
    close(got["o_glob"], o, 1e-12)
    close(got["lse_glob"], lse, 1e-12)


def test_prop1_holds_for_two_stage_summaries():
    # each second-stage summary logit is the weighted mean of the members' relative-RoPE logits
    grid, block, pool2 = (4, 6, 6), (2, 2, 2), (1, 2, 3)
    c = sparse_field(grid, 0.7, seed=9)
    q, k, _, _ = rand(1, 1, len(c), 12, seed=10)
    idx = orc.build_index(c, grid, block, pool2)
    ks, _ = orc.summaries(orc.rope(k.numpy(), c), k.numpy(), idx["members"], idx["groups"])
    A, _, _ = dref.summary_pooling(c, grid, block, pool2)
    qi, ci = q.numpy()[0, 0, 3], c[3]
    for m in range(idx["n_summaries"]):
        rel = orc.rope(k.numpy()[0, 0], c - ci)  # R(c_j - c_i) k_j
        want = float(A[m].numpy() @ (rel @ qi))
        assert abs(float(orc.rope(qi[None], ci[None])[0] @ ks[0, 0, m]) - want) < 1e-12


def test_sparse_packing_equivariance():
    grid, block = (4, 5, 6), (2, 2, 3)
    c = sparse_field(grid, 0.6, seed=11)
    q, k, v, a = rand(1, 2, len(c), 12, seed=12)
    base = orc.forward(q, k, v, a, c, grid, block, exclude_near=True, pool2=(2, 1, 1))
    perm = np.random.default_rng(13).permutation(len(c))
    rep = orc.forward(q[:, :, perm], k[:, :, perm], v[:, :, perm], a[:, :, perm], c[perm], grid,
                      block, exclude_near=True, pool2=(2, 1, 1))
    close(rep["o"], base["o"][:, :, perm], 1e-12)


# ------------------------------------------------------------------------ coordinate maps
def test_anisotropic_rope_equals_complex_rotation_of_scaled_coordinates():
    spacing = (0.5, 2.0, 1.25)
    c = sparse_field((4, 5, 6), 0.8, seed=14)
    x = torch.randn(2, len(c), 18, generator=torch.Generator().manual_seed(15),
                    dtype=torch.float64)
    close(orc.rope(x.numpy(), c, spacing=spacing),
          dref.rope_complex(x, T(c) * T(spacing)).numpy(), 1e-12)


@pytest.mark.parametrize("spacing", [(0.5, 2.0, 1.25), (1 / 4, 1 / 5, 1 / 6)])
def test_anisotropic_forward_is_translation_invariant_and_matches_dense(spacing):
    grid, block = (4, 5, 6), (2, 1, 3)
    c = sparse_field(grid, 0.75, seed=16)
    q, k, v, a = rand(1, 1, len(c), 12, seed=17)
    f = orc.forward(q, k, v, a, c, grid, block, spacing=spacing)
    want = dref.pack3d_dense(q, k, v, a, c, grid, block, spacing=spacing)
    close(f["o"], want["o"].numpy(), 1e-10)
    moved = orc.forward(q, k, v, a, c, grid, block, spacing=spacing,
                        rope_coords=c + np.array([7, -3, 11]))
    close(moved["o"], f["o"], 1e-9)


# ------------------------------------------------------------------- summary-centre RoPE
def test_summary_centre_with_unit_blocks_is_the_token_rotation():
    grid = (3, 4, 5)
    c = sparse_field(grid, 0.8, seed=18)
    q, k, v, a = rand(1, 1, len(c), 12, seed=19)
    tok = orc.forward(q, k, v, a, c, grid, (1, 1, 1))
    ctr = orc.forward(q, k, v, a, c, grid, (1, 1, 1), summary_rope="centre")
    close(ctr["o"], tok["o"], 1e-12)


@pytest.mark.parametrize("pool2", [(1, 1, 1), (2, 1, 1)])
def test_summary_centre_matches_dense_formulation(pool2):
    grid, block = (4, 5, 6), (2, 2, 3)
    c = sparse_field(grid, 0.7, seed=20)
    q, k, v, a = rand(1, 2, len(c), 12, seed=21)
    got = orc.forward(q, k, v, a, c, grid, block, pool2=pool2, summary_rope="centre",
                      exclude_near=True)
    want = dref.pack3d_dense(q, k, v, a, c, grid, block, pool2=pool2, summary_rope="centre",
                             exclude_near=True)
    for key in ("o", "ksum", "lse_glob"):
        close(got[key], want[key].numpy(), 1e-10)


@pytest.mark.parametrize("keys", ["random", "constant_per_block"])
def test_summary_centre_logit_error_bound(keys):
    # |<q~, R(ctr) mean k_j> - <q~, mean R(c_j) k_j>| <= |q| * mean_j |k_j| * max_j |c_j - ctr|_inf
    # (each plane's rotation difference has norm 2|sin(dphi/2)| <= theta_p |dc| <= |dc|, with
    # theta_0 = 1 the fastest frequency). With no key variation inside a block, the error comes
    # from the rotary spread alone and grows with the block diameter.
    grid = (8, 8, 8)
    c = inputs.coords_of(inputs.packing("raster", grid), grid).astype(np.int64)
    q, k, _, _ = rand(1, 1, len(c), 18, seed=22)
    errs = []
    for bs in (2, 4):
        block = (bs, bs, bs)
        idx = orc.build_index(c, grid, block)
        kk = k.numpy().copy()
        if keys == "constant_per_block":
            kk[0, 0] = k.numpy()[0, 0, idx["members"][idx["block_of"], 0]]
        tok, _ = orc.summaries(orc.rope(kk, c), kk, idx["members"])
        pooled, _ = orc.summaries(kk, kk, idx["members"])
        ctrs = orc.summary_centres(grid, block)
        cen = orc.rope(pooled, ctrs)
        worst = 0.0
        for i in range(0, len(c), 37):
            qi = orc.rope(q.numpy()[0, 0, i][None], c[i][None])[0]
            for m in range(idx["n_blocks"]):
                mem = idx["members"][m]
                bound = (np.linalg.norm(qi) * np.linalg.norm(kk[0, 0, mem], axis=1).mean()
                         * np.abs(c[mem] - ctrs[m]).max())
                err = abs(qi @ cen[0, 0, m] - qi @ tok[0, 0, m])
                assert err <= bound + 1e-12
                worst = max(worst, err)
        errs.append(worst)
    assert errs[0] > 0.0
    if keys == "constant_per_block":
        assert errs[1] > errs[0]


def test_pool_then_rotate_ignores_member_positions():
    # the project page's toy: swapping two token states inside a block moves the rotate-then-pool
    # summary but leaves the summary-centre one unchanged
    grid, block = (2, 2, 4), (2, 2, 4)
    c = inputs.coords_of(inputs.packing("raster", grid), grid).astype(np.int64)
    _, k, v, _ = rand(1, 1, len(c), 6, seed=23)
    k2 = k.clone()
    k2[:, :, [0, 5]] = k[:, :, [5, 0]]
    idx = orc.build_index(c, grid, block)
    ctr = orc.summary_centres(grid, block)

    def both(kk):
        kt, _ = orc.summaries(orc.rope(kk.numpy(), c), kk.numpy(), idx["members"])
        ku, _ = orc.summaries(kk.numpy(), kk.numpy(), idx["members"])
        return kt, orc.rope(ku, ctr)

    t1, c1 = both(k)
    t2, c2 = both(k2)
    assert np.abs(t1 - t2).max() > 1e-3
    close(c1, c2, 1e-14)


# --------------------------------------------------------------------------------- GQA
def test_mqa_forward_decomposes_into_single_head_calls():
    grid, block = (4, 4, 6), (2, 2, 3)
    c = sparse_field(grid, 0.8, seed=24)
    q, k, v, a = rand(1, 4, len(c), 12, seed=25, Hkv=1)
    full = orc.forward(q, k, v, a, c, grid, block, exclude_near=True)
    for h in range(4):
        one = orc.forward(q[:, h:h + 1], k, v, a[:, h:h + 1], c, grid, block, exclude_near=True)
        close(full["o"][:, h:h + 1], one["o"], 1e-12)


def test_gqa_forward_matches_dense_formulation():
    grid, block = (4, 5, 4), (2, 1, 2)
    c = sparse_field(grid, 0.8, seed=26)
    q, k, v, a = rand(2, 6, len(c), 12, seed=27, Hkv=2)
    got = orc.forward(q, k, v, a, c, grid, block, pool2=(1, 2, 1))
    want = dref.pack3d_dense(q, k, v, a, c, grid, block, pool2=(1, 2, 1))
    close(got["o"], want["o"].numpy(), 1e-10)


# ---------------------------------------------------------------------------- backward
CASES = {
    "sparse_partial_two_stage": dict(grid=(4, 5, 5), block=(2, 2, 3), keep=0.6, H=2, Hkv=2,
                                     kw=dict(pool2=(1, 2, 1), exclude_near=True)),
    "centre_anisotropic": dict(grid=(3, 4, 5), block=(2, 2, 2), keep=0.8, H=2, Hkv=2,
                               kw=dict(summary_rope="centre", spacing=(0.5, 1.5, 1.0))),
    "gqa": dict(grid=(4, 4, 4), block=(2, 2, 2), keep=0.7, H=4, Hkv=2, kw=dict()),
    "mqa_centre_two_stage": dict(grid=(4, 4, 6), block=(2, 2, 2), keep=0.75, H=3, Hkv=1,
                                 kw=dict(summary_rope="centre", pool2=(1, 1, 3),
                                         exclude_near=True)),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_extended_backward_matches_autograd_of_dense_formulation(name):
    cs = CASES[name]
    c = sparse_field(cs["grid"], cs["keep"], seed=28)
    q, k, v, a = rand(1, cs["H"], len(c), 12, seed=29, Hkv=cs["Hkv"])
    dO = torch.randn(q.shape, generator=torch.Generator().manual_seed(30), dtype=torch.float64)
    got = orc.backward(q, k, v, a, dO, c, cs["grid"], cs["block"], **cs["kw"])
    leaves = [t.clone().requires_grad_(True) for t in (q, k, v, a)]
    out = dref.pack3d_dense(*leaves, c, cs["grid"], cs["block"], **cs["kw"])
    (out["o"] * dO).sum().backward()
    for key, t in zip(("dq", "dk", "dv", "da"), leaves):
        close(got[key], t.grad.numpy(), 1e-9)


def test_extended_backward_central_differences():
    cs = CASES["mqa_centre_two_stage"]
    c = sparse_field(cs["grid"], cs["keep"], seed=31)
    q, k, v, a = (t.numpy() for t in rand(1, cs["H"], len(c), 6, seed=32, Hkv=cs["Hkv"]))
    dO = np.random.default_rng(33).standard_normal(q.shape)
    got = orc.backward(q, k, v, a, dO, c, cs["grid"], cs["block"], **cs["kw"])
    rng = np.random.default_rng(34)
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        for _ in range(4):
            pos = tuple(rng.integers(0, s) for s in x.shape)
            h = 1e-6
            xp, xm = x.copy(), x.copy()
            xp[pos] += h
            xm[pos] -= h
            args = {"q": q, "k": k, "v": v}
            key = name[1:]
            fp = orc.forward(**{**args, key: xp}, a=a, coords=c, grid=cs["grid"],
                             block=cs["block"], **cs["kw"])["o"]
            fm = orc.forward(**{**args, key: xm}, a=a, coords=c, grid=cs["grid"],
                             block=cs["block"], **cs["kw"])["o"]
            num = float(((fp - fm) * dO).sum() / (2 * h))
            assert abs(num - got[name][pos]) <= 1e-6 * max(1.0, abs(num)), (name, pos)


# ---------------------------------------------------------------------- printed counts
def test_second_stage_reproduces_the_printed_summary_counts(golden_facts):
    # 4x4x4 blocks pooled again over 1x2x2 groups: 256 tokens per summary, the pages' 1,024
    # summaries per KV head at 262,144 tokens and 4,096 at 1M tokens
    shapes = {262144: (64, 64, 64), 1048576: (64, 128, 128)}
    for case in golden_facts["summary_counts"]["cases"]:
        grid = shapes[case["tokens"]]
        assert len(orc.summary_boxes(grid, (4, 4, 4), (1, 2, 2))) == case["summaries"]
    # and the index agrees on a small field of the same block plan
    grid = (8, 16, 16)
    idx = orc.build_index(inputs.coords_of(inputs.packing("raster", grid), grid), grid,
                          (4, 4, 4), (1, 2, 2))
    assert idx["n_summaries"] == np.prod(grid) // 256
    assert np.all(idx["count2"] == 4) and np.all(idx["count"] == 64)
