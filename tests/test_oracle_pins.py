"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Closed forms, invariants the pages state, special cases that reduce to textbook routines
(torch's scaled_dot_product_attention), the pages' printed facts (tests/golden), brute force
on tiny grids, an independent dense formulation (tests/dense_reference.py), finite
differences and torch.autograd. CPU only.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import inputs
from oracle import pack3d_oracle as orc
from tests import dense_reference as dref

T = lambda x: torch.as_tensor(np.asarray(x), dtype=torch.float64)  # noqa: E731


def rand_field(B, H, n, d, seed):
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, n, d, generator=g, dtype=torch.float64) for _ in range(3))
    a = torch.randn(B, H, n, generator=g, dtype=torch.float64)
    return q, k, v, a


# ------------------------------------------------------------------------------ index tables
def test_neighbour_counts_closed_form():
    grid = (5, 4, 6)
    perm = inputs.packing("random", grid, seed=3)
    c = inputs.coords_of(perm, grid)
    idx = orc.build_index(c, grid, (1, 2, 3))
    counts = (idx["nbr"] >= 0).sum(1)
    per_axis = lambda x, G: 3 - (x == 0) - (x == G - 1)  # noqa: E731
    expect = per_axis(c[:, 0], 5) * per_axis(c[:, 1], 4) * per_axis(c[:, 2], 6)
    assert np.array_equal(counts, expect)
    assert set(np.unique(counts)) == {8, 12, 18, 27}
    assert counts.sum() == np.prod([3 * G - 2 for G in grid])


def test_neighbours_brute_force_random_packing():
    grid = (4, 5, 3)
    perm = inputs.packing("random", grid, seed=7)
    c = inputs.coords_of(perm, grid).astype(np.int64)
    idx = orc.build_index(c, grid, (2, 5, 3))
    for i in range(len(c)):
        brute = {j for j in range(len(c)) if np.abs(c[j] - c[i]).max() <= 1}
        got = [int(j) for j in idx["nbr"][i] if j >= 0]
        assert set(got) == brute and len(got) == len(brute)
        for o, (dz, dy, dx) in enumerate(itertools.product((-1, 0, 1), repeat=3)):
            j = idx["nbr"][i, o]
            if j >= 0:
                assert tuple(c[j] - c[i]) == (dz, dy, dx)


def test_inverse_and_block_tables():
    grid, block = (4, 6, 8), (2, 3, 4)
    perm = inputs.packing("morton", grid)
    c = inputs.coords_of(perm, grid).astype(np.int64)
    idx = orc.build_index(c, grid, block)
    r = (c[:, 0] * 6 + c[:, 1]) * 8 + c[:, 2]
    assert np.array_equal(idx["inv"][r], np.arange(len(c)))
    mem = idx["members"]
    assert sorted(mem.ravel().tolist()) == list(range(len(c)))
    assert np.all(idx["count"] == 24)
    boxes = orc.block_boxes(grid, block)
    for m in range(mem.shape[0]):
        lo, hi = np.array(boxes[m][0]), np.array(boxes[m][1])
        for s, j in enumerate(mem[m]):
            assert np.all(c[j] >= lo) and np.all(c[j] <= hi)
            rel = c[j] - lo
            assert s == (rel[0] * 3 + rel[1]) * 4 + rel[2]


def test_index_rejects_duplicates_and_range():
    with pytest.raises(orc.OracleIndexError):
        orc.build_index([[0, 0, 0], [0, 0, 0]], (2, 2, 2), (1, 1, 1))
    with pytest.raises(orc.OracleIndexError):
        orc.build_index([[0, 0, 2]], (2, 2, 2), (1, 1, 1))


def test_golden_raster_face_neighbours(golden_facts):
    f = golden_facts["raster_face_neighbours"]
    grid = tuple(f["grid"])
    perm = inputs.packing("raster", grid)
    idx = orc.build_index(inputs.coords_of(perm, grid), grid, (2, 2, 2))
    faces = [orc.OFFSETS.index(o) for o in [(-1, 0, 0), (0, -1, 0), (0, 0, -1), (0, 0, 1),
                                            (0, 1, 0), (1, 0, 0)]]
    for i in range(len(perm)):
        z, y, x = inputs.unravel([i], grid)[0]
        if 0 < z < 7 and 0 < y < 7 and 0 < x < 7:
            got = sorted(int(idx["nbr"][i, o]) - i for o in faces)
            assert got == sorted(f["sequence_offsets"])


def test_golden_lab_field_and_summary_counts(golden_facts):
    lab = golden_facts["two_indices_lab"]
    grid, block = tuple(lab["grid"]), tuple(lab["block"])
    idx = orc.build_index(inputs.coords_of(inputs.packing("raster", grid), grid), grid, block)
    assert len(idx["nbr"]) == lab["tokens"]
    assert (idx["nbr"] >= 0).sum(1).max() == golden_facts["neighbourhood_size"]["max_tokens"]
    assert idx["n_blocks"] == lab["tokens"] // 8
    # M = N / v: 256-token summaries reproduce both printed summary counts
    shapes = {262144: (64, 64, 64), 1048576: (64, 128, 128)}
    for case in golden_facts["summary_counts"]["cases"]:
        grid = shapes[case["tokens"]]
        assert np.prod(grid) == case["tokens"]
        assert len(orc.block_boxes(grid, (4, 8, 8))) == case["summaries"]


# ---------------------------------------------------------------------------------- RoPE
def test_rope_matches_complex_rotation_and_is_orthogonal():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(2, 3, 10, 24, generator=g, dtype=torch.float64)
    c = torch.randint(-50, 50, (10, 3), generator=g)
    r = orc.rope(x.numpy(), c.numpy())
    assert np.allclose(r, dref.rope_complex(x, c).numpy(), atol=1e-12)
    assert np.allclose(np.linalg.norm(r, axis=-1), x.norm(dim=-1).numpy(), atol=1e-12)
    assert np.allclose(orc.rope_inverse(r, c.numpy()), x.numpy(), atol=1e-12)
    assert np.allclose(orc.rope(x.numpy(), np.zeros((10, 3))), x.numpy())


def test_rope_d6_is_one_planar_rotation_per_axis():
    # d = 6: one pair per axis with theta_0 = 1, so each plane turns by the coordinate itself.
    x = np.arange(1.0, 7.0)[None, :]
    c = np.array([[0.3, -1.1, 2.0]])
    r = orc.rope(x, c)[0]
    for axis in range(3):
        ang = c[0, axis]
        rot = np.array([[math.cos(ang), -math.sin(ang)], [math.sin(ang), math.cos(ang)]])
        assert np.allclose(r[2 * axis:2 * axis + 2], rot @ x[0, 2 * axis:2 * axis + 2])


def test_rope_relative_identity():
    # <R(a) q, R(b) k> = <q, R(b - a) k>  (project page Ch.3 "A logit that only sees displacement")
    g = np.random.default_rng(1)
    q, k = g.standard_normal((1, 48)), g.standard_normal((1, 48))
    a, b = np.array([[3, -7, 12]]), np.array([[-2, 5, 40]])
    lhs = np.sum(orc.rope(q, a) * orc.rope(k, b))
    rhs = np.sum(q * orc.rope(k, b - a))
    assert abs(lhs - rhs) < 1e-10


# --------------------------------------------------------------------------------- local
@pytest.mark.parametrize("kind", ["raster", "random"])
def test_local_branch_equals_dense_chebyshev_attention(kind):
    grid, d = (4, 3, 5), 12
    perm = inputs.packing(kind, grid, seed=11)
    c = inputs.coords_of(perm, grid)
    q, k, v, _ = rand_field(2, 2, len(c), d, 5)
    idx = orc.build_index(c, grid, (2, 3, 5))
    qr, kr = orc.rope(q.numpy(), c), orc.rope(k.numpy(), c)
    o, lse = orc.local_branch(qr, kr, v.numpy(), idx["nbr"], 0.37)
    od, lsed = dref.masked_attention(dref.rope_complex(q, c), dref.rope_complex(k, c), v,
                                     dref.chebyshev_mask(c), 0.37)
    assert np.allclose(o, od.numpy(), atol=1e-12)
    assert np.allclose(lse, lsed.numpy(), atol=1e-12)


def test_local_branch_centre_of_3x3x3_is_plain_sdpa():
    grid, d = (3, 3, 3), 18
    c = inputs.coords_of(inputs.packing("random", grid, seed=2), grid)
    q, k, v, _ = rand_field(1, 2, 27, d, 9)
    idx = orc.build_index(c, grid, (3, 3, 3))
    i = int(idx["inv"][(1 * 3 + 1) * 3 + 1])
    qr, kr = orc.rope(q.numpy(), c), orc.rope(k.numpy(), c)
    o, _ = orc.local_branch(qr, kr, v.numpy(), idx["nbr"], 1 / math.sqrt(d), rows=[i])
    ref = torch.nn.functional.scaled_dot_product_attention(T(qr[:, :, i:i + 1]), T(kr), v)
    assert np.allclose(o, ref.numpy(), atol=1e-12)


# ------------------------------------------------------------------------- summaries/global
def test_prop1_summary_logit_is_mean_of_relative_logits():
    # q_rot . mean(k_rot) = mean_j <q_i, R(c_j - c_i) k_j>  (paper summary §B.5; project page Ch.3)
    grid, block, d = (4, 4, 4), (2, 2, 2), 24
    c = inputs.coords_of(inputs.packing("morton", grid), grid)
    q, k, v, _ = rand_field(1, 1, 64, d, 4)
    idx = orc.build_index(c, grid, block)
    qr, kr = orc.rope(q.numpy(), c), orc.rope(k.numpy(), c)
    ks, _ = orc.summaries(kr, v.numpy(), idx["members"])
    for i in (0, 17, 63):
        for m in range(idx["n_blocks"]):
            js = idx["members"][m]
            rel = np.array([np.dot(q.numpy()[0, 0, i],
                                   dref.rope_complex(k[0, 0, j:j + 1], c[j:j + 1] - c[i:i + 1]).numpy()[0])
                            for j in js])
            assert abs(np.dot(qr[0, 0, i], ks[0, 0, m]) - rel.mean()) < 1e-12


def test_unit_blocks_make_global_branch_dense_sdpa():
    grid, d = (2, 3, 4), 12
    c = inputs.coords_of(inputs.packing("random", grid, seed=5), grid)
    q, k, v, _ = rand_field(1, 2, 24, d, 8)
    idx = orc.build_index(c, grid, (1, 1, 1))
    qr, kr = orc.rope(q.numpy(), c), orc.rope(k.numpy(), c)
    ks, vs = orc.summaries(kr, v.numpy(), idx["members"])
    o, _ = orc.global_branch(qr, ks, vs, 1 / math.sqrt(d))
    ref = torch.nn.functional.scaled_dot_product_attention(T(qr), T(kr), v)
    assert np.allclose(o, ref.numpy(), atol=1e-12)


@pytest.mark.parametrize("exclude_near", [False, True])
def test_global_branch_equals_dense_formulation(exclude_near):
    grid, block, d = (4, 6, 8), (2, 2, 4), 12
    c = inputs.coords_of(inputs.packing("random", grid, seed=13), grid)
    q, k, v, a = rand_field(2, 1, len(c), d, 21)
    fw = orc.forward(q.numpy(), k.numpy(), v.numpy(), a.numpy(), c, grid, block,
                     exclude_near=exclude_near)
    de = dref.pack3d_dense(q, k, v, a, c, grid, block, exclude_near=exclude_near)
    for key in ("ksum", "vsum", "o_glob", "lse_glob", "o_loc", "o"):
        assert np.allclose(fw[key], de[key].numpy(), atol=1e-12), key


def test_exclusion_box_test_matches_block_ids_of_the_cube():
    grid, block = (6, 4, 9), (3, 2, 3)
    c = inputs.coords_of(inputs.packing("raster", grid), grid)
    assert np.array_equal(orc.excluded_summaries(c, grid, block),
                          dref.near_block_mask(c, grid, block).numpy())


def test_all_summaries_excluded_gives_zero_global_output():
    grid, block = (4, 4, 4), (2, 2, 2)
    c = inputs.coords_of(inputs.packing("raster", grid), grid)
    q, k, v, a = rand_field(1, 1, 64, 12, 3)
    fw = orc.forward(q.numpy(), k.numpy(), v.numpy(), a.numpy(), c, grid, block, exclude_near=True)
    i = (1 * 4 + 1) * 4 + 1  # site (1,1,1): its cube meets all eight blocks
    assert np.all(fw["o_glob"][0, 0, i] == 0) and fw["lse_glob"][0, 0, i] == -np.inf
    g = 1 / (1 + np.exp(-a.numpy()[0, 0, i]))
    assert np.allclose(fw["o"][0, 0, i], g * fw["o_loc"][0, 0, i])


def test_summary_set_order_invariance():
    # project page Ch.7: permuting summary keys and values together changes nothing
    g = np.random.default_rng(0)
    qr = g.standard_normal((1, 2, 20, 12))
    ks, vs = g.standard_normal((1, 2, 9, 12)), g.standard_normal((1, 2, 9, 12))
    p = g.permutation(9)
    o1, l1 = orc.global_branch(qr, ks, vs, 0.3)
    o2, l2 = orc.global_branch(qr, ks[:, :, p], vs[:, :, p], 0.3)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)


def test_rotate_then_pool_sees_member_positions():
    # project page Ch.3 "One block, two ways to summarize it": swapping two token states inside
    # a block moves the rotate-then-pool summary; a uniform pool-then-rotate summary cannot move.
    grid, block, d = (1, 1, 4), (1, 1, 4), 6
    c = inputs.coords_of(inputs.packing("raster", grid), grid)
    g = np.random.default_rng(3)
    k, v = g.standard_normal((1, 1, 4, d)), g.standard_normal((1, 1, 4, d))
    idx = orc.build_index(c, grid, block)
    sw = k.copy()
    sw[:, :, [0, 3]] = k[:, :, [3, 0]]
    ks1, _ = orc.summaries(orc.rope(k, c), v, idx["members"])
    ks2, _ = orc.summaries(orc.rope(sw, c), v, idx["members"])
    assert np.abs(ks1 - ks2).max() > 1e-2
    centre = np.array([[0, 0, 1.5]])
    pr1 = orc.rope(k.mean(axis=2, keepdims=True), centre)
    pr2 = orc.rope(sw.mean(axis=2, keepdims=True), centre)
    assert np.allclose(pr1, pr2, atol=1e-14)


def test_gate_limits_select_one_branch():
    grid, block = (4, 4, 4), (2, 2, 2)
    c = inputs.coords_of(inputs.packing("raster", grid), grid)
    q, k, v, _ = rand_field(1, 1, 64, 12, 6)
    for val, key in ((60.0, "o_loc"), (-60.0, "o_glob")):
        a = np.full((1, 1, 64), val)
        fw = orc.forward(q.numpy(), k.numpy(), v.numpy(), a, c, grid, block)
        assert np.allclose(fw["o"], fw[key], atol=1e-20)


# ------------------------------------------------------------------------ whole operator
@pytest.mark.parametrize("shift", [(5, -3, 7), (1000, 1000, 1000)])
def test_translation_invariance(shift):
    # paper summary §B.2: a common coordinate shift leaves every logit unchanged
    grid, block = (4, 4, 6), (2, 2, 3)
    c = inputs.coords_of(inputs.packing("morton", grid), grid)
    q, k, v, a = (t.numpy() for t in rand_field(1, 2, len(c), 12, 1))
    base = orc.forward(q, k, v, a, c, grid, block, exclude_near=True)
    moved = orc.forward(q, k, v, a, c, grid, block, exclude_near=True,
                        rope_coords=c + np.array(shift))
    assert np.abs(base["o"] - moved["o"]).max() < 1e-10
    for key in ("lse_loc", "lse_glob"):
        np.testing.assert_allclose(moved[key], base[key], rtol=0, atol=1e-10)


@pytest.mark.parametrize("exclude_near", [False, True])
def test_packing_equivariance(exclude_near):
    # project page Ch.4 Proposition 2 / paper summary §B.3: a coordinate-carrying repack only
    # permutes the output (the repack test of the project page's Chapter 10)
    grid, block, d = (4, 4, 8), (2, 2, 2), 12
    q, k, v, a = inputs.field(1, 2, grid, d, seed=0)
    outs = {}
    for kind in inputs.PACKINGS:
        perm = inputs.packing(kind, grid, block, seed=1)
        c = inputs.coords_of(perm, grid)
        fw = orc.forward(*(inputs.pack(t, perm).numpy() for t in (q, k, v, a)), c, grid, block,
                         exclude_near=exclude_near)
        outs[kind] = inputs.unpack(torch.from_numpy(fw["o"]), perm).numpy()
    for kind in inputs.PACKINGS:
        assert np.abs(outs[kind] - outs["raster"]).max() < 1e-12


def test_sequence_index_rope_is_not_equivariant():
    # paper summary §B.4 (negative control): RoPE at the memory slot changes with the packing.
    grid, block, d = (4, 4, 8), (2, 2, 2), 12
    q, k, v, a = inputs.field(1, 1, grid, d, seed=0)
    res = {}
    for kind in ("raster", "morton"):
        perm = inputs.packing(kind, grid, block)
        c = inputs.coords_of(perm, grid)
        seq = inputs.unravel(np.arange(len(perm)), grid)  # coordinates read off the slot index
        fw = orc.forward(*(inputs.pack(t, perm).numpy() for t in (q, k, v, a)), c, grid, block,
                         rope_coords=seq)
        res[kind] = inputs.unpack(torch.from_numpy(fw["o"]), perm).numpy()
    assert np.abs(res["raster"] - res["morton"]).max() > 1e-3


# ------------------------------------------------------------------------------ backward
def _loss(q, k, v, a, dO, c, grid, block, ex):
    return np.sum(dO * orc.forward(q, k, v, a, c, grid, block, exclude_near=ex)["o"])


@pytest.mark.parametrize("exclude_near", [False, True])
def test_backward_central_differences(exclude_near):
    grid, block, d = (3, 4, 4), (1, 2, 2), 6
    c = inputs.coords_of(inputs.packing("random", grid, seed=4), grid)
    q, k, v, a = (t.numpy() for t in rand_field(1, 1, len(c), d, 12))
    dO = np.random.default_rng(2).standard_normal(q.shape)
    gr = orc.backward(q, k, v, a, dO, c, grid, block, exclude_near=exclude_near)
    rng = np.random.default_rng(0)
    eps = 1e-6
    for name, arr, key in (("q", q, "dq"), ("k", k, "dk"), ("v", v, "dv"), ("a", a, "da")):
        for _ in range(6):
            pos = tuple(rng.integers(0, s) for s in arr.shape)
            ap, am = arr.copy(), arr.copy()
            ap[pos] += eps
            am[pos] -= eps
            args = {"q": q, "k": k, "v": v, "a": a}
            lp = _loss(*[ap if n == name else args[n] for n in "qkva"], dO, c, grid, block, exclude_near)
            lm = _loss(*[am if n == name else args[n] for n in "qkva"], dO, c, grid, block, exclude_near)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - gr[key][pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, gr[key][pos])


@pytest.mark.parametrize("exclude_near", [False, True])
def test_backward_matches_autograd_of_dense_formulation(exclude_near):
    grid, block, d = (4, 4, 6), (2, 2, 3), 12
    c = inputs.coords_of(inputs.packing("morton", grid), grid)
    q, k, v, a = rand_field(2, 1, len(c), d, 31)
    dO = torch.randn(q.shape, generator=torch.Generator().manual_seed(2), dtype=torch.float64)
    leaves = [t.clone().requires_grad_(True) for t in (q, k, v, a)]
    out = dref.pack3d_dense(*leaves, c, grid, block, exclude_near=exclude_near)["o"]
    (out * dO).sum().backward()
    gr = orc.backward(q.numpy(), k.numpy(), v.numpy(), a.numpy(), dO.numpy(), c, grid, block,
                      exclude_near=exclude_near)
    for t, key in zip(leaves, ("dq", "dk", "dv", "da")):
        assert np.allclose(gr[key], t.grad.numpy(), atol=1e-11), key


def test_backward_rows_agrees_with_full_backward():
    grid, block, d = (4, 4, 4), (2, 2, 2), 12
    c = inputs.coords_of(inputs.packing("random", grid, seed=9), grid)
    q, k, v, a = (t.numpy() for t in rand_field(1, 2, 64, d, 14))
    dO = np.random.default_rng(5).standard_normal(q.shape)
    full = orc.backward(q, k, v, a, dO, c, grid, block, exclude_near=True)
    rows = np.array([0, 5, 33, 63])
    part = orc.backward_rows(q, k, v, a, dO, c, grid, block, qrows=rows, krows=rows[::-1],
                             exclude_near=True)
    assert np.allclose(part["dq"], full["dq"][:, :, rows], atol=1e-12)
    assert np.allclose(part["da"], full["da"][:, :, rows], atol=1e-12)
    assert np.allclose(part["dk"], full["dk"][:, :, rows[::-1]], atol=1e-12)
    assert np.allclose(part["dv"], full["dv"][:, :, rows[::-1]], atol=1e-12)
