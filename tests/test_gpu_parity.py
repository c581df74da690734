"""GPU parity: the CUDA path (through the C ABI) against the float64 CPU oracle.

Bar: index tables bit-exact; float32 I/O max-abs-err <= 1e-4; bfloat16 I/O max-abs-err <= 2e-2
and relative L2 <= 5e-3 (o, lse, dq, dk, dv, dgate); coordinate-carrying repacks give outputs
that are exact permutations of the raster output.
"""
import math

import numpy as np
import pytest
import torch

import inputs
from oracle import pack3d_oracle as orc

pytestmark = pytest.mark.gpu

F32_TOL = 1e-4
BF16_ABS, BF16_REL = 2e-2, 5e-3


def p3d():
    import geometry_aware_local_pack3d_b200 as m
    return m


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: non-finite pattern differs"
    err = np.abs(got[fin] - ref[fin])
    mx = float(err.max()) if err.size else 0.0
    if dtype == "fp32":
        assert mx <= F32_TOL, f"{what}: max-abs-err {mx:.3e} > {F32_TOL}"
    else:
        rel = float(np.linalg.norm(got[fin] - ref[fin]) / max(np.linalg.norm(ref[fin]), 1e-30))
        assert mx <= BF16_ABS, f"{what}: max-abs-err {mx:.3e} > {BF16_ABS}"
        assert rel <= BF16_REL, f"{what}: rel-L2 {rel:.3e} > {BF16_REL}"


def tdtype(dt):
    return torch.bfloat16 if dt == "bf16" else torch.float32


def gpu_index(w, d, via="coords"):
    m = p3d()
    geom = m.make_geom(w["grid"], w["block"], d, pool2=w.get("pool2", (1, 1, 1)),
                       summary_rope=w.get("summary_rope", "token"),
                       spacing=w.get("spacing", (1.0, 1.0, 1.0)))
    if via == "coords":
        return m.pack3d_build_index(geom, coords=torch.from_numpy(w["coords"]).cuda())
    return m.pack3d_build_index(geom, perm=torch.from_numpy(np.asarray(w["perm"])).cuda())


def gpu_forward(w, exclude_near, save=False, ix=None, rotated=False):
    """rotated: summaries and rotated keys in one pass, then the forward on the rotated keys
    (the row-gather local branch)."""
    m = p3d()
    dt = tdtype(w["dtype"])
    ix = ix or gpu_index(w, w["d"])
    q, k, v, a = (w[n].to(dt).cuda().contiguous() for n in "qkva")
    if rotated:
        ksum, vsum, k_rot = m.pack3d_summarize_rotated(ix, k, v)
        out = m.pack3d_attn_fwd(ix, q, k_rot, v, a, ksum, vsum, exclude_near=exclude_near,
                                k_rotated=True, save_for_backward=True if save else False)
    else:
        ksum, vsum = m.pack3d_summarize(ix, k, v)
        out = m.pack3d_attn_fwd(ix, q, k, v, a, ksum, vsum, exclude_near=exclude_near,
                                save_for_backward=True if save else False)
    torch.cuda.synchronize()
    out.update(ksum=ksum, vsum=vsum, ix=ix, q=q, k=k, v=v, a=a)
    return out


def small(grid, block, B, H, d, dtype, packing, exclude_near=False, qkv_std=1.0, seed=0):
    cfg = dict(grid=grid, block=block, batch=B, heads=H, d=d, dtype=dtype, packing=packing,
               qkv_std=qkv_std, exclude_near=exclude_near)
    return inputs.make_workload(cfg, seed=seed)


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


# ----------------------------------------------------------------------------- index tables
def compare_tables(ix, w, ref):
    n = len(w["coords"])
    M, vol = ref["members"].shape
    c = w["coords"].astype(np.int64)
    packed = (c[:, 0] << 20) | (c[:, 1] << 10) | c[:, 2]
    assert np.array_equal(ix.table("coord", (n,)).cpu().numpy(), packed)
    assert np.array_equal(ix.table("inv", (len(ref["inv"]),)).cpu().numpy(), ref["inv"])
    assert np.array_equal(ix.table("nbr", (n, 27)).cpu().numpy(), ref["nbr"])
    assert np.array_equal(ix.table("block_of", (n,)).cpu().numpy(), ref["block_of"])
    assert np.array_equal(ix.table("slot_of", (n,)).cpu().numpy(), ref["slot_of"])
    assert np.array_equal(ix.table("members", (M, vol)).cpu().numpy(), ref["members"])
    assert np.array_equal(ix.table("count", (M,)).cpu().numpy(), ref["count"])
    # summaries: the second pooling stage's groups, per-summary block counts and empty bits
    S, gv = ref["groups"].shape
    assert ix.m == S == ref["n_summaries"] and int(ix.struct.n_blocks) == M
    assert np.array_equal(ix.table("sum_of", (n,)).cpu().numpy(), ref["sum_of"])
    assert np.array_equal(ix.table("groups", (S, gv)).cpu().numpy(), ref["groups"])
    assert np.array_equal(ix.table("count2", (S,)).cpu().numpy(), ref["count2"])
    words = ix.table("empty", ((S + 31) // 32,)).cpu().numpy().view(np.uint32)
    bits = (words[np.arange(S) // 32] >> (np.arange(S) % 32)) & 1
    assert np.array_equal(bits == 1, ref["count2"] == 0)
    assert int(ix.struct.n_empty) == int((ref["count2"] == 0).sum())


@pytest.mark.parametrize("grid,block", [((8, 8, 8), (2, 2, 2)), ((6, 10, 12), (3, 2, 4)),
                                        ((1, 5, 7), (1, 5, 7))])
@pytest.mark.parametrize("kind", inputs.PACKINGS)
def test_index_tables_bit_exact(grid, block, kind):
    if kind == "raster_block" and any(g % b for g, b in zip(grid, block)):
        pytest.skip("block packing needs divisible grid")
    w = small(grid, block, 1, 1, 48, "fp32", kind)
    ref = orc.build_index(w["coords"], grid, block)
    compare_tables(gpu_index(w, 48), w, ref)
    compare_tables(gpu_index(w, 48, via="perm"), w, ref)


@pytest.mark.parametrize("kind", inputs.PACKINGS)
def test_index_tables_bit_exact_65k_field(kind):
    w = dict(inputs.WORKLOADS["field65k_repack_bf16"])
    perm = inputs.packing(kind, w["grid"], w["block"], seed=1)
    w.update(perm=perm, coords=inputs.coords_of(perm, w["grid"]))
    ref = orc.build_index(w["coords"], w["grid"], w["block"])
    compare_tables(gpu_index(w, 96), w, ref)


def test_rope_table_matches_theta_plan():
    w = small((4, 6, 9), (1, 1, 1), 1, 1, 96, "fp32", "raster")
    w["spacing"] = (0.5, 1.0, 2.0)
    ix = gpu_index(w, 96)
    tab = ix.rope_table().cpu().numpy().astype(np.float64)  # [axis, coordinate, pair, 2]
    theta = orc.rope_theta(96)
    for a, sp in enumerate(w["spacing"]):
        ang = sp * np.arange(9)[:, None] * theta[None, :]
        assert np.abs(tab[a, ..., 0] - np.cos(ang)).max() < 1e-6
        assert np.abs(tab[a, ..., 1] - np.sin(ang)).max() < 1e-6


def test_index_errors_are_reported():
    m = p3d()
    geom = m.make_geom((2, 2, 2), (1, 1, 1), 48)
    c = torch.from_numpy(inputs.coords_of(np.arange(8), (2, 2, 2))).cuda()
    dup = c.clone()
    dup[3] = dup[5]
    with pytest.raises(m.Pack3DError) as e:
        m.pack3d_build_index(geom, coords=dup)
    assert e.value.status == 3
    bad = c.clone()
    bad[2, 1] = 2
    with pytest.raises(m.Pack3DError) as e:
        m.pack3d_build_index(geom, coords=bad)
    assert e.value.status == 4
    with pytest.raises(m.Pack3DError) as e:
        m.pack3d_build_index(geom, perm=torch.tensor([0, 1, 2, 3, 4, 5, 6, 8]).cuda())
    assert e.value.status == 4
    # the library stays usable after reported errors
    m.pack3d_build_index(geom, coords=c)


# -------------------------------------------------------------------------------- forward
@pytest.mark.parametrize("dtype,d", [("fp32", 48), ("fp32", 96), ("bf16", 48), ("bf16", 96)])
def test_summaries(dtype, d):
    w = small((4, 8, 8), (2, 4, 4), 2, 2, d, dtype, "random")
    g = gpu_forward(w, False)
    ix = orc.build_index(w["coords"], w["grid"], w["block"])
    ks, vs = orc.summaries(orc.rope(w["k"].numpy(), w["coords"]), w["v"].numpy(), ix["members"])
    m = p3d()
    assert_close(np64(m.summary_rows(g["ksum"], ix["n_blocks"])), ks, dtype, "ksum")
    assert_close(np64(m.summary_rows(g["vsum"], ix["n_blocks"])), vs, dtype, "vsum")
    # the zero padding of the last summary tile
    M = ix["n_blocks"]
    tail = m.summary_rows(g["ksum"], (M + 63) // 64 * 64)[:, :, M:]
    assert torch.count_nonzero(tail) == 0


def full_compare(w, exclude_near, what="", rotated=False):
    g = gpu_forward(w, exclude_near, save=True, rotated=rotated)
    ref = orc.forward(w["q"].numpy(), w["k"].numpy(), w["v"].numpy(), w["a"].numpy(),
                      w["coords"], w["grid"], w["block"], exclude_near=exclude_near)
    for key in ("o", "o_loc", "o_glob", "lse_loc", "lse_glob"):
        assert_close(np64(g[key]), ref[key], w["dtype"], f"{what}{key}")
    return g, ref


def test_forward_tiny_field_fp32():
    # the 8x8x8 / 2x2x2 field of the two-indices lab, fp32, d48, raster
    w = inputs.make_workload("tiny_8x8x8_fp32")
    full_compare(w, False)


@pytest.mark.parametrize("kind", inputs.PACKINGS)
@pytest.mark.parametrize("exclude_near", [False, True])
def test_forward_bf16_d96_packings(kind, exclude_near):
    w = small((8, 8, 16), (4, 4, 4), 1, 2, 96, "bf16", kind, qkv_std=96 ** -0.5)
    full_compare(w, exclude_near, f"{kind}/{exclude_near}/")


@pytest.mark.parametrize("dtype,d", [("fp32", 96), ("bf16", 48), ("fp32", 48)])
def test_forward_other_dtypes(dtype, d):
    w = small((6, 8, 10), (3, 2, 5), 2, 1, d, dtype, "morton")
    full_compare(w, True, f"{dtype}/{d}/")


def test_forward_all_summaries_excluded():
    w = small((4, 4, 4), (2, 2, 2), 1, 2, 48, "fp32", "random")
    g, ref = full_compare(w, True)
    lse = g["lse_glob"].cpu().numpy()
    assert np.isneginf(lse).sum() == np.isneginf(ref["lse_glob"]).sum() > 0
    assert np.all(g["o_glob"].cpu().numpy()[np.isneginf(lse)] == 0)


def test_forward_unit_blocks_and_thin_grid():
    w = small((1, 6, 5), (1, 1, 1), 1, 1, 48, "fp32", "random")
    full_compare(w, False)
    full_compare(w, True)


def sampled_rows(n, count, seed=0):
    rng = np.random.default_rng(seed)
    edge = [0, 1, 63, 64, 127, 128, n - 129, n - 128, n - 1]
    return np.unique(np.concatenate([rng.choice(n, count, replace=False), edge]))


def sampled_compare(w, exclude_near, heads=((0, 0), (-1, -1)), count=96, rotated=False):
    g = gpu_forward(w, exclude_near, save=True, rotated=rotated)
    idx = orc.build_index(w["coords"], w["grid"], w["block"])
    rows = sampled_rows(len(w["coords"]), count)
    for (b, h) in heads:
        sl = lambda t: t[b:b + 1 if b != -1 else None, h:h + 1 if h != -1 else None].numpy()  # noqa: E731
        ref = orc.forward(sl(w["q"]), sl(w["k"]), sl(w["v"]), sl(w["a"]), w["coords"], w["grid"],
                          w["block"], exclude_near=exclude_near, index=idx, rows=rows)
        for key in ("o", "lse_loc", "lse_glob", "o_loc", "o_glob"):
            gv = g[key][b, h][rows] if key.startswith("o") else g[key][b, h][rows]
            assert_close(np64(gv), ref[key][0, 0], w["dtype"], f"{key}[{b},{h}]")
        assert_close(np64(p3d().summary_rows(g["ksum"], idx["n_summaries"])[b, h]),
                     ref["ksum"][0, 0], w["dtype"], "ksum")
    return g


def test_forward_65k_field_sampled():
    sampled_compare(inputs.make_workload("field65k_bf16"), False)


def test_forward_262k_field_sampled():
    sampled_compare(inputs.make_workload("field262k_bf16"), False, heads=((0, 3),), count=64)


def test_forward_rotated_keys_262k_field_sampled():
    # the benchmarked path (summaries + rotated keys, two-tile local units) on the 64^3 field
    sampled_compare(inputs.make_workload("field262k_bf16"), False, heads=((0, 5),), count=64,
                    rotated=True)


def test_repacking_equivariance_is_exact_65k_field():
    # four coordinate-carrying packings: outputs are exact permutations of the raster output
    outs = {}
    for kind in inputs.PACKINGS:
        w = inputs.make_workload("field65k_repack_bf16", packing_kind=kind)
        g = gpu_forward(w, True)
        outs[kind] = inputs.unpack(g["o"].cpu(), w["perm"])
        del g
    for kind in inputs.PACKINGS:
        assert torch.equal(outs[kind], outs["raster"]), kind
    # and the raster output itself meets the oracle on sampled rows
    w = inputs.make_workload("field65k_repack_bf16", packing_kind="random")
    sampled_compare(w, True, heads=((1, 5),), count=48)


# ------------------------------------------------------------------------------- backward
def gpu_backward(w, exclude_near):
    m = p3d()
    g = gpu_forward(w, exclude_near, save=True)
    dO = inputs.pack(inputs.upstream_grad(w["batch"], w["heads"], w["grid"], w["d"]), w["perm"])
    if w["dtype"] == "bf16":
        dO = dO.to(torch.bfloat16).to(torch.float32)
    dOd = dO.to(tdtype(w["dtype"])).cuda().contiguous()
    gr = m.pack3d_attn_bwd(g["ix"], g["q"], g["k"], g["v"], g["a"], g["ksum"], g["vsum"], g, dOd,
                           exclude_near=exclude_near)
    torch.cuda.synchronize()
    return gr, dO


@pytest.mark.parametrize("dtype,d,exclude_near", [("fp32", 48, False), ("fp32", 96, True),
                                                  ("bf16", 96, True), ("bf16", 48, False)])
def test_backward_full(dtype, d, exclude_near):
    w = small((4, 4, 8), (2, 2, 4), 1, 2, d, dtype, "random",
              qkv_std=1.0 if dtype == "fp32" else d ** -0.5)
    gr, dO = gpu_backward(w, exclude_near)
    ref = orc.backward(w["q"].numpy(), w["k"].numpy(), w["v"].numpy(), w["a"].numpy(),
                       dO.numpy(), w["coords"], w["grid"], w["block"], exclude_near=exclude_near)
    for key, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dgate", "da")):
        assert_close(np64(gr[key]), ref[rk], dtype, key)


def test_backward_65k_field_sampled():
    w = inputs.make_workload("field65k_fwdbwd_bf16")
    gr, dO = gpu_backward(w, False)
    b, h = 1, 6
    sl = lambda t: t[b:b + 1, h:h + 1].numpy()  # noqa: E731
    rows = sampled_rows(len(w["coords"]), 24)
    idx = orc.build_index(w["coords"], w["grid"], w["block"])
    ref = orc.backward_rows(sl(w["q"]), sl(w["k"]), sl(w["v"]), sl(w["a"]), sl(dO), w["coords"],
                            w["grid"], w["block"], qrows=rows, krows=rows, index=idx)
    assert_close(np64(gr["dq"][b, h][rows]), ref["dq"][0, 0], "bf16", "dq")
    assert_close(np64(gr["dgate"][b, h][rows]), ref["da"][0, 0], "bf16", "dgate")
    assert_close(np64(gr["dk"][b, h][rows]), ref["dk"][0, 0], "bf16", "dk")
    assert_close(np64(gr["dv"][b, h][rows]), ref["dv"][0, 0], "bf16", "dv")


# ------------------------------------------------------------- bf16 tensor-core path edges
@pytest.mark.parametrize("d", [48, 96])
def test_bf16_all_summaries_excluded(d):
    w = small((4, 4, 4), (2, 2, 2), 2, 2, d, "bf16", "random", qkv_std=d ** -0.5)
    g, ref = full_compare(w, True)
    lse = g["lse_glob"].cpu().numpy()
    assert np.isneginf(lse).sum() == np.isneginf(ref["lse_glob"]).sum() > 0
    assert np.all(g["o_glob"].float().cpu().numpy()[np.isneginf(lse)] == 0)


@pytest.mark.parametrize("exclude_near", [False, True])
def test_bf16_ragged_rows_and_summary_chunks(exclude_near):
    # N = 1,920 (7.5 units of 256 rows) and M = 240 (one full and one partial chunk of 128)
    w = small((8, 12, 20), (2, 2, 2), 1, 3, 96, "bf16", "morton", qkv_std=96 ** -0.5)
    full_compare(w, exclude_near)


def test_bf16_thin_grid_unit_blocks():
    # M = N = 105: every token is its own summary; one partial unit
    w = small((3, 5, 7), (1, 1, 1), 1, 2, 48, "bf16", "random", qkv_std=48 ** -0.5)
    full_compare(w, True)
    full_compare(w, False)


# --------------------------------------------- rotated keys + row-gather local branch (bf16)
@pytest.mark.parametrize("d", [48, 96])
def test_summarize_rotated_keys_and_summaries(d):
    m = p3d()
    w = small((4, 8, 8), (2, 4, 4), 2, 2, d, "bf16", "random", qkv_std=d ** -0.5)
    ix = gpu_index(w, d)
    k, v = (w[n].to(torch.bfloat16).cuda().contiguous() for n in "kv")
    ks, vs, k_rot = m.pack3d_summarize_rotated(ix, k, v)
    ks0, vs0 = m.pack3d_summarize(ix, k, v)
    torch.cuda.synchronize()
    # the same summaries as the summaries-only pass, bit for bit
    assert torch.equal(ks, ks0) and torch.equal(vs, vs0)
    # rotated keys: the oracle's R(c) k rounded to bf16
    ref = orc.rope(w["k"].numpy(), w["coords"])
    assert_close(np64(k_rot), ref, "bf16", "k_rot")
    # the input keys are untouched
    assert torch.equal(k.cpu(), w["k"].to(torch.bfloat16))


@pytest.mark.parametrize("kind", inputs.PACKINGS)
@pytest.mark.parametrize("exclude_near", [False, True])
def test_forward_rotated_keys_packings(kind, exclude_near):
    w = small((8, 8, 16), (4, 4, 4), 1, 2, 96, "bf16", kind, qkv_std=96 ** -0.5)
    full_compare(w, exclude_near, f"rot/{kind}/{exclude_near}/", rotated=True)


@pytest.mark.parametrize("grid,block,d", [((6, 10, 12), (3, 2, 4), 48),   # partial bricks
                                          ((5, 6, 10), (5, 3, 2), 96),    # gx*4 % 16 != 0
                                          ((3, 5, 7), (1, 1, 1), 48),     # thin, unit blocks
                                          ((9, 4, 4), (3, 2, 2), 96)])    # one brick column
def test_forward_rotated_keys_ragged_grids(grid, block, d):
    w = small(grid, block, 2, 1, d, "bf16", "random", qkv_std=d ** -0.5)
    full_compare(w, False, "rot/", rotated=True)
    full_compare(w, True, "rot/excl/", rotated=True)


def test_forward_rotated_keys_65k_field_sampled():
    sampled_compare(inputs.make_workload("field65k_bf16"), False, rotated=True)


def test_forward_rotated_keys_match_unrotated_path_65k_field():
    # both local-branch forms see the same rotated keys up to bf16 rounding of R(c) k: the
    # outputs agree to bf16 resolution everywhere
    w = inputs.make_workload("field65k_bf16")
    a = gpu_forward(w, False, rotated=False)["o"].float()
    b = gpu_forward(w, False, rotated=True)["o"].float()
    assert float((a - b).abs().max()) <= 2e-2
    assert float((a - b).norm() / a.norm()) <= 5e-3


def test_repacking_equivariance_is_exact_rotated_keys():
    outs = {}
    for kind in inputs.PACKINGS:
        w = inputs.make_workload("field65k_repack_bf16", packing_kind=kind)
        g = gpu_forward(w, True, rotated=True)
        outs[kind] = inputs.unpack(g["o"].cpu(), w["perm"])
        del g
    for kind in inputs.PACKINGS:
        assert torch.equal(outs[kind], outs["raster"]), kind


@pytest.mark.parametrize("bh", [(1, 1), (3, 5), (40, 4)])
def test_forward_work_counter_returns_to_zero(bh):
    # the rotated-key local kernel takes its work units from a counter in status words 2 and 3
    # of the index: after every call (and after the global call that follows) both are zero
    # again, and a repeated call (units handed to other CTAs) gives the same output bit for
    # bit; (40, 4) has more units than SMs
    m = p3d()
    B, H = bh
    w = small((8, 8, 16), (4, 4, 4), B, H, 96, "bf16", "random", qkv_std=96 ** -0.5)
    ix = gpu_index(w, 96)
    q, k, v, a = (w[n].to(torch.bfloat16).cuda().contiguous() for n in "qkva")
    ks, vs, k_rot = m.pack3d_summarize_rotated(ix, k, v)
    outs = []
    for _ in range(3):
        o_loc, _ = m.pack3d_attn_local(ix, q, k_rot, v, k_rotated=True)
        torch.cuda.synchronize()
        st = ix.table("status", (4,)).cpu()
        assert int(st[0]) == 0 and int(st[2]) == 0 and int(st[3]) == 0, st
        o = m.pack3d_attn_global(ix, q, a, ks, vs, o_loc)
        torch.cuda.synchronize()
        st = ix.table("status", (4,)).cpu()
        assert int(st[0]) == 0 and int(st[2]) == 0 and int(st[3]) == 0, st
        outs.append(o.clone())
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_local_units_independent_of_batch_and_stream():
    # every (batch, head, unit) is computed on its own: one head's output from a batch of 30
    # heads (units spread over all SMs by the work counter) equals, bit for bit, the same head
    # computed alone on a side stream with the same index
    m = p3d()
    w = small((8, 8, 16), (4, 4, 4), 6, 5, 96, "bf16", "random", qkv_std=96 ** -0.5)
    ix = gpu_index(w, 96)
    q, k, v = (w[n].to(torch.bfloat16).cuda().contiguous() for n in "qkv")
    _, _, k_rot = m.pack3d_summarize_rotated(ix, k, v)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    o_all, _ = m.pack3d_attn_local(ix, q, k_rot, v, k_rotated=True, lse_loc=lse)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    for b, h in ((0, 0), (5, 4), (2, 3)):
        sl = lambda t: t[b:b + 1, h:h + 1].contiguous()  # noqa: E731
        q1, k1, v1 = sl(q), sl(k_rot), sl(v)
        with torch.cuda.stream(side):
            lse1 = torch.empty((1, 1, q.shape[2]), dtype=torch.float32, device=q.device)
            o1, _ = m.pack3d_attn_local(ix, q1, k1, v1, k_rotated=True, lse_loc=lse1,
                                        stream=side)
        side.synchronize()
        assert torch.equal(o1[0, 0], o_all[b, h]), (b, h)
        assert torch.equal(lse1[0, 0], lse[b, h]), (b, h)
    st = ix.table("status", (4,)).cpu()
    assert int(st[0]) == 0 and int(st[2]) == 0 and int(st[3]) == 0, st


@pytest.mark.parametrize("dtype,d,rotated", [("bf16", 96, True), ("bf16", 96, False),
                                             ("bf16", 48, True), ("fp32", 48, False)])
def test_split_local_global_calls_equal_fused_forward(dtype, d, rotated):
    # pack3d_attn_local + pack3d_attn_global run the same kernels as pack3d_attn_fwd
    m = p3d()
    w = small((8, 8, 16), (4, 4, 4), 2, 2, d, dtype, "morton", qkv_std=d ** -0.5)
    g = gpu_forward(w, True, save=True, rotated=rotated)
    kk = g["k"]
    if rotated:
        _, _, kk = m.pack3d_summarize_rotated(g["ix"], g["k"], g["v"])
    lse_loc = torch.empty_like(g["lse_loc"])
    o_loc, _ = m.pack3d_attn_local(g["ix"], g["q"], kk, g["v"], k_rotated=rotated,
                                   lse_loc=lse_loc)
    lse_glob = torch.empty_like(g["lse_glob"])
    o = m.pack3d_attn_global(g["ix"], g["q"], g["a"], g["ksum"], g["vsum"], o_loc,
                             exclude_near=True, lse_glob=lse_glob)
    torch.cuda.synchronize()
    assert torch.equal(o_loc, g["o_loc"]) and torch.equal(lse_loc, g["lse_loc"])
    assert torch.equal(o, g["o"]) and torch.equal(lse_glob, g["lse_glob"])
    # in place: the global call may mix into the o_loc buffer itself
    o2 = m.pack3d_attn_global(g["ix"], g["q"], g["a"], g["ksum"], g["vsum"], o_loc,
                              exclude_near=True, o=o_loc)
    torch.cuda.synchronize()
    assert torch.equal(o2, g["o"])


@pytest.mark.parametrize("grid,block,d,exclude_near", [
    ((8, 12, 20), (2, 2, 2), 96, True),    # N 1,920, M 240: two 128-summary tiles, ragged ranges
    ((8, 12, 20), (2, 2, 2), 48, False),
    ((3, 5, 7), (1, 1, 1), 48, True),      # M = N = 105: unit blocks, one partial query tile
    ((4, 4, 4), (2, 2, 2), 96, True),      # every summary excluded for some rows
])
def test_backward_bf16_tensor_core_edges(grid, block, d, exclude_near):
    # bf16 runs the global branch's backward on tensor cores (k_bwd_dsum_tc, k_bwd_dq_tc)
    w = small(grid, block, 1, 2, d, "bf16", "random", qkv_std=d ** -0.5)
    gr, dO = gpu_backward(w, exclude_near)
    ref = orc.backward(w["q"].numpy(), w["k"].numpy(), w["v"].numpy(), w["a"].numpy(),
                       dO.numpy(), w["coords"], w["grid"], w["block"], exclude_near=exclude_near)
    for key, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dgate", "da")):
        assert_close(np64(gr[key]), ref[rk], "bf16", key)
