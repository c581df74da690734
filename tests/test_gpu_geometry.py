"""GPU parity of the extended geometry against the float64 CPU oracle, through the C ABI.

Sparse fields (sites without a token) and partial edge blocks, the second pooling stage,
per-axis coordinate maps in RoPE, summary-centre RoPE and GQA / MQA, on every kernel path:
float32 (CUDA cores), bf16 with raw keys and bf16 with the rotated keys of
pack3d_summarize_rotated (tensor cores), forward and backward; the index tables bit for bit;
coordinate-carrying repacks of a sparse field bit for bit; and the pages' 1M-token timing
point (64 x 128 x 128 tokens, 4x4x4 blocks pooled again over 1x2x2 groups = 4,096 summaries
per KV head) on sampled rows.
"""
import numpy as np
import pytest
import torch

import inputs
from oracle import pack3d_oracle as orc
from tests.test_gpu_parity import (assert_close, compare_tables, gpu_index, np64, p3d,
                                   sampled_rows, tdtype)

pytestmark = pytest.mark.gpu


def workload(grid, block, B, H, d, dtype, packing, *, Hkv=None, occupancy=1.0, pool2=(1, 1, 1),
             summary_rope="token", spacing=(1.0, 1.0, 1.0), exclude_near=False, seed=0):
    cfg = dict(grid=grid, block=block, batch=B, heads=H, kv_heads=Hkv or H, d=d, dtype=dtype,
               packing=packing, qkv_std=1.0 if dtype == "fp32" else d ** -0.5,
               exclude_near=exclude_near, occupancy=occupancy, pool2=pool2,
               summary_rope=summary_rope, spacing=spacing)
    return inputs.make_workload(cfg, seed=seed)


def plan(w):
    return dict(pool2=w["pool2"], spacing=w["spacing"], summary_rope=w["summary_rope"])


def run_forward(w, path, save=True):
    """path: 'plain' (summaries + forward on raw keys) or 'rotated' (summaries and rotated keys
    in one pass, then the forward on the rotated keys)."""
    m = p3d()
    dt = tdtype(w["dtype"])
    ix = gpu_index(w, w["d"])
    q, k, v, a = (w[n].to(dt).cuda().contiguous() for n in "qkva")
    if path == "rotated":
        ksum, vsum, k_rot = m.pack3d_summarize_rotated(ix, k, v)
        out = m.pack3d_attn_fwd(ix, q, k_rot, v, a, ksum, vsum, exclude_near=w["exclude_near"],
                                k_rotated=True, save_for_backward=save)
    else:
        ksum, vsum = m.pack3d_summarize(ix, k, v)
        out = m.pack3d_attn_fwd(ix, q, k, v, a, ksum, vsum, exclude_near=w["exclude_near"],
                                save_for_backward=save)
    torch.cuda.synchronize()
    out.update(ix=ix, q=q, k=k, v=v, a=a, ksum=ksum, vsum=vsum)
    return out


def check_forward(w, g):
    ref = orc.forward(w["q"].numpy(), w["k"].numpy(), w["v"].numpy(), w["a"].numpy(),
                      w["coords"], w["grid"], w["block"], exclude_near=w["exclude_near"],
                      **plan(w))
    for key in ("o", "o_loc", "o_glob", "lse_loc", "lse_glob"):
        assert_close(np64(g[key]), ref[key], w["dtype"], key)
    ks = p3d().summary_rows(g["ksum"], ref["index"]["n_summaries"])
    assert_close(np64(ks), ref["ksum"], w["dtype"], "ksum")
    return ref


# name: grid, block, B, H, Hkv, d, occupancy, pool2, summary_rope, spacing, packing, exclude
CASES = {
    "partial_blocks": ((5, 6, 7), (2, 4, 3), 1, 2, 2, 48, 1.0, (1, 1, 1), "token", None,
                       "random", True),
    "sparse_two_stage": ((6, 8, 9), (2, 2, 2), 1, 2, 2, 96, 0.6, (1, 2, 2), "token", None,
                         "morton", True),
    "centre_anisotropic": ((4, 6, 8), (2, 2, 4), 1, 2, 2, 96, 0.8, (1, 1, 1), "centre",
                           (0.5, 1.5, 1.0), "random", False),
    "gqa_two_stage": ((4, 8, 8), (2, 2, 2), 2, 4, 2, 48, 1.0, (2, 1, 2), "token", None,
                      "raster", True),
    "mqa_centre_sparse": ((6, 6, 10), (2, 3, 2), 1, 3, 1, 96, 0.7, (1, 2, 1), "centre",
                          (1.0, 0.25, 2.0), "raster_block", True),
    # a long axis: the rotation table (3 x extent x d/6 pairs of (cos, sin)) is larger than
    # 64 KB, so the kernels that otherwise keep it in shared memory read it from L1 / L2
    "long_axis_d96": ((2, 3, 200), (2, 2, 4), 1, 2, 2, 96, 0.9, (1, 1, 1), "token", None,
                      "morton", False),
    "long_axis_d48_centre": ((2, 2, 400), (1, 2, 8), 1, 2, 1, 48, 1.0, (1, 1, 2), "centre",
                             None, "raster", True),
}


def case(name, dtype):
    grid, block, B, H, Hkv, d, occ, pool2, sr, sp, kind, ex = CASES[name]
    return workload(grid, block, B, H, d, dtype, kind, Hkv=Hkv, occupancy=occ, pool2=pool2,
                    summary_rope=sr, spacing=sp or (1.0, 1.0, 1.0), exclude_near=ex)


@pytest.mark.parametrize("name", sorted(CASES))
def test_extended_index_tables_bit_exact(name):
    w = case(name, "fp32")
    ref = orc.build_index(w["coords"], w["grid"], w["block"], w["pool2"])
    compare_tables(gpu_index(w, w["d"]), w, ref)
    compare_tables(gpu_index(w, w["d"], via="perm"), w, ref)


def test_summary_centre_table_matches_the_box_centres():
    w = case("mqa_centre_sparse", "fp32")
    ix = gpu_index(w, w["d"])
    tab = ix.centre_table().cpu().numpy().astype(np.float64)  # [M, d/2, 2]
    ctr = orc.summary_centres(w["grid"], w["block"], w["pool2"]) * np.asarray(w["spacing"])
    theta = orc.rope_theta(w["d"])
    ang = np.concatenate([ctr[:, a:a + 1] * theta[None, :] for a in range(3)], axis=1)
    assert np.abs(tab[..., 0] - np.cos(ang)).max() < 1e-6
    assert np.abs(tab[..., 1] - np.sin(ang)).max() < 1e-6


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("dtype,path", [("fp32", "plain"), ("bf16", "plain"),
                                        ("bf16", "rotated")])
def test_extended_forward(name, dtype, path):
    w = case(name, dtype)
    check_forward(w, run_forward(w, path))


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_extended_backward(name, dtype):
    m = p3d()
    w = case(name, dtype)
    g = run_forward(w, "plain")
    dO = inputs.pack(inputs.upstream_grad(w["batch"], w["heads"], w["grid"], w["d"]), w["perm"])
    if dtype == "bf16":
        dO = dO.to(torch.bfloat16).to(torch.float32)
    gr = m.pack3d_attn_bwd(g["ix"], g["q"], g["k"], g["v"], g["a"], g["ksum"], g["vsum"], g,
                           dO.to(tdtype(dtype)).cuda().contiguous(),
                           exclude_near=w["exclude_near"])
    torch.cuda.synchronize()
    ref = orc.backward(w["q"].numpy(), w["k"].numpy(), w["v"].numpy(), w["a"].numpy(),
                       dO.numpy(), w["coords"], w["grid"], w["block"],
                       exclude_near=w["exclude_near"], **plan(w))
    for key, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dgate", "da")):
        assert_close(np64(gr[key]), ref[rk], dtype, key)


def holed(dtype, pool2=(1, 1, 2)):
    """An 8 x 12 x 16 field (2x2x2 blocks) with no token in z < 4, y < 4, x < 8: sixteen empty
    blocks, so empty summaries drop out of every softmax."""
    w = workload((8, 12, 16), (2, 2, 2), 1, 2, 96, dtype, "random", pool2=pool2,
                 exclude_near=True)
    c = w["coords"]
    keep = ~((c[:, 0] < 4) & (c[:, 1] < 4) & (c[:, 2] < 8))
    sel = torch.as_tensor(np.nonzero(keep)[0])
    w["perm"] = np.asarray(w["perm"])[keep]
    w["coords"] = c[keep]
    for n in "qkva":
        w[n] = w[n].index_select(2, sel).contiguous()
    return w


@pytest.mark.parametrize("dtype,path", [("fp32", "plain"), ("bf16", "plain"),
                                        ("bf16", "rotated")])
def test_empty_summaries_forward_and_backward(dtype, path):
    m = p3d()
    w = holed(dtype)
    g = run_forward(w, path)
    assert int(g["ix"].struct.n_empty) == 8
    ref = check_forward(w, g)
    dO = inputs.pack(inputs.upstream_grad(1, 2, w["grid"], 96), np.asarray(w["perm"]))
    if dtype == "bf16":
        dO = dO.to(torch.bfloat16).to(torch.float32)
    gr = m.pack3d_attn_bwd(g["ix"], g["q"], g["k"], g["v"], g["a"], g["ksum"], g["vsum"], g,
                           dO.to(tdtype(dtype)).cuda().contiguous(), exclude_near=True)
    torch.cuda.synchronize()
    rb = orc.backward(w["q"].numpy(), w["k"].numpy(), w["v"].numpy(), w["a"].numpy(),
                      dO.numpy(), w["coords"], w["grid"], w["block"], exclude_near=True,
                      index=ref["index"], **plan(w))
    for key, rk in (("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dgate", "da")):
        assert_close(np64(gr[key]), rb[rk], dtype, key)


@pytest.mark.parametrize("occupancy", [0.55, 0.9])
def test_bf16_sparse_field_spanning_many_units(occupancy):
    # several two-tile local units and 64-summary chunks, a ragged edge on every axis, empty
    # summaries inside the field, both tensor-core local kernels
    w = workload((13, 10, 21), (2, 2, 3), 1, 2, 96, "bf16", "random", occupancy=occupancy,
                 exclude_near=True)
    for path in ("plain", "rotated"):
        check_forward(w, run_forward(w, path))


def test_sparse_repacking_is_an_exact_permutation():
    outs = {}
    for kind in inputs.PACKINGS:
        w = workload((8, 12, 16), (2, 2, 4), 1, 2, 96, "bf16", kind, occupancy=0.7,
                     pool2=(2, 1, 1), exclude_near=True)
        g = run_forward(w, "rotated", save=False)
        full = torch.zeros(1, 2, int(np.prod(w["grid"])), 96, dtype=torch.bfloat16)
        full[:, :, torch.as_tensor(w["perm"])] = g["o"].cpu()  # back to raster sites
        outs[kind] = full
    for kind in inputs.PACKINGS:
        assert torch.equal(outs[kind], outs["raster"]), kind


def test_forward_1m_token_field_sampled():
    # the pages' high-token timing point: 1,048,576 tokens, 4,096 summaries per KV head
    w = dict(grid=(64, 128, 128), block=(4, 4, 4), pool2=(1, 2, 2), batch=1, heads=8,
             kv_heads=8, d=96, dtype="bf16", packing="raster_block", qkv_std=96 ** -0.5,
             exclude_near=False, summary_rope="token", spacing=(1.0, 1.0, 1.0))
    w = inputs.make_workload(w)
    g = run_forward(w, "rotated")
    assert g["ix"].m == 4096
    rows = sampled_rows(len(w["coords"]), 48, seed=5)
    idx = orc.build_index(w["coords"], w["grid"], w["block"], w["pool2"], nbr_rows=rows)
    for b, h in ((0, 2), (0, 7)):
        sl = lambda t: t[b:b + 1, h:h + 1].numpy()  # noqa: E731
        ref = orc.forward(sl(w["q"]), sl(w["k"]), sl(w["v"]), sl(w["a"]), w["coords"],
                          w["grid"], w["block"], index=idx, rows=rows, **plan(w))
        for key in ("o", "lse_loc", "lse_glob", "o_loc", "o_glob"):
            assert_close(np64(g[key][b, h][rows]), ref[key][0, 0], "bf16", f"{key}[{b},{h}]")
        ks = p3d().summary_rows(g["ksum"], 4096)[b, h]
        assert_close(np64(ks), ref["ksum"][0, 0], "bf16", "ksum")
