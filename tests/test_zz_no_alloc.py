"""The backward entry point that allocates nothing (pack3d_attn_bwd_noalloc).

Some callers cannot allocate device memory (a host framework that owns every allocation
through its own pool, a latency-critical loop that cannot take cudaMalloc's implicit
synchronisation). For them the library serves the backward's scratch from a fixed buffer of
its own. This file is collected last on purpose; each test builds its own inputs, so it passes
alone in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import inputs

pytestmark = pytest.mark.gpu


def _run(dtype, d, grid, block, exclude_near):
    import geometry_aware_local_pack3d_b200 as p3d
    cfg = dict(grid=grid, block=block, batch=1, heads=2, d=d, dtype=dtype, packing="random",
               qkv_std=d ** -0.5, exclude_near=exclude_near)
    w = inputs.make_workload(cfg)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ix = p3d.pack3d_build_index(p3d.make_geom(grid, block, d),
                                coords=torch.from_numpy(w["coords"]).cuda())
    q, k, v, a = (w[n].to(dt).cuda().contiguous() for n in "qkva")
    ksum, vsum = p3d.pack3d_summarize(ix, k, v)
    saved = p3d.pack3d_attn_fwd(ix, q, k, v, a, ksum, vsum, exclude_near=exclude_near,
                                save_for_backward=True)
    dO = inputs.pack(inputs.upstream_grad(1, 2, grid, d), w["perm"]).to(dt).cuda().contiguous()
    ref = p3d.pack3d_attn_bwd(ix, q, k, v, a, ksum, vsum, saved, dO, exclude_near=exclude_near)
    outs = [p3d.pack3d_attn_bwd_noalloc(ix, q, k, v, a, ksum, vsum, saved, dO,
                                        exclude_near=exclude_near) for _ in range(2)]
    torch.cuda.synchronize()
    return ix, ref, outs


@pytest.mark.parametrize("dtype,d,exclude_near", [("fp32", 48, True), ("bf16", 96, False)])
def test_noalloc_backward_matches_workspace_backward_twice(dtype, d, exclude_near):
    # the same kernels run on the same inputs with only the scratch address changed, and they
    # are deterministic (no atomics), so the results agree bit for bit
    _, ref, outs = _run(dtype, d, (4, 8, 8), (2, 2, 4), exclude_near)
    for out in outs:  # two calls in a row share the library's buffer
        for key in ("dq", "dk", "dv", "dgate"):
            assert torch.equal(out[key], ref[key]), key


def test_noalloc_backward_rejects_problems_beyond_its_buffer():
    import geometry_aware_local_pack3d_b200 as p3d
    from geometry_aware_local_pack3d_b200 import binding as b
    ix, _, _ = _run("fp32", 48, (4, 4, 8), (2, 2, 2), False)
    heads = 20000  # workspace far beyond the built-in 32 MiB buffer
    assert p3d.pack3d_bwd_workspace_bytes(ix, 0, 1, heads) > b.NOALLOC_SCRATCH_BYTES
    buf = torch.empty(64, dtype=torch.float32, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    status = b.lib().pack3d_attn_bwd_noalloc(ctypes.byref(ix.struct), *([p] * 11), 0, 1, heads,
                                             0, 0.1, 0, p, p, p, p, None)
    assert status == 8  # PACK3D_ERR_WORKSPACE, before any launch
    assert b.lib().pack3d_last_launch_count() == 0
    # an argument error is the one pack3d_attn_bwd reports (unsupported batch x heads here)
    status = b.lib().pack3d_attn_bwd_noalloc(ctypes.byref(ix.struct), *([p] * 11), 0, 1, 70000,
                                             0, 0.1, 0, p, p, p, p, None)
    assert status == 2  # PACK3D_ERR_UNSUPPORTED
    assert b.lib().pack3d_last_launch_count() == 0
