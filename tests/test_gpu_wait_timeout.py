"""Failure detection without a GPU fault: a device-side wait that runs out.

Every wait of the tensor-core kernels is bounded by a cycle budget. Lowering the budget to one
cycle through the testing hook makes the first wait that is not already satisfied give up:
the kernel records PACK3D_ERR_TIMEOUT in the index's status word, drains its copies and MMAs,
frees its tensor memory and returns. Nothing traps or hangs; the test then restores the
default budget and checks that the same calls on the same index give the normal results.
"""
import pytest
import torch

import inputs

pytestmark = pytest.mark.gpu

TIMEOUT = 6  # PACK3D_ERR_TIMEOUT
OK = 0


def _field():
    import geometry_aware_local_pack3d_b200 as p3d
    cfg = dict(grid=(8, 8, 16), block=(4, 4, 4), batch=1, heads=2, d=96, dtype="bf16",
               packing="random", qkv_std=96 ** -0.5, exclude_near=False)
    w = inputs.make_workload(cfg)
    ix = p3d.pack3d_build_index(p3d.make_geom(w["grid"], w["block"], 96),
                                coords=torch.from_numpy(w["coords"]).cuda())
    q, k, v, a = (w[n].to(torch.bfloat16).cuda().contiguous() for n in "qkva")
    dO = inputs.pack(inputs.upstream_grad(1, 2, w["grid"], 96), w["perm"])
    return p3d, w, ix, q, k, v, a, dO.to(torch.bfloat16).cuda().contiguous()


def _forward(p3d, ix, q, k, v, a):
    ksum, vsum, k_rot = p3d.pack3d_summarize_rotated(ix, k, v)
    out = p3d.pack3d_attn_fwd(ix, q, k_rot, v, a, ksum, vsum, k_rotated=True,
                              save_for_backward=True)
    return ksum, vsum, out


def test_forward_wait_timeout_is_reported_and_the_index_stays_usable():
    p3d, w, ix, q, k, v, a, _ = _field()
    _, _, ref = _forward(p3d, ix, q, k, v, a)
    torch.cuda.synchronize()
    assert p3d.pack3d_device_status(ix) == OK
    prev = p3d.pack3d_testing_set_wait_budget(1)
    try:
        _forward(p3d, ix, q, k, v, a)
        torch.cuda.synchronize()
    finally:
        p3d.pack3d_testing_set_wait_budget(prev)
    assert p3d.pack3d_device_status(ix) == TIMEOUT  # read and cleared
    assert p3d.pack3d_device_status(ix) == OK
    # the default budget is back; the local kernel's work counter was put back to zero by the
    # aborted launch's last CTA, so the same index gives the same results bit for bit
    _, _, again = _forward(p3d, ix, q, k, v, a)
    torch.cuda.synchronize()
    assert p3d.pack3d_device_status(ix) == OK
    for key in ("o", "o_loc", "o_glob", "lse_loc", "lse_glob"):
        assert torch.equal(again[key], ref[key]), key


def test_backward_wait_timeout_is_reported_and_the_index_stays_usable():
    p3d, w, ix, q, k, v, a, dO = _field()
    ksum, vsum, saved = _forward(p3d, ix, q, k, v, a)
    ref = p3d.pack3d_attn_bwd(ix, q, k, v, a, ksum, vsum, saved, dO)
    torch.cuda.synchronize()
    prev = p3d.pack3d_testing_set_wait_budget(1)
    try:
        p3d.pack3d_attn_bwd(ix, q, k, v, a, ksum, vsum, saved, dO)
        torch.cuda.synchronize()
    finally:
        p3d.pack3d_testing_set_wait_budget(prev)
    assert p3d.pack3d_device_status(ix) == TIMEOUT
    again = p3d.pack3d_attn_bwd(ix, q, k, v, a, ksum, vsum, saved, dO)
    torch.cuda.synchronize()
    assert p3d.pack3d_device_status(ix) == OK
    for key in ("dq", "dk", "dv", "dgate"):
        assert torch.equal(again[key], ref[key]), key


def test_wait_budget_hook_restores_the_default():
    import geometry_aware_local_pack3d_b200 as p3d
    prev = p3d.pack3d_testing_set_wait_budget(0)
    assert prev > 0
    assert p3d.pack3d_testing_set_wait_budget(0) == 4_000_000_000
