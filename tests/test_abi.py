"""The C-ABI library loads, exports every symbol include/*.h declares, and rejects bad
arguments on the host before any launch. No GPU needed (no compute calls)."""
import ctypes
import glob
import os
import re

import pytest

from geometry_aware_local_pack3d_b200 import binding as b

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(pack3d_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_calls_the_pages_name():
    names = declared_functions()
    for n in ("pack3d_build_index", "pack3d_summarize", "pack3d_attn_fwd", "pack3d_attn_bwd"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = b.lib()
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_strerror_covers_every_status():
    for code in range(0, 9):
        assert b.pack3d_strerror(code) != "unknown status"


def test_index_bytes_rejects_bad_geometry():
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (9, 2, 2), 48), 512) == 0  # block > grid
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (2, 2, 2), 50), 512) == 0  # d % 6
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 2000), (2, 2, 2), 48), 512) == 0
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (2, 2, 2), 48), 513) == 0  # N > sites
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (2, 2, 2), 48, pool2=(1, -1, 1)),
                                512) == 0
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (2, 2, 2), 48,
                                            spacing=(1.0, -2.0, 1.0)), 512) == 0
    g = b.make_geom((8, 8, 8), (2, 2, 2), 48)
    g.summary_rope = 7
    assert b.pack3d_index_bytes(g, 512) == 0
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (2, 2, 2), 48), 512) > 512 * 27 * 4
    # partial blocks, a sparse field, a second pooling stage and summary-centre RoPE are valid
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (3, 2, 2), 48), 512) > 0
    assert b.pack3d_index_bytes(b.make_geom((8, 8, 8), (2, 2, 2), 48, pool2=(2, 2, 1),
                                            summary_rope="centre"), 300) > 0


def test_build_index_argument_errors_return_before_launch():
    L = b.lib()
    g = b.make_geom((4, 4, 4), (2, 2, 2), 48)
    out = b.pack3d_index()
    fake = ctypes.c_void_p(0x1000)
    # neither coords nor perm
    assert L.pack3d_build_index(ctypes.byref(g), None, None, 64, fake, 1 << 20,
                                ctypes.byref(out), None) == 1
    # both coords and perm
    assert L.pack3d_build_index(ctypes.byref(g), fake, fake, 64, fake, 1 << 20,
                                ctypes.byref(out), None) == 1
    # more tokens than lattice sites
    assert L.pack3d_build_index(ctypes.byref(g), fake, None, 65, fake, 1 << 20,
                                ctypes.byref(out), None) == 1
    # head_dim 42 is a multiple of 6 but unsupported
    g2 = b.make_geom((4, 4, 4), (2, 2, 2), 42)
    assert L.pack3d_build_index(ctypes.byref(g2), fake, None, 64, fake, 1 << 20,
                                ctypes.byref(out), None) == 2
    # buffer too small, misaligned buffer
    assert L.pack3d_build_index(ctypes.byref(g), fake, None, 64, fake, 16,
                                ctypes.byref(out), None) == 8
    assert L.pack3d_build_index(ctypes.byref(g), fake, None, 64, ctypes.c_void_p(0x1010),
                                1 << 20, ctypes.byref(out), None) == 5


def test_attn_calls_reject_bad_arguments_before_launch():
    L = b.lib()
    ix = b.pack3d_index()
    fake = ctypes.c_void_p(0x100000)
    # empty index struct
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 1, 1, 1, 0,
                             0.1, 0, fake, None, None, None, None, None) == 1
    ix.coord = ix.nbr = ix.members = ix.rope = 0x100000
    ix.sum_of = ix.groups = ix.count2 = ix.empty = ix.rope_c = 0x100000
    ix.geom = b.make_geom((4, 4, 4), (2, 2, 2), 48)
    ix.n, ix.m = 64, 8
    # bad dtype, bad batch, misaligned pointer, bad flags, null workspace
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 7, 1, 1, 0,
                             0.1, 0, fake, None, None, None, None, None) == 1
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 1, 0, 1, 0,
                             0.1, 0, fake, None, None, None, None, None) == 1
    assert L.pack3d_attn_fwd(ctypes.byref(ix), ctypes.c_void_p(0x100004), fake, fake, fake, fake,
                             fake, 1, 1, 1, 0, 0.1, 0, fake, None, None, None, None, None) == 5
    # KV heads that do not divide the query heads
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 1, 1, 4, 3,
                             0.1, 0, fake, None, None, None, None, None) == 1
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 1, 1, 4, 8,
                             0.1, 0, fake, None, None, None, None, None) == 1
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 1, 1, 1, 0,
                             0.1, 8, fake, None, None, None, None, None) == 1
    assert L.pack3d_summarize(ctypes.byref(ix), fake, None, 1, 1, 1, fake, fake, None) == 1
    # rotated keys: no output buffer, output aliasing the input keys, misaligned output
    assert L.pack3d_summarize_rotated(ctypes.byref(ix), fake, fake, 1, 1, 1, fake, fake, None,
                                      None) == 1
    assert L.pack3d_summarize_rotated(ctypes.byref(ix), fake, fake, 1, 1, 1, fake, fake, fake,
                                      None) == 1
    assert L.pack3d_summarize_rotated(ctypes.byref(ix), fake, fake, 1, 1, 1, fake, fake,
                                      ctypes.c_void_p(0x100008), None) == 5
    # split calls: missing output, wrong flags for each half
    assert L.pack3d_attn_local(ctypes.byref(ix), fake, fake, fake, 1, 1, 1, 0, 0.1, 0, None,
                               None, None) == 1
    assert L.pack3d_attn_local(ctypes.byref(ix), fake, fake, fake, 1, 1, 1, 0, 0.1,
                               b.PACK3D_EXCLUDE_NEAR, fake, None, None) == 1
    assert L.pack3d_attn_global(ctypes.byref(ix), fake, None, fake, fake, fake, 1, 1, 1, 0, 0.1,
                                0, fake, None, None, None) == 1
    assert L.pack3d_attn_global(ctypes.byref(ix), fake, fake, fake, fake, fake, 1, 1, 1, 0, 0.1,
                                b.PACK3D_K_ROTATED, fake, None, None, None) == 1
    # PACK3D_K_ROTATED is a bf16 tensor-core feature: fp32 is refused before any launch
    assert L.pack3d_attn_fwd(ctypes.byref(ix), fake, fake, fake, fake, fake, fake, 0, 1, 1, 0,
                             0.1, b.PACK3D_K_ROTATED, fake, None, None, None, None, None) == 2
    assert L.pack3d_attn_bwd(ctypes.byref(ix), *([fake] * 8), None, None, fake, 1, 1, 1, 0, 0.1,
                             0, fake, fake, fake, fake, fake, 1 << 30, None) == 1
    assert b.pack3d_bwd_workspace_bytes(ix, 1, 1, 1) > 0
    # GQA adds the per-query-head key gradients to the workspace; bad KV head counts give 0
    assert b.pack3d_bwd_workspace_bytes(ix, 1, 1, 4, 2) > b.pack3d_bwd_workspace_bytes(ix, 1, 1, 4)
    assert b.pack3d_bwd_workspace_bytes(ix, 1, 1, 4, 3) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(b, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(b, "_lib", None)
    with pytest.raises(ImportError):
        b.lib()
