"""PACK3D attention on B200 (sm_100a): C-ABI library + thin ctypes binding.

The operator ("Geometry Matters in Packed 3D Attention", NeurIPS 2026) runs entirely in the
CUDA kernels of lib/libpack3d.so; this package only marshals torch tensors to the C calls.
"""
from .binding import (  # noqa: F401
    Index, Pack3DError, PACK3D_BF16, PACK3D_EXCLUDE_NEAR, PACK3D_F32, PACK3D_K_ROTATED,
    make_geom, lib, pack3d_attn_bwd, pack3d_attn_bwd_noalloc, pack3d_attn_fwd,
    pack3d_attn_global, pack3d_attn_local,
    pack3d_build_index, pack3d_bwd_workspace_bytes, pack3d_device_status, pack3d_index_bytes,
    pack3d_last_launch_count, pack3d_strerror, pack3d_summarize, pack3d_summarize_rotated,
    pack3d_testing_set_wait_budget,
    pack3d_summary_bytes, summary_rows, summary_tiles_shape,
)
