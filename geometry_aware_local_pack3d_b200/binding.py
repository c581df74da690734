"""ctypes binding of the PACK3D C ABI (include/pack3d.h).

Argument marshalling only: torch tensors supply device memory and the current CUDA stream;
every step of the operator runs in the library's kernels. The functions carry the C names.
There is no CPU fallback: if the shared library is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libpack3d.so")

PACK3D_OK = 0
PACK3D_F32 = 0
PACK3D_BF16 = 1
PACK3D_EXCLUDE_NEAR = 1
PACK3D_K_ROTATED = 2
PACK3D_ROPE_TOKEN = 0
PACK3D_ROPE_CENTRE = 1

STATUS_NAMES = {0: "PACK3D_OK", 1: "PACK3D_ERR_INVALID_ARG", 2: "PACK3D_ERR_UNSUPPORTED",
                3: "PACK3D_ERR_DUP_COORD", 4: "PACK3D_ERR_COORD_RANGE", 5: "PACK3D_ERR_ALIGN",
                6: "PACK3D_ERR_TIMEOUT", 7: "PACK3D_ERR_CUDA", 8: "PACK3D_ERR_WORKSPACE"}


class Pack3DError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} "
                         f"({lib().pack3d_strerror(status).decode()})")


class pack3d_geom(ctypes.Structure):
    _fields_ = [("gz", ctypes.c_int32), ("gy", ctypes.c_int32), ("gx", ctypes.c_int32),
                ("bz", ctypes.c_int32), ("by", ctypes.c_int32), ("bx", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("rope_base", ctypes.c_float),
                ("pz", ctypes.c_int32), ("py", ctypes.c_int32), ("px", ctypes.c_int32),
                ("summary_rope", ctypes.c_int32), ("spacing", ctypes.c_float * 3)]


_P = ctypes.c_void_p


class pack3d_index(ctypes.Structure):
    _fields_ = [("geom", pack3d_geom), ("n", ctypes.c_int64), ("m", ctypes.c_int64),
                ("n_blocks", ctypes.c_int64), ("block_volume", ctypes.c_int32),
                ("rope_pairs", ctypes.c_int32), ("rope_rows", ctypes.c_int32),
                ("group_volume", ctypes.c_int32), ("sum_ext", ctypes.c_int32 * 3),
                ("sum_grid", ctypes.c_int32 * 3), ("n_empty", ctypes.c_int32),
                ("reserved", ctypes.c_int32),
                ("coord", _P), ("inv", _P), ("nbr", _P), ("block_of", _P), ("slot_of", _P),
                ("members", _P), ("count", _P), ("sum_of", _P), ("groups", _P),
                ("count2", _P), ("empty", _P), ("rope", _P), ("rope_c", _P), ("status", _P)]


_lib = None


def lib():
    """Load libpack3d.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"PACK3D CUDA library not built: {_LIB_PATH} is missing "
                              "(run python -m geometry_aware_local_pack3d_b200.build)")
        L = ctypes.CDLL(_LIB_PATH)
        st, sz, i32, i64, u32, f32 = (ctypes.c_int, ctypes.c_size_t, ctypes.c_int32,
                                      ctypes.c_int64, ctypes.c_uint32, ctypes.c_float)
        gp, ip = ctypes.POINTER(pack3d_geom), ctypes.POINTER(pack3d_index)
        L.pack3d_strerror.restype = ctypes.c_char_p
        L.pack3d_strerror.argtypes = [st]
        L.pack3d_index_bytes.restype = sz
        L.pack3d_index_bytes.argtypes = [gp, i64]
        L.pack3d_build_index.restype = st
        L.pack3d_build_index.argtypes = [gp, _P, _P, i64, _P, sz, ip, _P]
        L.pack3d_summarize.restype = st
        L.pack3d_summarize.argtypes = [ip, _P, _P, st, st, st, _P, _P, _P]
        L.pack3d_attn_fwd.restype = st
        L.pack3d_attn_local.restype = st
        L.pack3d_attn_local.argtypes = [ip, _P, _P, _P, st, st, st, st, f32, u32, _P, _P, _P]
        L.pack3d_attn_global.restype = st
        L.pack3d_attn_global.argtypes = [ip, _P, _P, _P, _P, _P, st, st, st, st, f32, u32, _P,
                                         _P, _P, _P]
        L.pack3d_summarize_rotated.restype = st
        L.pack3d_summarize_rotated.argtypes = [ip, _P, _P, st, st, st, _P, _P, _P, _P]
        L.pack3d_attn_fwd.argtypes = [ip, _P, _P, _P, _P, _P, _P, st, st, st, st, f32, u32, _P,
                                      _P, _P, _P, _P, _P]
        L.pack3d_summary_bytes.restype = sz
        L.pack3d_summary_bytes.argtypes = [ip, st, st, st]
        L.pack3d_bwd_workspace_bytes.restype = sz
        L.pack3d_bwd_workspace_bytes.argtypes = [ip, st, st, st, st]
        L.pack3d_attn_bwd.restype = st
        L.pack3d_attn_bwd.argtypes = [ip, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, st, st, st,
                                      st, f32, u32, _P, _P, _P, _P, _P, sz, _P]
        L.pack3d_attn_bwd_noalloc.restype = st
        L.pack3d_attn_bwd_noalloc.argtypes = [ip, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, st,
                                              st, st, st, f32, u32, _P, _P, _P, _P, _P]
        L.pack3d_device_status.restype = st
        L.pack3d_device_status.argtypes = [ip, _P]
        L.pack3d_last_launch_count.restype = ctypes.c_int
        L.pack3d_last_launch_count.argtypes = []
        L.pack3d_testing_set_wait_budget.restype = ctypes.c_longlong
        L.pack3d_testing_set_wait_budget.argtypes = [ctypes.c_longlong]
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, where):
    if status != PACK3D_OK:
        raise Pack3DError(status, where)


def _dtype_code(t):
    if t.dtype == torch.float32:
        return PACK3D_F32
    if t.dtype == torch.bfloat16:
        return PACK3D_BF16
    raise TypeError(f"PACK3D supports float32 and bfloat16 tensors, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("PACK3D tensors must be contiguous CUDA tensors")


class Index:
    """A built index: the device buffer (owned by torch) plus the filled C struct."""

    def __init__(self, buf, struct):
        self.buf = buf
        self.struct = struct

    @property
    def n(self):
        return int(self.struct.n)

    @property
    def m(self):
        return int(self.struct.m)

    def table(self, name, shape):
        """View one device table (int32) of the index as a torch tensor (for checks)."""
        base = self.buf.data_ptr()
        off = getattr(self.struct, name) - base
        count = int(torch.tensor(shape).prod())
        return self.buf[off:off + 4 * count].view(torch.int32).view(*shape)

    def rope_table(self):
        """[3 axes, rope_rows, pairs, 2] (cos, sin) of the per-axis RoPE angles."""
        base = self.buf.data_ptr()
        off = self.struct.rope - base
        rows, pairs = int(self.struct.rope_rows), int(self.struct.rope_pairs)
        return self.buf[off:off + 24 * rows * pairs].view(torch.float32).view(3, rows, pairs, 2)

    def centre_table(self):
        """[M, d/2, 2] (cos, sin) of the summary-centre angles."""
        base = self.buf.data_ptr()
        off = self.struct.rope_c - base
        m, half = self.m, int(self.struct.geom.head_dim) // 2
        return self.buf[off:off + 8 * m * half].view(torch.float32).view(m, half, 2)


def make_geom(grid, block, head_dim, rope_base=10000.0, pool2=(1, 1, 1), summary_rope="token",
              spacing=(1.0, 1.0, 1.0)):
    """pool2: second pooling stage (groups of blocks); summary_rope: "token" or "centre";
    spacing: per-axis scale of the RoPE coordinate."""
    sr = {"token": PACK3D_ROPE_TOKEN, "centre": PACK3D_ROPE_CENTRE}[summary_rope]
    return pack3d_geom(int(grid[0]), int(grid[1]), int(grid[2]), int(block[0]), int(block[1]),
                       int(block[2]), int(head_dim), float(rope_base), int(pool2[0]),
                       int(pool2[1]), int(pool2[2]), sr,
                       (ctypes.c_float * 3)(*[float(x) for x in spacing]))


def pack3d_index_bytes(geom, n):
    return int(lib().pack3d_index_bytes(ctypes.byref(geom), int(n)))


def pack3d_build_index(geom, coords=None, perm=None, stream=None):
    """coords: int32 CUDA [N,3] or perm: int64 CUDA [N]. Returns an :class:`Index`."""
    src = coords if coords is not None else perm
    if src is None:
        raise ValueError("pass coords or perm")
    _need_cuda(src)
    n = src.shape[0]
    nbytes = pack3d_index_bytes(geom, n)
    if nbytes == 0:
        raise Pack3DError(1, "pack3d_index_bytes")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=src.device)
    st = pack3d_index()
    status = lib().pack3d_build_index(ctypes.byref(geom), _ptr(coords), _ptr(perm), int(n),
                                      _ptr(buf), nbytes, ctypes.byref(st), _stream(stream))
    _check(status, "pack3d_build_index")
    return Index(buf, st)


def summary_tiles_shape(index, batch, heads, d):
    """Shape of a summary buffer: [B, H, T, d/8, 64, 8] with T = ceil(M / 64) (summary tiles)."""
    return (batch, heads, (index.m + 63) // 64, d // 8, 64, 8)


def summary_rows(tiles, m):
    """Plain [B, H, M, d] view (a copy) of a summary-tile buffer, for inspection and tests."""
    B, H, T, dc, _, _ = tiles.shape
    return tiles.permute(0, 1, 2, 4, 3, 5).reshape(B, H, T * 64, dc * 8)[:, :, :m]


def pack3d_summary_bytes(index, dtype_code, batch, heads):
    st = index.struct if isinstance(index, Index) else index
    return int(lib().pack3d_summary_bytes(ctypes.byref(st), dtype_code, batch, heads))


def pack3d_summarize(index, k, v, ksum=None, vsum=None, stream=None):
    """Block summaries of k, v into summary-tile buffers (allocated here when not given)."""
    _need_cuda(k, v)
    B, H, N, d = k.shape
    shape = summary_tiles_shape(index, B, H, d)
    if ksum is None:
        ksum = torch.empty(shape, dtype=k.dtype, device=k.device)
    if vsum is None:
        vsum = torch.empty(shape, dtype=k.dtype, device=k.device)
    need = pack3d_summary_bytes(index, _dtype_code(k), B, H)
    for t in (ksum, vsum):
        if t.numel() * t.element_size() < need:
            raise ValueError(f"summary buffer holds {t.numel() * t.element_size()} bytes, "
                             f"needs {need}")
    _check(lib().pack3d_summarize(ctypes.byref(index.struct), _ptr(k), _ptr(v), _dtype_code(k),
                                  B, H, _ptr(ksum), _ptr(vsum), _stream(stream)),
           "pack3d_summarize")
    return ksum, vsum


def pack3d_summarize_rotated(index, k, v, ksum=None, vsum=None, k_rot=None, stream=None):
    """Block summaries plus the rotated keys R(c) k in one pass; returns (ksum, vsum, k_rot)."""
    _need_cuda(k, v)
    B, H, N, d = k.shape
    shape = summary_tiles_shape(index, B, H, d)
    if ksum is None:
        ksum = torch.empty(shape, dtype=k.dtype, device=k.device)
    if vsum is None:
        vsum = torch.empty(shape, dtype=k.dtype, device=k.device)
    if k_rot is None:
        k_rot = torch.empty_like(k)
    need = pack3d_summary_bytes(index, _dtype_code(k), B, H)
    for t in (ksum, vsum):
        if t.numel() * t.element_size() < need:
            raise ValueError(f"summary buffer holds {t.numel() * t.element_size()} bytes, "
                             f"needs {need}")
    _check(lib().pack3d_summarize_rotated(ctypes.byref(index.struct), _ptr(k), _ptr(v),
                                          _dtype_code(k), B, H, _ptr(ksum), _ptr(vsum),
                                          _ptr(k_rot), _stream(stream)),
           "pack3d_summarize_rotated")
    return ksum, vsum, k_rot


def pack3d_attn_fwd(index, q, k, v, gate, ksum, vsum, *, scale=None, exclude_near=False,
                    k_rotated=False, o=None, lse_loc=None, lse_glob=None, o_loc=None,
                    o_glob=None, save_for_backward=False, stream=None):
    """Returns a dict with o and, when requested, lse_loc, lse_glob, o_loc, o_glob.
    k_rotated: k is the k_rot of pack3d_summarize_rotated (bf16, tensor-core path)."""
    _need_cuda(q, k, v, gate, ksum, vsum)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dev = q.device
    if o is None:
        o = torch.empty_like(q)
    if save_for_backward:
        lse_loc = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse_loc is None else lse_loc
        lse_glob = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse_glob is None else lse_glob
        o_loc = torch.empty_like(q) if o_loc is None else o_loc
        o_glob = torch.empty_like(q) if o_glob is None else o_glob
    flags = (PACK3D_EXCLUDE_NEAR if exclude_near else 0) | (PACK3D_K_ROTATED if k_rotated else 0)
    _check(lib().pack3d_attn_fwd(ctypes.byref(index.struct), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(gate), _ptr(ksum), _ptr(vsum), _dtype_code(q), B, H,
                                 k.shape[1], scale, flags, _ptr(o), _ptr(lse_loc),
                                 _ptr(lse_glob), _ptr(o_loc), _ptr(o_glob), _stream(stream)),
           "pack3d_attn_fwd")
    return dict(o=o, lse_loc=lse_loc, lse_glob=lse_glob, o_loc=o_loc, o_glob=o_glob)


def pack3d_attn_local(index, q, k, v, *, scale=None, k_rotated=False, o_loc=None,
                      lse_loc=None, stream=None):
    """Local branch alone: returns (o_loc, lse_loc); lse_loc only when a buffer is passed."""
    _need_cuda(q, k, v)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o_loc is None:
        o_loc = torch.empty_like(q)
    flags = PACK3D_K_ROTATED if k_rotated else 0
    _check(lib().pack3d_attn_local(ctypes.byref(index.struct), _ptr(q), _ptr(k), _ptr(v),
                                   _dtype_code(q), B, H, k.shape[1], scale, flags, _ptr(o_loc),
                                   _ptr(lse_loc), _stream(stream)), "pack3d_attn_local")
    return o_loc, lse_loc


def pack3d_attn_global(index, q, gate, ksum, vsum, o_loc, *, scale=None, exclude_near=False,
                       o=None, lse_glob=None, o_glob=None, stream=None):
    """Global branch + mixer over a given o_loc (o may be o_loc itself): returns o. The
    summaries' head count (ksum.shape[1]) is the KV head count."""
    _need_cuda(q, gate, ksum, vsum, o_loc)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    if o is None:
        o = torch.empty_like(q)
    flags = PACK3D_EXCLUDE_NEAR if exclude_near else 0
    _check(lib().pack3d_attn_global(ctypes.byref(index.struct), _ptr(q), _ptr(gate), _ptr(ksum),
                                    _ptr(vsum), _ptr(o_loc), _dtype_code(q), B, H, ksum.shape[1],
                                    scale, flags, _ptr(o), _ptr(lse_glob), _ptr(o_glob),
                                    _stream(stream)), "pack3d_attn_global")
    return o


def pack3d_bwd_workspace_bytes(index, dtype_code, batch, heads, kv_heads=0):
    st = index.struct if isinstance(index, Index) else index
    return int(lib().pack3d_bwd_workspace_bytes(ctypes.byref(st), dtype_code, batch, heads,
                                                kv_heads))


def pack3d_attn_bwd(index, q, k, v, gate, ksum, vsum, saved, dO, *, scale=None,
                    exclude_near=False, workspace=None, stream=None):
    """saved: the dict returned by pack3d_attn_fwd(save_for_backward=True)."""
    _need_cuda(q, k, v, gate, ksum, vsum, dO)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    code = _dtype_code(q)
    nbytes = pack3d_bwd_workspace_bytes(index, code, B, H, k.shape[1])
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dgate = torch.empty_like(gate)
    flags = PACK3D_EXCLUDE_NEAR if exclude_near else 0
    _check(lib().pack3d_attn_bwd(ctypes.byref(index.struct), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(gate), _ptr(ksum), _ptr(vsum), _ptr(saved["o_loc"]),
                                 _ptr(saved["o_glob"]), _ptr(saved["lse_loc"]),
                                 _ptr(saved["lse_glob"]), _ptr(dO), code, B, H, k.shape[1],
                                 scale, flags, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgate),
                                 _ptr(workspace), workspace.numel(), _stream(stream)),
           "pack3d_attn_bwd")
    return dict(dq=dq, dk=dk, dv=dv, dgate=dgate)


def pack3d_attn_bwd_noalloc(index, q, k, v, gate, ksum, vsum, saved, dO, *, scale=None,
                            exclude_near=False, stream=None):
    """pack3d_attn_bwd with the library's built-in scratch buffer (no workspace argument)."""
    _need_cuda(q, k, v, gate, ksum, vsum, dO)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dgate = torch.empty_like(gate)
    flags = PACK3D_EXCLUDE_NEAR if exclude_near else 0
    _check(lib().pack3d_attn_bwd_noalloc(ctypes.byref(index.struct), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(gate), _ptr(ksum), _ptr(vsum), _ptr(saved["o_loc"]),
                                         _ptr(saved["o_glob"]), _ptr(saved["lse_loc"]),
                                         _ptr(saved["lse_glob"]), _ptr(dO), _dtype_code(q), B, H,
                                         k.shape[1], scale, flags, _ptr(dq), _ptr(dk), _ptr(dv),
                                         _ptr(dgate), _stream(stream)), "pack3d_attn_bwd_noalloc")
    return dict(dq=dq, dk=dk, dv=dv, dgate=dgate)


NOALLOC_SCRATCH_BYTES = 32 << 20


def pack3d_device_status(index, stream=None):
    return int(lib().pack3d_device_status(ctypes.byref(index.struct), _stream(stream)))


def pack3d_last_launch_count():
    return int(lib().pack3d_last_launch_count())


def pack3d_testing_set_wait_budget(cycles):
    """Testing hook: SM-cycle budget of the kernels' device-side waits (<= 0: default)."""
    return int(lib().pack3d_testing_set_wait_budget(int(cycles)))


def pack3d_strerror(status):
    return lib().pack3d_strerror(int(status)).decode()
