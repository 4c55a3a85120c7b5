"""ctypes binding of ``libatlas.so`` (declared in ``include/atlas.h``).

Argument marshalling only: shapes, dtypes and device pointers are read off
torch tensors (torch is used for device memory and streams) and passed to the
C-ABI; every step of the path runs in the library's CUDA kernels. There is no
CPU fallback: if the library has not been built, the first call raises.

Passages (page title, section) for each call are given in the header; in
short: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie 1
Fase 1 (temporally scaled RoPE), Fase 2 (cube reorder, window attention) and
Methodologie 2 (asymmetric hierarchical attention, position alignment).
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
# The in-tree build; ATLAS_LIBRARY may name another build of the same C-ABI.
LIB_PATH = os.environ.get("ATLAS_LIBRARY") or os.path.join(HERE, "libatlas.so")

OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_ALIAS, ERR_CUDA, \
    ERR_TIMEOUT, ERR_DEVICE, ERR_CAPACITY = range(10)
BF16, FP32 = 0, 1


class Grid3(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("W", ctypes.c_int64)]


class Cube3(ctypes.Structure):
    _fields_ = [("ct", ctypes.c_int32), ("ch", ctypes.c_int32), ("cw", ctypes.c_int32)]


class Rope(ctypes.Structure):
    _fields_ = [("theta", ctypes.c_double), ("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32),
                ("d_w", ctypes.c_int32), ("scale_t", ctypes.c_double),
                ("scale_h", ctypes.c_double), ("scale_w", ctypes.c_double)]


class AttnLayout(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("window_len", ctypes.c_int64),
                ("window_offsets", ctypes.c_void_p), ("n_windows", ctypes.c_int64),
                ("global_window_offsets", ctypes.c_void_p)]


def make_rope(theta, split, scales) -> Rope:
    d_t, d_h, d_w = (int(v) for v in split)
    s_t, s_h, s_w = (float(v) for v in scales)
    return Rope(float(theta), d_t, d_h, d_w, s_t, s_h, s_w)


class AtlasError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


def _declare(lib):
    lib.atlas_cube_reorder.restype = ctypes.c_int
    lib.atlas_cube_reorder.argtypes = [_vp, _vp, Grid3, Cube3, _i32, _i32, ctypes.c_int,
                                       ctypes.POINTER(Rope), _vp]
    lib.atlas_cube_reorder_noalloc.restype = ctypes.c_int
    lib.atlas_cube_reorder_noalloc.argtypes = lib.atlas_cube_reorder.argtypes
    lib.atlas_cube_unorder.restype = ctypes.c_int
    lib.atlas_cube_unorder.argtypes = [_vp, _vp, Grid3, Cube3, _i32, _i32, ctypes.c_int, _vp]
    lib.atlas_rope3d.restype = ctypes.c_int
    lib.atlas_rope3d.argtypes = [_vp, _vp, Grid3, _i32, _i32, ctypes.c_int,
                                 ctypes.POINTER(Rope), _vp]
    lib.atlas_local_global_attn.restype = ctypes.c_int
    lib.atlas_local_global_attn.argtypes = [_vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64,
                                            _i32, _i32, ctypes.c_float, ctypes.c_int, _vp, _vp,
                                            _vp, _vp]
    lib.atlas_local_global_attn_windows.restype = ctypes.c_int
    lib.atlas_local_global_attn_windows.argtypes = [_vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp, _vp,
                                                    _i64, _i32, _i32, ctypes.c_float, ctypes.c_int,
                                                    _vp, _vp, _vp, _vp]
    lib.atlas_local_global_attn_ex.restype = ctypes.c_int
    lib.atlas_local_global_attn_ex.argtypes = [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64,
                                               ctypes.POINTER(AttnLayout), _i32, _i32,
                                               ctypes.c_float, ctypes.c_int, _vp, _vp, _vp, _vp]
    lib.atlas_local_global_attn_bwd.restype = ctypes.c_int
    lib.atlas_local_global_attn_bwd.argtypes = (
        [_vp] * 5 + [_i64] + [_vp] * 5 + [_i64, ctypes.POINTER(AttnLayout), _i32, _i32,
                                         ctypes.c_float, ctypes.c_int, _vp, _vp] + [_vp] * 7)
    lib.atlas_qkv_proj_reorder.restype = ctypes.c_int
    lib.atlas_qkv_proj_reorder.argtypes = [_vp, _vp, _i64, Grid3, Cube3, _i32, _i32, _i32,
                                           ctypes.c_int, ctypes.POINTER(Rope), _vp, _vp, _vp,
                                           _vp]
    lib.atlas_out_proj_unorder.restype = ctypes.c_int
    lib.atlas_out_proj_unorder.argtypes = [_vp, _vp, _i64, Grid3, Cube3, _i32, _i32,
                                           ctypes.c_int, _vp, _vp]
    for name in ("atlas_aligned_global_reorder", "atlas_aligned_global_unorder"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [_vp, _vp, _i64, Grid3, Cube3, Grid3, _i32, _i32, ctypes.c_int,
                       ctypes.POINTER(Rope), _vp]
    lib.atlas_aligned_global_offsets.restype = ctypes.c_int
    lib.atlas_aligned_global_offsets.argtypes = [Grid3, Cube3, Grid3, _vp, _i64,
                                                 ctypes.POINTER(_i64)]
    lib.atlas_aligned_global_cube.restype = ctypes.c_int
    lib.atlas_aligned_global_cube.argtypes = [Grid3, Cube3, Grid3, ctypes.POINTER(Cube3)]
    lib.atlas_cube_reorder_batched.restype = ctypes.c_int
    lib.atlas_cube_reorder_batched.argtypes = [_vp, _vp, _i64, Grid3, Cube3, _i32, _i32,
                                               ctypes.c_int, ctypes.POINTER(Rope), _vp]
    lib.atlas_cube_unorder_batched.restype = ctypes.c_int
    lib.atlas_cube_unorder_batched.argtypes = [_vp, _vp, _i64, Grid3, Cube3, _i32, _i32,
                                               ctypes.c_int, _vp]
    lib.atlas_cube_unorder_rope.restype = ctypes.c_int
    lib.atlas_cube_unorder_rope.argtypes = [_vp, _vp, _i64, Grid3, Cube3, _i32, _i32,
                                            ctypes.c_int, ctypes.POINTER(Rope), _vp]
    lib.atlas_rope3d_batched.restype = ctypes.c_int
    lib.atlas_rope3d_batched.argtypes = [_vp, _vp, _i64, Grid3, _i32, _i32, ctypes.c_int,
                                         ctypes.POINTER(Rope), _vp]
    lib.atlas_cube_window_offsets.restype = ctypes.c_int
    lib.atlas_cube_window_offsets.argtypes = [Grid3, Cube3, _vp, _i64, ctypes.POINTER(_i64)]
    lib.atlas_status_string.restype = ctypes.c_char_p
    lib.atlas_status_string.argtypes = [ctypes.c_int]
    lib.atlas_last_device_error.restype = ctypes.c_int
    lib.atlas_last_device_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.atlas_debug_stall_next_attention.restype = ctypes.c_int
    lib.atlas_debug_stall_next_attention.argtypes = []
    lib.atlas_release_caches.restype = ctypes.c_int
    lib.atlas_release_caches.argtypes = []
    lib.atlas_cached_rope_tables.restype = ctypes.c_int64
    lib.atlas_cached_rope_tables.argtypes = []
    lib.atlas_version.restype = ctypes.c_int32
    lib.atlas_version.argtypes = []
    return lib


def lib():
    """The loaded library. Raises if ``libatlas.so`` has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m video_dit_windowed_b200.build` (no CPU fallback exists)")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def status_string(status: int) -> str:
    return lib().atlas_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != OK:
        raise AtlasError(status, where)


# ---------------------------------------------------------------------------
# torch-facing wrappers (torch only supplies pointers, shapes and streams)
# ---------------------------------------------------------------------------

def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(t, stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return ctypes.c_void_p(stream.cuda_stream)


def cube_reorder(src, dst, grid, cube, rope: Rope | None = None, stream=None):
    """Raster -> cube order of ``src`` [T*H*W, heads, head_dim] into ``dst``;
    with ``rope`` the rows are also rotated by 3D RoPE at their grid position."""
    n, heads, hd = src.shape
    st = lib().atlas_cube_reorder(
        _ptr(src), _ptr(dst), Grid3(*grid), Cube3(*cube), heads, hd, _dtype_code(src),
        ctypes.byref(rope) if rope is not None else None, _stream(src, stream))
    _check(st, "atlas_cube_reorder")
    return dst


def cube_reorder_noalloc(src, dst, grid, cube, rope: Rope | None = None, stream=None):
    """``cube_reorder`` through the entry point that allocates no device
    memory (its RoPE table sits in a fixed 32768-pair array shared by all
    calls on the device; overlapping calls race, see include/atlas.h)."""
    n, heads, hd = src.shape
    st = lib().atlas_cube_reorder_noalloc(
        _ptr(src), _ptr(dst), Grid3(*grid), Cube3(*cube), heads, hd, _dtype_code(src),
        ctypes.byref(rope) if rope is not None else None, _stream(src, stream))
    _check(st, "atlas_cube_reorder_noalloc")
    return dst


def cube_unorder(src, dst, grid, cube, stream=None):
    """Cube order -> raster order (exact inverse of ``cube_reorder``)."""
    n, heads, hd = src.shape
    st = lib().atlas_cube_unorder(_ptr(src), _ptr(dst), Grid3(*grid), Cube3(*cube), heads, hd,
                                  _dtype_code(src), _stream(src, stream))
    _check(st, "atlas_cube_unorder")
    return dst


def rope3d(src, dst, grid, rope: Rope, stream=None):
    """3D RoPE of raster-ordered tokens (``dst`` may be ``src``)."""
    n, heads, hd = src.shape
    st = lib().atlas_rope3d(_ptr(src), _ptr(dst), Grid3(*grid), heads, hd, _dtype_code(src),
                            ctypes.byref(rope), _stream(src, stream))
    _check(st, "atlas_rope3d")
    return dst


def local_global_attn(q_d, k_d, v_d, window_len, q_g, k_g, v_g, o_d, o_g, lse=None,
                      softmax_scale: float = 0.0, stream=None):
    """Asymmetric global-local attention; detail tensors in cube order.
    ``q_d`` (or ``q_g``) may have 0 rows. Returns (o_d, o_g, lse)."""
    ref = q_d if q_d is not None and q_d.shape[0] > 0 else q_g
    heads, hd = ref.shape[1], ref.shape[2]
    n_d = q_d.shape[0] if q_d is not None else 0
    n_g = q_g.shape[0] if q_g is not None else 0
    nz = lambda t, n: _ptr(t) if (t is not None and n > 0) else None
    st = lib().atlas_local_global_attn(
        nz(q_d, n_d), nz(k_d, n_d), nz(v_d, n_d), n_d, int(window_len),
        nz(q_g, n_g), nz(k_g, n_g), nz(v_g, n_g), n_g, heads, hd, float(softmax_scale),
        _dtype_code(ref), nz(o_d, n_d), nz(o_g, n_g), _ptr(lse), _stream(ref, stream))
    _check(st, "atlas_local_global_attn")
    return o_d, o_g, lse


def cube_window_offsets(grid, cube):
    """Window boundaries of the cube order as a host int32 tensor [n+1]
    (partial cubes at the far edges included)."""
    import torch
    n = _i64(0)
    _check(lib().atlas_cube_window_offsets(Grid3(*grid), Cube3(*cube), None, 0, ctypes.byref(n)),
           "atlas_cube_window_offsets")
    out = torch.empty(n.value + 1, dtype=torch.int32)
    _check(lib().atlas_cube_window_offsets(Grid3(*grid), Cube3(*cube),
                                           ctypes.c_void_p(out.data_ptr()), out.numel(),
                                           ctypes.byref(n)), "atlas_cube_window_offsets")
    return out


def local_global_attn_windows(q_d, k_d, v_d, window_offsets, q_g, k_g, v_g, o_d, o_g,
                              lse=None, softmax_scale: float = 0.0, stream=None):
    """Like ``local_global_attn`` with variable-length windows given by the
    device int32 tensor ``window_offsets`` [n_windows + 1]."""
    ref = q_d if q_d is not None and q_d.shape[0] > 0 else q_g
    heads, hd = ref.shape[1], ref.shape[2]
    n_d = q_d.shape[0] if q_d is not None else 0
    n_g = q_g.shape[0] if q_g is not None else 0
    nz = lambda t, n: _ptr(t) if (t is not None and n > 0) else None
    st = lib().atlas_local_global_attn_windows(
        nz(q_d, n_d), nz(k_d, n_d), nz(v_d, n_d), n_d, nz(window_offsets, n_d),
        window_offsets.numel() - 1 if window_offsets is not None else 0,
        nz(q_g, n_g), nz(k_g, n_g), nz(v_g, n_g), n_g, heads, hd, float(softmax_scale),
        _dtype_code(ref), nz(o_d, n_d), nz(o_g, n_g), _ptr(lse), _stream(ref, stream))
    _check(st, "atlas_local_global_attn_windows")
    return o_d, o_g, lse


def local_global_attn_ex(q_d, k_d, v_d, q_g, k_g, v_g, o_d, o_g, lse=None, *, batch=1,
                         window_len=0, window_offsets=None, global_window_offsets=None,
                         softmax_scale: float = 0.0, stream=None):
    """General layout: ``batch`` problems stacked along the rows (detail
    tensors [batch*N, heads, D], global [batch*G, heads, D], lse [batch,
    heads, N+G]); windows of ``window_len`` rows or the device int32
    ``window_offsets`` of one problem; with ``global_window_offsets`` (device
    int32 [n_windows+1], one problem) the queries of window w see only those
    global keys (the aligned variant)."""
    ref = q_d if q_d is not None and q_d.shape[0] > 0 else q_g
    heads, hd = ref.shape[1], ref.shape[2]
    n_d = (q_d.shape[0] if q_d is not None else 0) // batch
    n_g = (q_g.shape[0] if q_g is not None else 0) // batch
    nz = lambda t, n: _ptr(t) if (t is not None and n > 0) else None
    if window_offsets is not None:
        n_win = window_offsets.numel() - 1
    elif global_window_offsets is not None:
        n_win = global_window_offsets.numel() - 1
    else:
        n_win = 0
    wo = _ptr(window_offsets) if window_offsets is not None else None
    gwo = _ptr(global_window_offsets) if global_window_offsets is not None else None
    ly = AttnLayout(int(batch), int(window_len), wo.value if wo is not None else None,
                    int(n_win), gwo.value if gwo is not None else None)
    st = lib().atlas_local_global_attn_ex(
        nz(q_d, n_d), nz(k_d, n_d), nz(v_d, n_d), n_d, nz(q_g, n_g), nz(k_g, n_g), nz(v_g, n_g),
        n_g, ctypes.byref(ly), heads, hd, float(softmax_scale), _dtype_code(ref),
        nz(o_d, n_d), nz(o_g, n_g), _ptr(lse), _stream(ref, stream))
    _check(st, "atlas_local_global_attn_ex")
    return o_d, o_g, lse


def local_global_attn_bwd(q_d, k_d, v_d, o_d, do_d, q_g, k_g, v_g, o_g, do_g, lse,
                          dq_d, dk_d, dv_d, dq_g, dk_g, dv_g, delta=None, *, batch=1,
                          window_len=0, window_offsets=None, global_window_offsets=None,
                          softmax_scale: float = 0.0, stream=None):
    """Gradients of ``local_global_attn_ex`` (same layout arguments): fills
    dq_*, dk_*, dv_* from the forward's inputs, outputs ``o_*``, its ``lse``
    [batch, heads, N+G] and the output gradients ``do_*``. ``delta`` (fp32,
    shape of lse) is the workspace; allocated here when not given."""
    import torch
    ref = q_d if q_d is not None and q_d.shape[0] > 0 else q_g
    heads, hd = ref.shape[1], ref.shape[2]
    n_d = (q_d.shape[0] if q_d is not None else 0) // batch
    n_g = (q_g.shape[0] if q_g is not None else 0) // batch
    if delta is None:
        delta = torch.empty_like(lse)
    nz = lambda t, n: _ptr(t) if (t is not None and n > 0) else None
    if window_offsets is not None:
        n_win = window_offsets.numel() - 1
    elif global_window_offsets is not None:
        n_win = global_window_offsets.numel() - 1
    else:
        n_win = 0
    wo = _ptr(window_offsets) if window_offsets is not None else None
    gwo = _ptr(global_window_offsets) if global_window_offsets is not None else None
    ly = AttnLayout(int(batch), int(window_len), wo.value if wo is not None else None,
                    int(n_win), gwo.value if gwo is not None else None)
    st = lib().atlas_local_global_attn_bwd(
        nz(q_d, n_d), nz(k_d, n_d), nz(v_d, n_d), nz(o_d, n_d), nz(do_d, n_d), n_d,
        nz(q_g, n_g), nz(k_g, n_g), nz(v_g, n_g), nz(o_g, n_g), nz(do_g, n_g), n_g,
        ctypes.byref(ly), heads, hd, float(softmax_scale), _dtype_code(ref), _ptr(lse),
        _ptr(delta), nz(dq_d, n_d), nz(dk_d, n_d), nz(dv_d, n_d), nz(dq_g, n_g),
        nz(dk_g, n_g), nz(dv_g, n_g), _stream(ref, stream))
    _check(st, "atlas_local_global_attn_bwd")
    return dq_d, dk_d, dv_d, dq_g, dk_g, dv_g


def qkv_proj_reorder(x, w, grid, cube, q, k, v, rope: Rope | None = None, batch=1,
                     stream=None):
    """[Q | K | V] = x w^T with RoPE on Q and K and every row written at its
    cube position. x [batch*T*H*W, C] raster order; w [3*heads*head_dim, C];
    q, k, v [batch*T*H*W, heads, head_dim] (outputs)."""
    heads, hd = q.shape[1], q.shape[2]
    st = lib().atlas_qkv_proj_reorder(
        _ptr(x), _ptr(w), int(batch), Grid3(*grid), Cube3(*cube), x.shape[1], heads, hd,
        _dtype_code(x), ctypes.byref(rope) if rope is not None else None, _ptr(q), _ptr(k),
        _ptr(v), _stream(x, stream))
    _check(st, "atlas_qkv_proj_reorder")
    return q, k, v


def out_proj_unorder(o, w, grid, cube, y, batch=1, stream=None):
    """y = unorder(o) w^T: o [batch*T*H*W, heads, head_dim] (or [rows, C_in])
    in cube order, w [C_out, C_in], y [batch*T*H*W, C_out] raster order."""
    rows = o.shape[0]
    c_in = o.numel() // rows if rows else w.shape[1]
    st = lib().atlas_out_proj_unorder(_ptr(o), _ptr(w), int(batch), Grid3(*grid), Cube3(*cube),
                                      c_in, y.shape[1], _dtype_code(o), _ptr(y),
                                      _stream(o, stream))
    _check(st, "atlas_out_proj_unorder")
    return y


def aligned_global_reorder(src, dst, grid, cube, global_grid, rope: Rope | None = None,
                           batch=1, stream=None):
    """Global-proxy tokens (raster order of ``global_grid``) into the aligned
    order of ``grid`` cut into ``cube``; any grid ratios."""
    n, heads, hd = src.shape
    st = lib().atlas_aligned_global_reorder(
        _ptr(src), _ptr(dst), int(batch), Grid3(*grid), Cube3(*cube), Grid3(*global_grid), heads,
        hd, _dtype_code(src), ctypes.byref(rope) if rope is not None else None,
        _stream(src, stream))
    _check(st, "atlas_aligned_global_reorder")
    return dst


def aligned_global_unorder(src, dst, grid, cube, global_grid, rope: Rope | None = None,
                           batch=1, stream=None):
    """Inverse of ``aligned_global_reorder`` (optionally rotating, e.g. by the
    transposed RoPE for gradients)."""
    n, heads, hd = src.shape
    st = lib().atlas_aligned_global_unorder(
        _ptr(src), _ptr(dst), int(batch), Grid3(*grid), Cube3(*cube), Grid3(*global_grid), heads,
        hd, _dtype_code(src), ctypes.byref(rope) if rope is not None else None,
        _stream(src, stream))
    _check(st, "atlas_aligned_global_unorder")
    return dst


def aligned_global_offsets(grid, cube, global_grid):
    """Global key range of every detail window in the aligned order, as a
    host int32 tensor [n_windows + 1]."""
    import torch
    n = _i64(0)
    args = (Grid3(*grid), Cube3(*cube), Grid3(*global_grid))
    _check(lib().atlas_aligned_global_offsets(*args, None, 0, ctypes.byref(n)),
           "atlas_aligned_global_offsets")
    out = torch.empty(n.value + 1, dtype=torch.int32)
    _check(lib().atlas_aligned_global_offsets(*args, ctypes.c_void_p(out.data_ptr()),
                                              out.numel(), ctypes.byref(n)),
           "atlas_aligned_global_offsets")
    return out


def aligned_global_cube(grid, cube, global_grid):
    """The global-grid cube whose cubes are the aligned sets of the detail
    cubes (ratios must be integers dividing the cube)."""
    out = Cube3()
    _check(lib().atlas_aligned_global_cube(Grid3(*grid), Cube3(*cube), Grid3(*global_grid),
                                           ctypes.byref(out)), "atlas_aligned_global_cube")
    return (out.ct, out.ch, out.cw)


def cube_reorder_batched(src, dst, batch, grid, cube, rope: Rope | None = None, stream=None):
    """``cube_reorder`` of ``batch`` problems stacked along the rows."""
    n, heads, hd = src.shape
    st = lib().atlas_cube_reorder_batched(
        _ptr(src), _ptr(dst), int(batch), Grid3(*grid), Cube3(*cube), heads, hd,
        _dtype_code(src), ctypes.byref(rope) if rope is not None else None, _stream(src, stream))
    _check(st, "atlas_cube_reorder_batched")
    return dst


def cube_unorder_batched(src, dst, batch, grid, cube, stream=None):
    """``cube_unorder`` of ``batch`` problems stacked along the rows."""
    n, heads, hd = src.shape
    st = lib().atlas_cube_unorder_batched(_ptr(src), _ptr(dst), int(batch), Grid3(*grid),
                                          Cube3(*cube), heads, hd, _dtype_code(src),
                                          _stream(src, stream))
    _check(st, "atlas_cube_unorder_batched")
    return dst


def cube_unorder_rope(src, dst, grid, cube, rope: Rope, batch=1, stream=None):
    """Cube -> raster order with each row rotated at its raster position
    (with negated scales: the gradient of ``cube_reorder`` with RoPE)."""
    n, heads, hd = src.shape
    st = lib().atlas_cube_unorder_rope(_ptr(src), _ptr(dst), int(batch), Grid3(*grid),
                                       Cube3(*cube), heads, hd, _dtype_code(src),
                                       ctypes.byref(rope), _stream(src, stream))
    _check(st, "atlas_cube_unorder_rope")
    return dst


def transpose_rope(rope: Rope) -> Rope:
    """The same RoPE with negated position scales: rotation by -phi, the
    transpose (and inverse) of ``rope``."""
    return Rope(rope.theta, rope.d_t, rope.d_h, rope.d_w, -rope.scale_t, -rope.scale_h,
                -rope.scale_w)


def rope3d_batched(src, dst, batch, grid, rope: Rope, stream=None):
    """``rope3d`` of ``batch`` problems stacked along the rows."""
    n, heads, hd = src.shape
    st = lib().atlas_rope3d_batched(_ptr(src), _ptr(dst), int(batch), Grid3(*grid), heads, hd,
                                    _dtype_code(src), ctypes.byref(rope), _stream(src, stream))
    _check(st, "atlas_rope3d_batched")
    return dst


def last_device_error(stream=None) -> int:
    """Synchronise and read/clear the device error word (0 = clean)."""
    import torch
    s = ctypes.c_void_p(stream.cuda_stream if stream is not None
                        else torch.cuda.current_stream().cuda_stream)
    code = ctypes.c_uint32(0)
    st = lib().atlas_last_device_error(s, ctypes.byref(code))
    if st not in (OK, ERR_TIMEOUT):
        raise AtlasError(st, "atlas_last_device_error")
    return int(code.value)


def debug_stall_next_attention():
    """Test hook: the next bf16 attention launch leaves one K tile unloaded,
    so its bounded waits expire and it reports ATLAS_ERR_TIMEOUT."""
    _check(lib().atlas_debug_stall_next_attention(), "atlas_debug_stall_next_attention")


def cached_rope_tables() -> int:
    """RoPE tables the library holds in device memory it allocated."""
    return int(lib().atlas_cached_rope_tables())


def release_caches():
    _check(lib().atlas_release_caches(), "atlas_release_caches")


def version() -> int:
    return int(lib().atlas_version())
