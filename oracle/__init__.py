"""fp64 CPU oracle for AtlasVid's detail-branch attention path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline legs of ``bench.py`` may import this package. The CUDA library in
``video_dit_windowed_b200`` never imports it, and the two share no code: this
package compiles and wraps the plain C file ``atlas_oracle.c`` (see its header
for the passages each function follows and the readings it takes).

Pages cited (title, section):
  * "Technische Samenvatting: AtlasVid" (gist.science; same text in the French
    "Resume Technique" and Portuguese "Resumo Tecnico"), Methodologie 1
    (Fase 1: temporally scaled RoPE; Fase 2: cube reorder and window
    attention) and 2 (asymmetric hierarchical attention, position alignment).
  * "AtlasVid: Efficient Ultra-High-Resolution Long Video Generation via
    Decoupled Global-Local Modeling", abstract.
  * The projections on either side of the path (QKV in, output out) are the
    attention layer's linear maps; the summary's training strategy adapts
    exactly these ("attention projections"). Their oracle is numpy's matmul
    composed with the pinned reorder and RoPE functions.

Every function takes and returns numpy arrays; floating-point inputs are
converted to float64 exactly before the C code sees them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "atlas_oracle.c")
BUILD_DIR = os.path.join(_HERE, "_build")
LIB_PATH = os.path.join(BUILD_DIR, "liboracle_atlas.so")

_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_f64 = ctypes.c_double
_ptr = ctypes.c_void_p


def build(source: str = SOURCE, out: str = LIB_PATH, extra_flags=()) -> str:
    """Compile ``source`` into the shared library ``out`` with gcc (-O2, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           *extra_flags, "-o", out, source, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _declare(lib):
    lib.atlas_oracle_cube_position.restype = _i64
    lib.atlas_oracle_cube_position.argtypes = [_i64] * 7
    lib.atlas_oracle_cube_windows.restype = _i64
    lib.atlas_oracle_cube_windows.argtypes = [_i64] * 6 + [_ptr]
    lib.atlas_oracle_cube_positions.restype = None
    lib.atlas_oracle_cube_positions.argtypes = [_i64] * 6 + [_ptr]
    for name in ("atlas_oracle_cube_reorder", "atlas_oracle_cube_unorder"):
        fn = getattr(lib, name)
        fn.restype = ctypes.c_int
        fn.argtypes = [_ptr, _ptr] + [_i64] * 7
    lib.atlas_oracle_rope3d_rows.restype = None
    lib.atlas_oracle_rope3d_rows.argtypes = (
        [_ptr, _ptr, _i64, _ptr] + [_i64] * 5 + [_f64] + [_i64] * 3 + [_f64] * 3)
    lib.atlas_oracle_attention_head_windows.restype = ctypes.c_int
    lib.atlas_oracle_attention_head_windows.argtypes = (
        [_i64, _i64, _ptr, _i64, _i64, _i64, _f64, _ptr, _ptr, _i64, _i64, _ptr, _ptr,
         _i64, _ptr, _ptr, _ptr, _ptr, ctypes.c_int])
    lib.atlas_oracle_attention_head_aligned.restype = ctypes.c_int
    lib.atlas_oracle_attention_head_aligned.argtypes = (
        [_i64] * 10 + [_f64, _ptr, _ptr, _i64, _i64, _ptr, _ptr, _i64, _ptr, _ptr, _ptr, _ptr,
                       ctypes.c_int])
    lib.atlas_oracle_attention_bwd_head_windows.restype = ctypes.c_int
    lib.atlas_oracle_attention_bwd_head_windows.argtypes = (
        [_i64, _i64, _ptr, _i64, _i64, _i64, _f64] + [_ptr] * 7 + [ctypes.c_int])
    lib.atlas_oracle_attention_bwd_head_aligned.restype = ctypes.c_int
    lib.atlas_oracle_attention_bwd_head_aligned.argtypes = (
        [_i64] * 10 + [_f64] + [_ptr] * 7 + [ctypes.c_int])
    lib.atlas_oracle_attention_bwd_head_sampled.restype = ctypes.c_int
    lib.atlas_oracle_attention_bwd_head_sampled.argtypes = (
        [_i64, _i64, _ptr, _i64, _i64, _i64, _f64] + [_ptr] * 4 + [_i64, _ptr, _i64, _ptr]
        + [_ptr] * 3 + [ctypes.c_int])
    lib.atlas_oracle_attention_head.restype = ctypes.c_int
    lib.atlas_oracle_attention_head.argtypes = (
        [_i64, _i64, _i64, _i64, _f64, _ptr, _ptr, _i64, _i64, _ptr, _ptr,
         _i64, _ptr, _ptr, _ptr, _ptr, ctypes.c_int])
    lib.atlas_oracle_max_threads.restype = ctypes.c_int
    lib.atlas_oracle_max_threads.argtypes = []
    return lib


def load(path: str | None = None):
    """Load (building first if missing or stale) the oracle library."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            stale = (not os.path.exists(LIB_PATH)
                     or os.path.getmtime(LIB_PATH) < os.path.getmtime(SOURCE))
            if stale:
                build()
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


class Oracle:
    """numpy front end over one loaded copy of the oracle library."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    # -- cube reorder ---------------------------------------------------
    def cube_positions(self, grid, cube) -> np.ndarray:
        """pos[r] = cube-contiguous position of raster token r."""
        T, H, W = grid
        n = T * H * W
        pos = np.empty(n, dtype=np.int64)
        self.lib.atlas_oracle_cube_positions(T, H, W, *cube, pos.ctypes.data)
        return pos

    def cube_windows(self, grid, cube) -> np.ndarray:
        """offsets[c] = first cube-order position of cube c; the last entry
        is T*H*W (partial cubes at the far edges included)."""
        T, H, W = grid
        ct, ch, cw = cube
        n = -(-T // ct) * -(-H // ch) * -(-W // cw)
        off = np.empty(n + 1, dtype=np.int64)
        got = self.lib.atlas_oracle_cube_windows(T, H, W, ct, ch, cw, off.ctypes.data)
        assert got == n
        return off

    def cube_position(self, grid, cube, r: int) -> int:
        return int(self.lib.atlas_oracle_cube_position(*grid, *cube, int(r)))

    def _permute(self, fn, x: np.ndarray, grid, cube) -> np.ndarray:
        T, H, W = grid
        x = np.ascontiguousarray(x)
        if x.shape[0] != T * H * W:
            raise ValueError("leading dim must be T*H*W")
        out = np.empty_like(x)
        row_bytes = x.nbytes // max(1, x.shape[0])
        if fn(x.ctypes.data, out.ctypes.data, T, H, W, *cube, row_bytes) != 0:
            raise RuntimeError("cube positions are not a permutation")
        return out

    def cube_reorder(self, x: np.ndarray, grid, cube) -> np.ndarray:
        """Byte-exact permutation of rows of ``x`` (raster -> cube order)."""
        return self._permute(self.lib.atlas_oracle_cube_reorder, x, grid, cube)

    def cube_unorder(self, x: np.ndarray, grid, cube) -> np.ndarray:
        """Byte-exact inverse permutation (cube order -> raster)."""
        return self._permute(self.lib.atlas_oracle_cube_unorder, x, grid, cube)

    # -- RoPE -----------------------------------------------------------
    def rope3d_rows(self, x: np.ndarray, raster_idx, grid, theta: float,
                    split, scales) -> np.ndarray:
        """3D RoPE of rows ``x`` [n, heads, head_dim] at raster indices
        ``raster_idx`` of ``grid``; ``split`` = (d_t, d_h, d_w); ``scales`` =
        (s_t, s_h, s_w). Returns float64 [n, heads, head_dim]."""
        x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
        n, heads, head_dim = x.shape
        idx = np.ascontiguousarray(np.asarray(raster_idx, dtype=np.int64))
        assert idx.shape == (n,)
        y = np.empty_like(x)
        T, H, W = grid
        self.lib.atlas_oracle_rope3d_rows(
            x.ctypes.data, y.ctypes.data, n, idx.ctypes.data, T, H, W,
            heads, head_dim, float(theta), *[int(d) for d in split],
            *[float(s) for s in scales])
        return y

    def rope3d_grid(self, x: np.ndarray, grid, theta, split, scales):
        """3D RoPE of a whole raster-ordered grid ``x`` [T*H*W, heads, D]."""
        n = x.shape[0]
        return self.rope3d_rows(x, np.arange(n, dtype=np.int64), grid, theta,
                                split, scales)

    # -- attention ------------------------------------------------------
    def attention_head(self, n_detail: int, window_len: int, n_global: int,
                       scale: float, k_d, v_d, kd_lo: int, k_g, v_g, q_ids,
                       q, n_threads: int = 1, win_off=None):
        """Asymmetric global-local attention for one head.

        ``k_d``/``v_d``: detail rows ``kd_lo .. kd_lo+len-1`` [rows, D];
        ``k_g``/``v_g``: all global rows [G, D]; ``q_ids``: query ids in
        [0, N+G) (>= N means global row id-N); ``q``: [n_q, D]. Windows are
        ``window_len`` consecutive detail positions, or the ranges of
        ``win_off`` (n_win+1 offsets) when given.
        Returns (o [n_q, D] float64, lse [n_q] float64, natural log).
        """
        f = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float64))
        q = f(q)
        n_q, D = q.shape
        k_d = f(k_d).reshape(-1, D) if k_d is not None else np.zeros((0, D))
        v_d = f(v_d).reshape(-1, D) if v_d is not None else np.zeros((0, D))
        k_g = f(k_g).reshape(-1, D) if k_g is not None else np.zeros((0, D))
        v_g = f(v_g).reshape(-1, D) if v_g is not None else np.zeros((0, D))
        assert k_d.shape == v_d.shape and k_g.shape == v_g.shape
        assert k_g.shape[0] == n_global
        ids = np.ascontiguousarray(np.asarray(q_ids, dtype=np.int64))
        assert ids.shape == (n_q,)
        o = np.empty((n_q, D), dtype=np.float64)
        lse = np.empty(n_q, dtype=np.float64)
        if win_off is not None:
            off = np.ascontiguousarray(np.asarray(win_off, dtype=np.int64))
            off_ptr, n_win = off.ctypes.data, off.size - 1
        else:
            off, off_ptr, n_win = None, None, 0
        st = self.lib.atlas_oracle_attention_head_windows(
            n_detail, window_len, off_ptr, n_win, n_global, D, float(scale),
            k_d.ctypes.data, v_d.ctypes.data, kd_lo, kd_lo + k_d.shape[0],
            k_g.ctypes.data, v_g.ctypes.data, n_q, ids.ctypes.data,
            q.ctypes.data, o.ctypes.data, lse.ctypes.data, int(n_threads))
        if st == 1:
            raise ValueError("an allowed detail key lies outside the rows given")
        if st != 0:
            raise MemoryError("oracle allocation failed")
        return o, lse

    def attention_head_aligned(self, grid, cube, global_grid, scale, k_d, v_d, kd_lo: int,
                               k_g, v_g, q_ids, q, n_threads: int = 1):
        """"Aligned proxy tokens only" variant for one head: detail rows in
        cube order of ``grid`` cut into ``cube``; global rows in raster order
        of ``global_grid``. A detail query sees its own cube and the global
        keys whose scaled position lies in that cube; a global query sees
        every global key. Arguments and results as :meth:`attention_head`."""
        f = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float64))
        q = f(q)
        n_q, D = q.shape
        k_d = f(k_d).reshape(-1, D) if k_d is not None else np.zeros((0, D))
        v_d = f(v_d).reshape(-1, D) if v_d is not None else np.zeros((0, D))
        k_g = f(k_g).reshape(-1, D) if k_g is not None else np.zeros((0, D))
        v_g = f(v_g).reshape(-1, D) if v_g is not None else np.zeros((0, D))
        assert k_d.shape == v_d.shape and k_g.shape == v_g.shape
        assert k_g.shape[0] == global_grid[0] * global_grid[1] * global_grid[2]
        ids = np.ascontiguousarray(np.asarray(q_ids, dtype=np.int64))
        assert ids.shape == (n_q,)
        o = np.empty((n_q, D), dtype=np.float64)
        lse = np.empty(n_q, dtype=np.float64)
        st = self.lib.atlas_oracle_attention_head_aligned(
            *grid, *cube, *global_grid, D, float(scale), k_d.ctypes.data, v_d.ctypes.data,
            kd_lo, kd_lo + k_d.shape[0], k_g.ctypes.data, v_g.ctypes.data, n_q,
            ids.ctypes.data, q.ctypes.data, o.ctypes.data, lse.ctypes.data, int(n_threads))
        if st == 1:
            raise ValueError("an allowed detail key lies outside the rows given")
        if st == 3:
            raise RuntimeError("cube positions are not a permutation")
        if st != 0:
            raise MemoryError("oracle allocation failed")
        return o, lse

    def attention_full_aligned(self, q_d, k_d, v_d, grid, cube, q_g, k_g, v_g, global_grid,
                               scale, n_threads: int = 1):
        """All rows, all heads, of the aligned variant. Detail tensors
        [N, heads, D] in cube order, global [G, heads, D] in raster order.
        Returns (o_d, o_g, lse [heads, N+G])."""
        q_d = np.asarray(q_d, dtype=np.float64)
        q_g = np.asarray(q_g, dtype=np.float64)
        N, heads, D = q_d.shape
        G = q_g.shape[0]
        o_d, o_g, lse = np.empty((N, heads, D)), np.empty((G, heads, D)), np.empty((heads, N + G))
        for hh in range(heads):
            q_all = np.concatenate([q_d[:, hh, :], q_g[:, hh, :]], axis=0)
            o, l = self.attention_head_aligned(
                grid, cube, global_grid, scale, np.asarray(k_d)[:, hh, :],
                np.asarray(v_d)[:, hh, :], 0, np.asarray(k_g)[:, hh, :],
                np.asarray(v_g)[:, hh, :], np.arange(N + G, dtype=np.int64), q_all, n_threads)
            o_d[:, hh, :], o_g[:, hh, :], lse[hh] = o[:N], o[N:], l
        return o_d, o_g, lse

    def attention_full(self, q_d, k_d, v_d, window_len, q_g, k_g, v_g,
                       scale, n_threads: int = 1, win_off=None):
        """All rows, all heads. Detail tensors [N, heads, D] in cube order,
        global [G, heads, D]. Returns (o_d, o_g, lse [heads, N+G])."""
        q_d = np.asarray(q_d, dtype=np.float64)
        q_g = np.asarray(q_g, dtype=np.float64)
        N, heads, D = q_d.shape
        G = q_g.shape[0]
        o_d = np.empty((N, heads, D))
        o_g = np.empty((G, heads, D))
        lse = np.empty((heads, N + G))
        for h in range(heads):
            q_all = np.concatenate([q_d[:, h, :], q_g[:, h, :]], axis=0)
            ids = np.arange(N + G, dtype=np.int64)
            o, l = self.attention_head(
                N, window_len, G, scale, np.asarray(k_d)[:, h, :],
                np.asarray(v_d)[:, h, :], 0, np.asarray(k_g)[:, h, :],
                np.asarray(v_g)[:, h, :], ids, q_all, n_threads, win_off)
            o_d[:, h, :] = o[:N]
            o_g[:, h, :] = o[N:]
            lse[h] = l
        return o_d, o_g, lse

    # -- backward -------------------------------------------------------
    def _bwd(self, call, q_d, k_d, v_d, q_g, k_g, v_g, do_d, do_g):
        """Stack detail and global rows per head, run ``call`` (the C
        backward of one head) and split the gradients again."""
        a = [np.asarray(t, dtype=np.float64) for t in (q_d, k_d, v_d, do_d)]
        g = [np.asarray(t, dtype=np.float64) for t in (q_g, k_g, v_g, do_g)]
        N, heads, D = a[0].shape
        G = g[0].shape[0]
        out = [np.empty((N, heads, D)) for _ in range(3)] + [np.empty((G, heads, D))
                                                            for _ in range(3)]
        for hh in range(heads):
            q, k, v, do = (np.ascontiguousarray(np.concatenate([x[:, hh], y[:, hh]]))
                           for x, y in zip(a, g))
            dq, dk, dv = (np.empty((N + G, D)) for _ in range(3))
            st = call(D, q.ctypes.data, k.ctypes.data, v.ctypes.data, do.ctypes.data,
                      dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
            if st != 0:
                raise RuntimeError(f"oracle backward failed ({st})")
            for idx, x in enumerate((dq, dk, dv)):
                out[idx][:, hh] = x[:N]
                out[3 + idx][:, hh] = x[N:]
        return tuple(out)

    def attention_bwd_full(self, q_d, k_d, v_d, window_len, q_g, k_g, v_g, do_d, do_g, scale,
                           n_threads: int = 1, win_off=None):
        """Gradients (dq_d, dk_d, dv_d, dq_g, dk_g, dv_g) of the attention
        output contracted with (do_d, do_g); shapes as attention_full."""
        N = np.asarray(q_d).shape[0]
        G = np.asarray(q_g).shape[0]
        if win_off is not None:
            off = np.ascontiguousarray(np.asarray(win_off, dtype=np.int64))
            off_ptr, n_win = off.ctypes.data, off.size - 1
        else:
            off, off_ptr, n_win = None, None, 0
        f = lambda D, *p: self.lib.atlas_oracle_attention_bwd_head_windows(
            N, window_len, off_ptr, n_win, G, D, float(scale), *p, int(n_threads))
        return self._bwd(f, q_d, k_d, v_d, q_g, k_g, v_g, do_d, do_g)

    def attention_bwd_sampled(self, q, k, v, do, n_detail, window_len, scale, q_rows, k_rows,
                              n_threads: int = 1, win_off=None):
        """One head, all N+G rows given ([N+G, D] each, detail rows first):
        dq for the query rows ``q_rows`` and (dk, dv) for the key rows
        ``k_rows``; returns (dq [len(q_rows), D], dk, dv [len(k_rows), D])."""
        f = lambda a: np.ascontiguousarray(np.asarray(a, dtype=np.float64))
        q, k, v, do = f(q), f(k), f(v), f(do)
        R, D = q.shape
        qs = np.ascontiguousarray(np.asarray(q_rows, dtype=np.int64))
        ks = np.ascontiguousarray(np.asarray(k_rows, dtype=np.int64))
        dq = np.empty((qs.size, D))
        dk = np.empty((ks.size, D))
        dv = np.empty((ks.size, D))
        if win_off is not None:
            off = np.ascontiguousarray(np.asarray(win_off, dtype=np.int64))
            off_ptr, n_win = off.ctypes.data, off.size - 1
        else:
            off, off_ptr, n_win = None, None, 0
        st = self.lib.atlas_oracle_attention_bwd_head_sampled(
            n_detail, window_len, off_ptr, n_win, R - n_detail, D, float(scale), q.ctypes.data,
            k.ctypes.data, v.ctypes.data, do.ctypes.data, qs.size, qs.ctypes.data, ks.size,
            ks.ctypes.data, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, int(n_threads))
        if st != 0:
            raise RuntimeError(f"oracle backward failed ({st})")
        return dq, dk, dv

    def attention_bwd_full_aligned(self, q_d, k_d, v_d, grid, cube, q_g, k_g, v_g, global_grid,
                                   do_d, do_g, scale, n_threads: int = 1):
        """Gradients of the aligned variant (layout as attention_full_aligned)."""
        f = lambda D, *p: self.lib.atlas_oracle_attention_bwd_head_aligned(
            *grid, *cube, *global_grid, D, float(scale), *p, int(n_threads))
        return self._bwd(f, q_d, k_d, v_d, q_g, k_g, v_g, do_d, do_g)

    # -- projections around the path (QKV in, output out) ------------------
    def qkv_proj_reorder(self, x, w, grid, cube, heads, head_dim, theta=10000.0, split=None,
                         scales=None):
        """[Q | K | V] = x w^T (x: [rows, C] raster order, w: [3*heads*head_dim, C]),
        Q and K rotated by 3D RoPE at their raster positions when ``split``
        is given, all three reordered to cube order. fp64; returns (q, k, v),
        each [rows, heads, head_dim]. ``rows`` may hold several problems of
        ``grid`` stacked."""
        x = np.asarray(x, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64)
        y = x @ w.T                              # library matmul, fp64
        n = grid[0] * grid[1] * grid[2]
        hd = heads * head_dim
        out = []
        for i in range(3):
            t = y[:, i * hd:(i + 1) * hd].reshape(-1, heads, head_dim)
            parts = []
            for b in range(t.shape[0] // n):
                tb = np.ascontiguousarray(t[b * n:(b + 1) * n])
                if i < 2 and split is not None:
                    tb = self.rope3d_grid(tb, grid, theta, split, scales)
                parts.append(self.cube_reorder(tb, grid, cube))
            out.append(np.concatenate(parts) if parts else t.copy())
        return tuple(out)

    def out_proj_unorder(self, o, w, grid, cube):
        """y = unorder(o) w^T (o: [rows, heads*head_dim] in cube order, w:
        [C_out, heads*head_dim]); fp64, [rows, C_out] in raster order."""
        o = np.asarray(o, dtype=np.float64)
        w = np.asarray(w, dtype=np.float64)
        n = grid[0] * grid[1] * grid[2]
        raster = np.concatenate([self.cube_unorder(np.ascontiguousarray(o[b * n:(b + 1) * n]),
                                                   grid, cube)
                                 for b in range(o.shape[0] // n)])
        return raster @ w.T

    def max_threads(self) -> int:
        return int(self.lib.atlas_oracle_max_threads())
