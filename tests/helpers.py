"""Shared test utilities: the GPU path driven through the C-ABI binding, and
comparison rules against the fp64 oracle.

Tolerances (floating point):
  * RoPE: each output within 1 ulp of the I/O type of the fp64 value, plus
    2^-20 * max(|x0|, |x1|) of its input pair (fp64-built cos/sin tables
    rounded to fp32, fp32 rotation, one rounding to the I/O type).
  * Attention: max-abs error <= 2e-2 and mean-abs error <= 2e-3 against the
    fp64 oracle (bf16 I/O), LSE abs error <= 5e-3; fp32 I/O uses 1e-4 /
    1e-5 / 1e-4 (exact fp32 products, expf).
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from video_dit_windowed_b200 import atlas

ATTN_TOL = {"bf16": dict(max_abs=2e-2, mean_abs=2e-3, lse=5e-3),
            "fp32": dict(max_abs=1e-4, mean_abs=1e-5, lse=1e-4)}

_ORC = None


def orc():
    global _ORC
    if _ORC is None:
        _ORC = oracle.Oracle()
    return _ORC


def n_threads():
    return max(1, os.cpu_count() or 1)


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a (possibly device, bf16/fp32) tensor."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def aligned_positions(grid, cube, gg):
    """pos[g] = place of global raster token g in the aligned order, from the
    reading of position alignment: global index x of an axis of e tokens sits
    at detail position x*E/e, in detail cube floor(x*E/(c*e)); tokens are
    listed cube by cube (raster order of the cube grid), raster order inside."""
    nh = -(-grid[1] // cube[1])
    nw = -(-grid[2] // cube[2])
    keys = []
    for g in range(gg[0] * gg[1] * gg[2]):
        x = (g // (gg[1] * gg[2]), (g // gg[2]) % gg[1], g % gg[2])
        b = [x[a] * grid[a] // (cube[a] * gg[a]) for a in range(3)]
        keys.append(((b[0] * nh + b[1]) * nw + b[2], g))
    order = [g for _, g in sorted(keys)]
    pos = np.empty(len(order), dtype=np.int64)
    pos[np.array(order, dtype=np.int64)] = np.arange(len(order))
    return pos


def ulp(v: np.ndarray, dtype: str) -> np.ndarray:
    _, e = np.frexp(np.abs(v))
    bits = 8 if dtype == "bf16" else 24
    u = np.ldexp(1.0, e - bits)
    tiny = 2.0 ** (-133 if dtype == "bf16" else -149)
    return np.where(np.abs(v) < 2.0 ** -126, tiny, u)


def assert_rope_close(got: np.ndarray, exact: np.ndarray, x_in: np.ndarray, dtype: str):
    """``got``/``exact``/``x_in``: [..., head_dim] with interleaved pairs."""
    pair_mag = np.maximum(np.abs(x_in[..., 0::2]), np.abs(x_in[..., 1::2]))
    slack = np.repeat(pair_mag, 2, axis=-1) * 2.0 ** -20
    bound = ulp(exact, dtype) + slack
    err = np.abs(got - exact)
    bad = err > bound
    assert not bad.any(), (
        f"{int(bad.sum())} RoPE outputs out of bound; worst err {err.max():.3e}")


def assert_attn_close(o_gpu: np.ndarray, o_ref: np.ndarray, dtype: str, what: str = ""):
    tol = ATTN_TOL[dtype]
    err = np.abs(o_gpu - o_ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= tol["max_abs"], f"{what} max-abs {mx:.3e} > {tol['max_abs']}"
    assert mean <= tol["mean_abs"], f"{what} mean-abs {mean:.3e} > {tol['mean_abs']}"
    return mx, mean


def assert_lse_close(l_gpu: np.ndarray, l_ref: np.ndarray, dtype: str, what: str = ""):
    err = float(np.abs(l_gpu - l_ref).max())
    assert err <= ATTN_TOL[dtype]["lse"], f"{what} LSE err {err:.3e}"
    return err


def check_no_device_error():
    code = atlas.last_device_error()
    assert code == 0, f"device error word 0x{code:x}"


def attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g, with_lse=True):
    """Run the C-ABI attention on device tensors; returns (o_d, o_g, lse)."""
    dev = (q_d if q_d.shape[0] else q_g).device
    o_d = torch.empty_like(q_d)
    o_g = torch.empty_like(q_g)
    heads = (q_d if q_d.shape[0] else q_g).shape[1]
    lse = (torch.empty(heads, q_d.shape[0] + q_g.shape[0], dtype=torch.float32, device=dev)
           if with_lse else None)
    atlas.local_global_attn(q_d, k_d, v_d, L, q_g, k_g, v_g, o_d, o_g, lse)
    return o_d, o_g, lse


def oracle_attention_rows(q_d, k_d, v_d, L, q_g, k_g, v_g, head, det_rows, glob_rows,
                          scale):
    """fp64 oracle for selected rows of one head. Detail rows must come from
    whole windows listed in ``det_rows`` (cube order); ``glob_rows`` index the
    global rows. Inputs are device or host tensors [rows, heads, D]."""
    N = q_d.shape[0]
    G = q_g.shape[0]
    outs, lses = [], []
    kg = f64(k_g[:, head]) if G else None
    vg = f64(v_g[:, head]) if G else None
    det_rows = np.asarray(det_rows, dtype=np.int64)
    if det_rows.size:
        # windows touched, processed one at a time (only their rows are copied)
        wins = np.unique(det_rows // L)
        o_all = np.empty((det_rows.size, q_d.shape[2]))
        l_all = np.empty(det_rows.size)
        for w in wins:
            sel = np.nonzero(det_rows // L == w)[0]
            rows = det_rows[sel]
            lo = int(w) * L
            kd = f64(k_d[lo:lo + L, head])
            vd = f64(v_d[lo:lo + L, head])
            q = f64(q_d[torch.as_tensor(rows, device=q_d.device), head])
            o, l = orc().attention_head(N, L, G, scale, kd, vd, lo, kg, vg, rows, q,
                                        n_threads())
            o_all[sel] = o
            l_all[sel] = l
        outs.append(o_all)
        lses.append(l_all)
    glob_rows = np.asarray(glob_rows, dtype=np.int64)
    if glob_rows.size:
        q = f64(q_g[torch.as_tensor(glob_rows, device=q_g.device), head])
        o, l = orc().attention_head(N, max(L, 1), G, scale, None, None, 0, kg, vg,
                                    glob_rows + N, q, n_threads())
        outs.append(o)
        lses.append(l)
    return outs, lses
