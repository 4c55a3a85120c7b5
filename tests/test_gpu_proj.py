"""GPU parity of the projections with the path's permutation in the GEMM
epilogue (QKV projection + RoPE + reorder; output projection + unorder)
against the fp64 oracle (numpy matmul composed with the pinned reorder and
RoPE), through the C-ABI.

Bound per output element (derived from the arithmetic): one bf16 ulp of the
exact value (the epilogue rounds once, to nearest) plus the fp32
accumulation's worst case K * 2^-24 * sum_c |x_c w_c| (for a rotated pair,
the sum of its two columns' sums, plus 2^-22 of the pair's magnitude for the
fp32 cos/sin table).
"""
import numpy as np
import pytest
import torch

from helpers import check_no_device_error, f64, orc, ulp
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def weights(n_out, c_in, stream, seed=0):
    w = normal((n_out, c_in), stream, torch.float32, seed=seed, device=DEV) / c_in ** 0.5
    return w.to(torch.bfloat16)


def qkv_bound(x, w, ref, heads, hd, rotated):
    """Per-element bound of the QKV outputs (see the module docstring),
    shaped like ref [3][rows, heads, hd] in the oracle's (cube) order."""
    K = x.shape[1]
    s = np.abs(x) @ np.abs(w).T                      # sum_c |x_c w_c|, [rows, 3*heads*hd]
    out = []
    for i in range(3):
        si = s[:, i * heads * hd:(i + 1) * heads * hd].reshape(-1, heads, hd)
        if rotated and i < 2:
            pair = si[..., 0::2] + si[..., 1::2]
            si = np.repeat(pair, 2, axis=-1)
        out.append(si * K * 2.0 ** -24)
    return out


CASES = [
    # grid, cube, batch, c_in, heads, hd, rope scales (None: no rotation)
    ((4, 8, 8), (2, 4, 4), 2, 256, 2, 128, (1.0, 1.0, 1.0)),
    ((5, 7, 9), (2, 3, 4), 1, 128, 4, 64, (2.0, 1.0, 1.0)),
    ((3, 5, 7), (3, 5, 7), 1, 192, 2, 128, None),
    ((2, 12, 20), (1, 1, 1), 1, 320, 2, 128, (4.0, 4.0, 4.0)),    # global proxy: no permutation
]


@pytest.mark.parametrize("grid,cube,batch,c_in,heads,hd,scales", CASES)
def test_qkv_proj_reorder(grid, cube, batch, c_in, heads, hd, scales):
    n = grid[0] * grid[1] * grid[2]
    split = (16, 24, 24) if hd == 64 else (44, 42, 42)
    x = normal((batch * n, c_in), "q_d", torch.bfloat16, seed=31, device=DEV)
    w = weights(3 * heads * hd, c_in, "k_d", seed=31)
    q, k, v = (torch.empty(batch * n, heads, hd, dtype=torch.bfloat16, device=DEV)
               for _ in range(3))
    rope = atlas.make_rope(10000.0, split, scales) if scales else None
    atlas.qkv_proj_reorder(x, w, grid, cube, q, k, v, rope, batch=batch)
    torch.cuda.synchronize()
    check_no_device_error()
    xd, wd = f64(x), f64(w)
    ref = orc().qkv_proj_reorder(xd, wd, grid, cube, heads, hd, 10000.0,
                                 split if scales else None, scales)
    # the bound's accumulation term, permuted like the outputs
    bnd = qkv_bound(xd, wd, ref, heads, hd, scales is not None)
    for i, (got, r) in enumerate(zip((q, k, v), ref)):
        b = np.concatenate([orc().cube_reorder(bnd[i][p * n:(p + 1) * n], grid, cube)
                            for p in range(batch)])
        extra = (2.0 ** -22) * np.abs(r) if (scales and i < 2) else 0.0
        err = np.abs(f64(got) - r)
        limit = ulp(r, "bf16") + b + extra
        assert np.all(err <= limit), f"{'qkv'[i]}: worst err/limit {np.max(err / limit):.2f}"


@pytest.mark.parametrize("grid,cube,batch,c_in,c_out", [
    ((4, 8, 8), (2, 4, 4), 2, 256, 512),
    ((5, 7, 9), (2, 3, 4), 1, 128, 256),
    ((3, 5, 7), (1, 5, 7), 1, 320, 256),
])
def test_out_proj_unorder(grid, cube, batch, c_in, c_out):
    n = grid[0] * grid[1] * grid[2]
    o = normal((batch * n, c_in), "v_d", torch.bfloat16, seed=32, device=DEV)
    w = weights(c_out, c_in, "v_g", seed=32)
    y = torch.empty(batch * n, c_out, dtype=torch.bfloat16, device=DEV)
    atlas.out_proj_unorder(o, w, grid, cube, y, batch=batch)
    torch.cuda.synchronize()
    check_no_device_error()
    od, wd = f64(o), f64(w)
    ref = orc().out_proj_unorder(od, wd, grid, cube)
    s = np.concatenate([orc().cube_unorder(np.abs(od[p * n:(p + 1) * n]), grid, cube)
                        for p in range(batch)]) @ np.abs(wd).T
    limit = ulp(ref, "bf16") + c_in * 2.0 ** -24 * s
    err = np.abs(f64(y) - ref)
    assert np.all(err <= limit), f"worst err/limit {np.max(err / limit):.2f}"


def test_qkv_proj_wide_sampled():
    """Model width 5120, 40 heads (the 720p workload's projection), a
    768-token grid: every output row of a sample of columns against the
    oracle."""
    grid, cube, heads, hd, c_in = (3, 16, 16), (3, 16, 16), 40, 128, 5120
    n = 768
    x = normal((n, c_in), "q_d", torch.bfloat16, seed=33, device=DEV)
    w = weights(3 * heads * hd, c_in, "k_d", seed=33)
    q, k, v = (torch.empty(n, heads, hd, dtype=torch.bfloat16, device=DEV) for _ in range(3))
    rope = atlas.make_rope(10000.0, (44, 42, 42), (1.0, 1.0, 1.0))
    atlas.qkv_proj_reorder(x, w, grid, cube, q, k, v, rope)
    torch.cuda.synchronize()
    check_no_device_error()
    cols = [0, 1, 7, 39]                     # heads checked in q, k and v
    xd = f64(x)
    for i, got in enumerate((q, k, v)):
        wsel = np.concatenate([f64(w[i * heads * hd + h * hd:i * heads * hd + (h + 1) * hd])
                               for h in cols])
        ref = orc().qkv_proj_reorder(xd, np.concatenate([wsel] * 3), grid, cube, len(cols), hd,
                                     10000.0, (44, 42, 42), (1.0, 1.0, 1.0))[i]
        s = np.abs(xd) @ np.abs(wsel).T
        s = orc().cube_reorder(s.reshape(n, len(cols), hd), grid, cube)
        if i < 2:
            s = np.repeat(s[..., 0::2] + s[..., 1::2], 2, axis=-1)
        limit = ulp(ref, "bf16") + c_in * 2.0 ** -24 * s + (2.0 ** -22 * np.abs(ref) if i < 2 else 0)
        err = np.abs(f64(got[:, cols]) - ref)
        assert np.all(err <= limit), f"{'qkv'[i]}: worst err/limit {np.max(err / limit):.2f}"
