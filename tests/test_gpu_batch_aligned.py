"""GPU parity, through the C-ABI, for two generalisations of the path:

* batch > 1: problems of one shape stacked along the rows; every problem is
  permuted, rotated and attended on its own (a query sees only keys of its
  own problem);
* the "aligned proxy tokens only" variant ("Technische Samenvatting:
  AtlasVid", Methodologie 2: a detail query sees the aligned global tokens;
  position alignment scales global coordinates by the resolution ratios).
  Reading: global token (tg, hg, wg) sits at (tg*T/t, hg*H/h, wg*W/w) of the
  detail grid and is aligned with the cube holding that point. The GPU path
  lists the global tokens in the aligned order (cube by cube of the detail
  grid) and passes per-window global offsets; with integer ratios dividing
  the cube that order is the global grid's own cube order.

The oracle takes the global tokens in raster order and decides alignment
from coordinates; the GPU results are mapped back to raster order.
"""
import numpy as np
import pytest
import torch

from helpers import (aligned_positions, assert_attn_close, assert_rope_close,
                     check_no_device_error, f64, n_threads, orc)
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import normal

pytestmark = pytest.mark.gpu
DEV = "cuda"
LSE_TOL = {"bf16": 5e-3, "fp32": 1e-4}


def tdt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def split_for(hd):
    return (16, 24, 24) if hd == 64 else (44, 42, 42)


def mk(rows, heads, hd, stream, dtype, seed=0):
    return normal((rows, heads, hd), stream, tdt(dtype), seed=seed, device=DEV)


# ---------------------------------------------------------------------------
# Batched permutations
# ---------------------------------------------------------------------------

PERM_CASES = [
    ((4, 8, 8), (2, 4, 4), 3, 2, 64, "bf16"),
    ((5, 7, 9), (2, 3, 4), 2, 3, 128, "fp32"),
    ((3, 17, 23), (3, 16, 16), 3, 2, 128, "bf16"),
]


@pytest.mark.parametrize("grid,cube,B,heads,hd,dtype", PERM_CASES)
def test_batched_permutations_match_per_problem(grid, cube, B, heads, hd, dtype):
    n = grid[0] * grid[1] * grid[2]
    x = mk(B * n, heads, hd, "q_d", dtype, seed=5)
    rope = atlas.make_rope(10000.0, split_for(hd), (2.0, 1.0, 1.0))
    y, z, yr, xr = (torch.empty_like(x) for _ in range(4))
    atlas.cube_reorder_batched(x, y, B, grid, cube)
    atlas.cube_unorder_batched(y, z, B, grid, cube)
    atlas.cube_reorder_batched(x, yr, B, grid, cube, rope)
    atlas.rope3d_batched(x, xr, B, grid, rope)
    torch.cuda.synchronize()
    check_no_device_error()
    assert torch.equal(z.view(torch.uint8), x.view(torch.uint8))
    for b in range(B):
        rows = slice(b * n, (b + 1) * n)
        xb = x[rows].contiguous()
        ref_y, ref_yr, ref_xr = (torch.empty_like(xb) for _ in range(3))
        atlas.cube_reorder(xb, ref_y, grid, cube)
        atlas.cube_reorder(xb, ref_yr, grid, cube, rope)
        atlas.rope3d(xb, ref_xr, grid, rope)
        torch.cuda.synchronize()
        assert torch.equal(y[rows].view(torch.uint8), ref_y.view(torch.uint8))
        assert torch.equal(yr[rows].view(torch.uint8), ref_yr.view(torch.uint8))
        assert torch.equal(xr[rows].view(torch.uint8), ref_xr.view(torch.uint8))
        raw = xb.cpu().view(torch.uint8).numpy().reshape(n, -1)
        assert y[rows].cpu().view(torch.uint8).numpy().reshape(n, -1).tobytes() == \
            orc().cube_reorder(raw, grid, cube).tobytes()
        xd = f64(xb)
        exact = orc().cube_reorder(orc().rope3d_grid(xd, grid, 10000.0, split_for(hd),
                                                     (2.0, 1.0, 1.0)), grid, cube)
        assert_rope_close(f64(yr[rows]), exact, orc().cube_reorder(xd, grid, cube), dtype)


# ---------------------------------------------------------------------------
# Batched attention
# ---------------------------------------------------------------------------

# grid, cube, G, B, heads, hd, dtype, variable windows
BATCH_CASES = [
    ((4, 8, 8), (2, 4, 4), 37, 3, 2, 64, "bf16", False),
    ((4, 8, 8), (2, 4, 4), 37, 3, 2, 64, "fp32", False),
    ((5, 7, 9), (2, 3, 4), 29, 2, 2, 128, "bf16", True),
    ((5, 7, 9), (2, 3, 4), 29, 2, 2, 128, "fp32", True),
    ((6, 16, 16), (3, 8, 8), 300, 2, 3, 128, "bf16", False),
    ((0, 0, 0), (1, 1, 1), 300, 3, 2, 128, "bf16", False),
]


@pytest.mark.parametrize("grid,cube,G,B,heads,hd,dtype,varlen", BATCH_CASES)
def test_batched_attention(grid, cube, G, B, heads, hd, dtype, varlen):
    N = grid[0] * grid[1] * grid[2]
    L = cube[0] * cube[1] * cube[2]
    t = {s: mk(B * (N if s.endswith("_d") else G), heads, hd, s, dtype, seed=7)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    o_d, o_g = torch.empty_like(t["q_d"]), torch.empty_like(t["q_g"])
    lse = torch.empty(B, heads, N + G, dtype=torch.float32, device=DEV)
    off = atlas.cube_window_offsets(grid, cube) if varlen and N else None
    kw = dict(window_offsets=off.to(DEV)) if off is not None else dict(window_len=L if N else 0)
    atlas.local_global_attn_ex(t["q_d"], t["k_d"], t["v_d"], t["q_g"], t["k_g"], t["v_g"], o_d,
                               o_g, lse, batch=B, **kw)
    torch.cuda.synchronize()
    check_no_device_error()
    win = off.numpy().astype(np.int64) if off is not None else None
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        # the same problem through the unbatched entry: identical bits
        pb = {s: t[s][sd if s.endswith("_d") else sg].contiguous() for s in t}
        a_d, a_g = torch.empty_like(pb["q_d"]), torch.empty_like(pb["q_g"])
        a_l = torch.empty(heads, N + G, dtype=torch.float32, device=DEV)
        if off is not None:
            atlas.local_global_attn_windows(pb["q_d"], pb["k_d"], pb["v_d"], off.to(DEV),
                                            pb["q_g"], pb["k_g"], pb["v_g"], a_d, a_g, a_l)
        else:
            atlas.local_global_attn(pb["q_d"], pb["k_d"], pb["v_d"], L if N else 1, pb["q_g"],
                                    pb["k_g"], pb["v_g"], a_d, a_g, a_l)
        torch.cuda.synchronize()
        assert torch.equal(o_d[sd], a_d) and torch.equal(o_g[sg], a_g)
        assert torch.equal(lse[b], a_l)
        # and the oracle
        ref_d, ref_g, ref_l = orc().attention_full(
            f64(pb["q_d"]), f64(pb["k_d"]), f64(pb["v_d"]), L if N else 1, f64(pb["q_g"]),
            f64(pb["k_g"]), f64(pb["v_g"]), hd ** -0.5, n_threads(), win_off=win)
        got = np.concatenate([f64(o_d[sd]), f64(o_g[sg])])
        assert_attn_close(got, np.concatenate([ref_d, ref_g]), dtype, f"problem {b}")
        assert np.max(np.abs(f64(lse[b]) - ref_l)) <= LSE_TOL[dtype]


# ---------------------------------------------------------------------------
# "Aligned proxy tokens only"
# ---------------------------------------------------------------------------

# detail grid, cube, global grid, batch, heads, hd, dtype
ALIGNED_CASES = [
    ((6, 16, 16), (3, 8, 8), (6, 4, 4), 1, 2, 128, "bf16"),
    ((5, 12, 20), (2, 8, 8), (5, 3, 5), 1, 2, 64, "bf16"),
    ((5, 12, 20), (2, 8, 8), (5, 3, 5), 1, 2, 64, "fp32"),
    ((4, 8, 8), (2, 4, 4), (2, 4, 4), 2, 2, 128, "bf16"),
    ((4, 8, 8), (2, 4, 4), (2, 4, 4), 2, 2, 64, "fp32"),
]


def aligned_chain(x, grid, cube, gg, B, hd, detail_scales, global_scales):
    """Raster inputs -> reorder (+RoPE) of detail and global tokens -> aligned
    attention -> unorder. Returns raster (o_d, o_g) and lse [B, heads, N+G]
    with each problem's global columns in global cube order."""
    gcube = atlas.aligned_global_cube(grid, cube, gg)
    rd = atlas.make_rope(10000.0, split_for(hd), detail_scales)
    rg = atlas.make_rope(10000.0, split_for(hd), global_scales)
    y = {s: torch.empty_like(x[s]) for s in x}
    for s in ("q_d", "k_d"):
        atlas.cube_reorder_batched(x[s], y[s], B, grid, cube, rd)
    atlas.cube_reorder_batched(x["v_d"], y["v_d"], B, grid, cube)
    for s in ("q_g", "k_g"):
        atlas.cube_reorder_batched(x[s], y[s], B, gg, gcube, rg)
    atlas.cube_reorder_batched(x["v_g"], y["v_g"], B, gg, gcube)
    win = atlas.cube_window_offsets(grid, cube).to(DEV)
    gwin = atlas.cube_window_offsets(gg, gcube).to(DEV)
    assert win.numel() == gwin.numel()
    N, G = grid[0] * grid[1] * grid[2], gg[0] * gg[1] * gg[2]
    heads = x["q_d"].shape[1]
    o_d, o_g = torch.empty_like(y["q_d"]), torch.empty_like(y["q_g"])
    lse = torch.empty(B, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(y["q_d"], y["k_d"], y["v_d"], y["q_g"], y["k_g"], y["v_g"], o_d,
                               o_g, lse, batch=B, window_offsets=win,
                               global_window_offsets=gwin)
    r_d, r_g = torch.empty_like(o_d), torch.empty_like(o_g)
    atlas.cube_unorder_batched(o_d, r_d, B, grid, cube)
    atlas.cube_unorder_batched(o_g, r_g, B, gg, gcube)
    torch.cuda.synchronize()
    check_no_device_error()
    return r_d, r_g, lse, gcube


@pytest.mark.parametrize("grid,cube,gg,B,heads,hd,dtype", ALIGNED_CASES)
def test_aligned_chain(grid, cube, gg, B, heads, hd, dtype):
    N, G = grid[0] * grid[1] * grid[2], gg[0] * gg[1] * gg[2]
    ratios = tuple(float(a // b) for a, b in zip(grid, gg))
    x = {s: mk(B * (N if s.endswith("_d") else G), heads, hd, s, dtype, seed=11)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    r_d, r_g, lse, gcube = aligned_chain(x, grid, cube, gg, B, hd, (1.0, 1.0, 1.0), ratios)
    o = orc()
    gpos = o.cube_positions(gg, gcube)
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        rot = lambda s, g, sc: o.rope3d_grid(f64(x[s][sd if s.endswith("_d") else sg]), g,
                                             10000.0, split_for(hd), sc)
        qd = o.cube_reorder(rot("q_d", grid, (1, 1, 1)), grid, cube)
        kd = o.cube_reorder(rot("k_d", grid, (1, 1, 1)), grid, cube)
        vd = o.cube_reorder(f64(x["v_d"][sd]), grid, cube)
        ref_d, ref_g, ref_l = o.attention_full_aligned(
            qd, kd, vd, grid, cube, rot("q_g", gg, ratios), rot("k_g", gg, ratios),
            f64(x["v_g"][sg]), gg, hd ** -0.5, n_threads())
        got = np.concatenate([f64(r_d[sd]), f64(r_g[sg])])
        ref = np.concatenate([o.cube_unorder(ref_d, grid, cube), ref_g])
        assert_attn_close(got, ref, dtype, f"{grid} {gg} problem {b}")
        l_gpu = f64(lse[b])
        # detail columns in cube order on both sides; global columns of the
        # GPU in global cube order, of the oracle in raster order
        l_gpu_g = l_gpu[:, N + gpos]
        assert np.max(np.abs(l_gpu[:, :N] - ref_l[:, :N])) <= LSE_TOL[dtype]
        assert np.max(np.abs(l_gpu_g - ref_l[:, N:])) <= LSE_TOL[dtype]


def test_aligned_differs_from_all_globals():
    """The variant is a different mask: with global values far from the
    detail ones, the detail outputs move when every global key is allowed."""
    grid, cube, gg, hd = (4, 8, 8), (2, 4, 4), (2, 4, 4), 64
    N, G = 256, 32
    x = {s: mk(N if s.endswith("_d") else G, 1, hd, s, "bf16", seed=12)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    gcube = atlas.aligned_global_cube(grid, cube, gg)
    y = {s: torch.empty_like(x[s]) for s in x}
    for s in ("q_d", "k_d", "v_d"):
        atlas.cube_reorder(x[s], y[s], grid, cube)
    for s in ("q_g", "k_g", "v_g"):
        atlas.cube_reorder(x[s], y[s], gg, gcube)
    y["v_g"] += 4.0
    gwin = atlas.cube_window_offsets(gg, gcube).to(DEV)
    a_d, a_g = torch.empty_like(y["q_d"]), torch.empty_like(y["q_g"])
    b_d, b_g = torch.empty_like(y["q_d"]), torch.empty_like(y["q_g"])
    atlas.local_global_attn_ex(y["q_d"], y["k_d"], y["v_d"], y["q_g"], y["k_g"], y["v_g"], a_d,
                               a_g, window_len=32, global_window_offsets=gwin)
    atlas.local_global_attn_ex(y["q_d"], y["k_d"], y["v_d"], y["q_g"], y["k_g"], y["v_g"], b_d,
                               b_g, window_len=32)
    torch.cuda.synchronize()
    assert torch.equal(a_g, b_g)                       # global rows: same keys
    assert (a_d.float() - b_d.float()).abs().mean() > 0.3


def test_aligned_720p_sampled():
    """720p geometry (detail 21x48x80, cubes 3x16x16, global 21x12x20, 8
    heads): 48 aligned global keys per window. Sampled windows and global
    rows on the first and last head against the oracle."""
    grid, cube, gg, heads, hd = (21, 48, 80), (3, 16, 16), (21, 12, 20), 8, 128
    N, G, L = 80640, 5040, 768
    gcube = atlas.aligned_global_cube(grid, cube, gg)
    assert gcube == (3, 4, 4)
    q_d, k_d, v_d = (mk(N, heads, hd, s, "bf16", seed=13) for s in ("q_d", "k_d", "v_d"))
    xg = {s: mk(G, heads, hd, s, "bf16", seed=13) for s in ("q_g", "k_g", "v_g")}
    yg = {s: torch.empty_like(xg[s]) for s in xg}
    for s in xg:
        atlas.cube_reorder(xg[s], yg[s], gg, gcube)
    gwin = atlas.cube_window_offsets(gg, gcube).to(DEV)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(yg["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(q_d, k_d, v_d, yg["q_g"], yg["k_g"], yg["v_g"], o_d, o_g, lse,
                               window_len=L, global_window_offsets=gwin)
    torch.cuda.synchronize()
    check_no_device_error()
    gpos = orc().cube_positions(gg, gcube)
    for head in (0, heads - 1):
        kg, vg = f64(xg["k_g"][:, head]), f64(xg["v_g"][:, head])
        for w in (0, 57, N // L - 1):
            lo = w * L
            rows = np.arange(lo, lo + L)
            ref, ref_l = orc().attention_head_aligned(
                grid, cube, gg, hd ** -0.5, f64(k_d[lo:lo + L, head]), f64(v_d[lo:lo + L, head]),
                lo, kg, vg, rows, f64(q_d[lo:lo + L, head]), n_threads())
            assert_attn_close(f64(o_d[lo:lo + L, head]), ref, "bf16", f"window {w} head {head}")
            assert np.max(np.abs(f64(lse[0, head, lo:lo + L]) - ref_l)) <= LSE_TOL["bf16"]
        g_rows = np.array([0, 1, 777, G - 1])
        ref, _ = orc().attention_head_aligned(
            grid, cube, gg, hd ** -0.5, None, None, 0, kg, vg, N + g_rows,
            f64(xg["q_g"][torch.as_tensor(g_rows, device=DEV), head]), n_threads())
        got = f64(o_g[torch.as_tensor(gpos[g_rows], device=DEV), head])
        assert_attn_close(got, ref, "bf16", f"global rows head {head}")


# ---------------------------------------------------------------------------
# The aligned order: any grid ratios
# ---------------------------------------------------------------------------

def general_aligned_chain(x, grid, cube, gg, B, hd, global_scales):
    """Raster inputs -> detail cube reorder (+RoPE) and global aligned-order
    reorder (+RoPE at global raster coordinates) -> attention with per-window
    global ranges -> back to raster order."""
    rd = atlas.make_rope(10000.0, split_for(hd), (1.0, 1.0, 1.0))
    rg = atlas.make_rope(10000.0, split_for(hd), global_scales)
    y = {s: torch.empty_like(x[s]) for s in x}
    for s in ("q_d", "k_d", "v_d"):
        atlas.cube_reorder_batched(x[s], y[s], B, grid, cube, rd if s != "v_d" else None)
    for s in ("q_g", "k_g", "v_g"):
        atlas.aligned_global_reorder(x[s], y[s], grid, cube, gg, rg if s != "v_g" else None,
                                     batch=B)
    win = atlas.cube_window_offsets(grid, cube).to(DEV)
    gwin = atlas.aligned_global_offsets(grid, cube, gg).to(DEV)
    assert win.numel() == gwin.numel()
    N, G = grid[0] * grid[1] * grid[2], gg[0] * gg[1] * gg[2]
    heads = x["q_d"].shape[1]
    o_d, o_g = torch.empty_like(y["q_d"]), torch.empty_like(y["q_g"])
    lse = torch.empty(B, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(y["q_d"], y["k_d"], y["v_d"], y["q_g"], y["k_g"], y["v_g"], o_d,
                               o_g, lse, batch=B, window_offsets=win,
                               global_window_offsets=gwin)
    r_d, r_g = torch.empty_like(o_d), torch.empty_like(o_g)
    atlas.cube_unorder_batched(o_d, r_d, B, grid, cube)
    atlas.aligned_global_unorder(o_g, r_g, grid, cube, gg, batch=B)
    torch.cuda.synchronize()
    check_no_device_error()
    return r_d, r_g, lse, y


# detail grid, cube, global grid, batch, heads, hd, dtype. Ratios that are
# not integers, ratios below one, windows with no aligned global token
# (5/2 tokens per global step in t with cubes of 2: cube 2 of t gets none).
GENERAL_CASES = [
    ((5, 7, 9), (2, 3, 4), (2, 3, 4), 1, 2, 128, "bf16"),
    ((5, 7, 9), (2, 3, 4), (2, 3, 4), 2, 2, 64, "fp32"),
    ((6, 20, 30), (3, 8, 8), (4, 6, 7), 1, 2, 128, "bf16"),
    ((6, 20, 30), (3, 8, 8), (4, 6, 7), 2, 1, 64, "fp32"),
    ((4, 8, 8), (2, 4, 4), (3, 10, 5), 1, 2, 128, "bf16"),
    ((9, 36, 44), (3, 16, 16), (5, 7, 11), 1, 2, 128, "bf16"),
]


@pytest.mark.parametrize("grid,cube,gg,B,heads,hd,dtype", GENERAL_CASES)
def test_aligned_order_chain(grid, cube, gg, B, heads, hd, dtype):
    N, G = grid[0] * grid[1] * grid[2], gg[0] * gg[1] * gg[2]
    ratios = tuple(a / b for a, b in zip(grid, gg))
    x = {s: mk(B * (N if s.endswith("_d") else G), heads, hd, s, dtype, seed=14)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    r_d, r_g, lse, y = general_aligned_chain(x, grid, cube, gg, B, hd, ratios)
    o = orc()
    pos = aligned_positions(grid, cube, gg)
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        # the permutation alone: bit-exact against the order's definition
        raw = x["v_g"][sg].cpu().view(torch.uint8).numpy().reshape(G, -1)
        want = np.empty_like(raw)
        want[pos] = raw
        assert y["v_g"][sg].cpu().view(torch.uint8).numpy().reshape(G, -1).tobytes() == \
            want.tobytes()
        rot = lambda s, g, sc: o.rope3d_grid(f64(x[s][sd if s.endswith("_d") else sg]), g,
                                             10000.0, split_for(hd), sc)
        qd = o.cube_reorder(rot("q_d", grid, (1, 1, 1)), grid, cube)
        kd = o.cube_reorder(rot("k_d", grid, (1, 1, 1)), grid, cube)
        vd = o.cube_reorder(f64(x["v_d"][sd]), grid, cube)
        ref_d, ref_g, ref_l = o.attention_full_aligned(
            qd, kd, vd, grid, cube, rot("q_g", gg, ratios), rot("k_g", gg, ratios),
            f64(x["v_g"][sg]), gg, hd ** -0.5, n_threads())
        got = np.concatenate([f64(r_d[sd]), f64(r_g[sg])])
        ref = np.concatenate([o.cube_unorder(ref_d, grid, cube), ref_g])
        assert_attn_close(got, ref, dtype, f"{grid} {gg} problem {b}")
        l_gpu = f64(lse[b])
        assert np.max(np.abs(l_gpu[:, :N] - ref_l[:, :N])) <= LSE_TOL[dtype]
        assert np.max(np.abs(l_gpu[:, N + pos] - ref_l[:, N:])) <= LSE_TOL[dtype]


@pytest.mark.parametrize("grid,cube,gg", [((6, 16, 16), (3, 8, 8), (6, 4, 4)),
                                          ((21, 48, 80), (3, 16, 16), (21, 12, 20)),
                                          ((4, 8, 8), (2, 4, 4), (2, 4, 4))])
def test_aligned_order_is_cube_order_for_integral_ratios(grid, cube, gg):
    """With integer ratios dividing the cube the aligned order is the global
    grid's cube order: same bits, same window ranges."""
    gcube = atlas.aligned_global_cube(grid, cube, gg)
    G = gg[0] * gg[1] * gg[2]
    x = mk(2 * G, 3, 128, "k_g", "bf16", seed=15)
    rg = atlas.make_rope(10000.0, split_for(128), tuple(a / b for a, b in zip(grid, gg)))
    a, b = torch.empty_like(x), torch.empty_like(x)
    atlas.aligned_global_reorder(x, a, grid, cube, gg, rg, batch=2)
    atlas.cube_reorder_batched(x, b, 2, gg, gcube, rg)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert torch.equal(atlas.aligned_global_offsets(grid, cube, gg),
                       atlas.cube_window_offsets(gg, gcube))
    # the inverse: of the rotated order, the rotated raster tokens; of the
    # plain order, the input bits
    z, xr, p = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    atlas.aligned_global_unorder(a, z, grid, cube, gg, batch=2)
    atlas.rope3d_batched(x, xr, 2, gg, rg)
    torch.cuda.synchronize()
    assert torch.equal(z.view(torch.uint8), xr.view(torch.uint8))
    atlas.aligned_global_reorder(x, p, grid, cube, gg, batch=2)
    atlas.aligned_global_unorder(p, z, grid, cube, gg, batch=2)
    torch.cuda.synchronize()
    assert torch.equal(z.view(torch.uint8), x.view(torch.uint8))


def test_aligned_order_8k_sampled():
    """8K geometry with partial cubes (detail 8x270x480, cubes 3x16x16,
    global 8x27x48: ratios 1, 10, 10, which do not divide the 16-token cube
    sides), 4 heads: sampled windows and global rows against the oracle."""
    grid, cube, gg, heads, hd = (8, 270, 480), (3, 16, 16), (8, 27, 48), 4, 128
    N, G = 8 * 270 * 480, 8 * 27 * 48
    x = {s: mk(N if s.endswith("_d") else G, heads, hd, s, "bf16", seed=16)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    y = {s: torch.empty_like(x[s]) for s in x}
    for s in ("q_d", "k_d", "v_d"):
        atlas.cube_reorder(x[s], y[s], grid, cube)
    for s in ("q_g", "k_g", "v_g"):
        atlas.aligned_global_reorder(x[s], y[s], grid, cube, gg)
    win = atlas.cube_window_offsets(grid, cube)
    gwin = atlas.aligned_global_offsets(grid, cube, gg)
    o_d, o_g = torch.empty_like(y["q_d"]), torch.empty_like(y["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(y["q_d"], y["k_d"], y["v_d"], y["q_g"], y["k_g"], y["v_g"], o_d,
                               o_g, lse, window_offsets=win.to(DEV),
                               global_window_offsets=gwin.to(DEV))
    r_g = torch.empty_like(o_g)
    atlas.aligned_global_unorder(o_g, r_g, grid, cube, gg)
    torch.cuda.synchronize()
    check_no_device_error()
    wo = win.numpy().astype(np.int64)
    nwin = wo.size - 1
    for head in (0, heads - 1):
        kg, vg = f64(x["k_g"][:, head]), f64(x["v_g"][:, head])
        for w in (0, 31, nwin // 2 + 7, nwin - 1):
            lo, hi = int(wo[w]), int(wo[w + 1])
            rows = np.arange(lo, hi)
            ref, ref_l = orc().attention_head_aligned(
                grid, cube, gg, hd ** -0.5, f64(y["k_d"][lo:hi, head]),
                f64(y["v_d"][lo:hi, head]), lo, kg, vg, rows, f64(y["q_d"][lo:hi, head]),
                n_threads())
            assert_attn_close(f64(o_d[lo:hi, head]), ref, "bf16", f"window {w} head {head}")
            assert np.max(np.abs(f64(lse[0, head, lo:hi]) - ref_l)) <= LSE_TOL["bf16"]
        g_rows = np.array([0, 5, 1234, G - 1])
        ref, _ = orc().attention_head_aligned(
            grid, cube, gg, hd ** -0.5, None, None, 0, kg, vg, N + g_rows,
            f64(x["q_g"][torch.as_tensor(g_rows, device=DEV), head]), n_threads())
        got = f64(r_g[torch.as_tensor(g_rows, device=DEV), head])
        assert_attn_close(got, ref, "bf16", f"global rows head {head}")


def test_aligned_order_random_shapes():
    """Forty random grid / cube / global-grid triples (ratios above and below
    one, partial cubes): the aligned order matches its definition bit for
    bit, batched, and the unorder inverts it."""
    rng = np.random.default_rng(77)
    for _ in range(40):
        grid = tuple(int(v) for v in rng.integers(1, 30, size=3))
        cube = tuple(int(min(g, v)) for g, v in zip(grid, rng.integers(1, 17, size=3)))
        gg = tuple(int(v) for v in rng.integers(1, 20, size=3))
        G = gg[0] * gg[1] * gg[2]
        B = int(rng.integers(1, 3))
        x = mk(B * G, 1, 64, "v_g", "bf16", seed=int(rng.integers(0, 1000)))
        y, z = torch.empty_like(x), torch.empty_like(x)
        atlas.aligned_global_reorder(x, y, grid, cube, gg, batch=B)
        atlas.aligned_global_unorder(y, z, grid, cube, gg, batch=B)
        torch.cuda.synchronize()
        check_no_device_error()
        pos = aligned_positions(grid, cube, gg)
        raw = x.cpu().view(torch.uint8).numpy().reshape(B, G, -1)
        want = np.empty_like(raw)
        want[:, pos] = raw
        assert y.cpu().view(torch.uint8).numpy().reshape(B, G, -1).tobytes() == want.tobytes(), \
            (grid, cube, gg)
        assert torch.equal(z.view(torch.uint8), x.view(torch.uint8))


def test_aligned_unorder_with_rope_is_rope_after_unorder():
    """The unorder with a rotation (used with the transposed RoPE to bring
    global dQ/dK back to raster order) rotates each token at its global raster
    position: the same bits as the plain unorder followed by the rotation."""
    grid, cube, gg = (6, 20, 30), (3, 8, 8), (4, 6, 7)
    G = gg[0] * gg[1] * gg[2]
    for dtype in ("bf16", "fp32"):
        x = mk(2 * G, 3, 128, "q_g", dtype, seed=17)
        rg = atlas.make_rope(10000.0, split_for(128), tuple(a / b for a, b in zip(grid, gg)))
        rt = atlas.transpose_rope(rg)
        a, b, c = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
        atlas.aligned_global_unorder(x, a, grid, cube, gg, rt, batch=2)
        atlas.aligned_global_unorder(x, b, grid, cube, gg, batch=2)
        atlas.rope3d_batched(b, c, 2, gg, rt)
        torch.cuda.synchronize()
        check_no_device_error()
        assert torch.equal(a.view(torch.uint8), c.view(torch.uint8)), dtype
