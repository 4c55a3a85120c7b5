"""GPU parity for grids the cube does not divide (partial cubes, variable
windows) against the fp64 oracle, through the C-ABI.

Reading of "Technische Samenvatting: AtlasVid", Methodologie 1 Fase 2 (the
tokens of one cube are made contiguous) where the pages are silent: the last
cube along an axis the cube size does not divide is partial, stays
contiguous, and is its own, shorter window.
"""
import numpy as np
import pytest
import torch

from helpers import (assert_attn_close, assert_rope_close, check_no_device_error, f64, n_threads,
                     orc)
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import normal

pytestmark = pytest.mark.gpu
DEV = "cuda"

# grid, cube, heads, head_dim, dtype
CASES = [
    ((5, 7, 9), (2, 3, 4), 2, 64, "fp32"),
    ((5, 7, 9), (2, 3, 4), 3, 128, "bf16"),
    ((4, 8, 10), (2, 4, 4), 2, 64, "bf16"),
    ((3, 17, 23), (3, 16, 16), 2, 128, "bf16"),
    ((1, 3, 2), (3, 4, 5), 1, 64, "bf16"),
]


def tdt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def split_for(hd):
    return (16, 24, 24) if hd == 64 else (44, 42, 42)


@pytest.mark.parametrize("grid,cube,heads,hd,dtype", CASES)
def test_partial_reorder_unorder_bit_exact(grid, cube, heads, hd, dtype):
    n = grid[0] * grid[1] * grid[2]
    x = normal((n, heads, hd), "v_d", tdt(dtype), device=DEV)
    y, z, y2 = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    atlas.cube_reorder(x, y, grid, cube)
    atlas.cube_unorder(y, z, grid, cube)
    atlas.cube_reorder_noalloc(x, y2, grid, cube)
    torch.cuda.synchronize()
    check_no_device_error()
    expect = orc().cube_reorder(x.cpu().view(torch.uint8).numpy().reshape(n, -1), grid, cube)
    assert y.cpu().view(torch.uint8).numpy().reshape(n, -1).tobytes() == expect.tobytes()
    assert torch.equal(z.view(torch.uint8), x.view(torch.uint8))
    assert torch.equal(y2.view(torch.uint8), y.view(torch.uint8))


@pytest.mark.parametrize("grid,cube,heads,hd,dtype", CASES)
def test_partial_reorder_rope(grid, cube, heads, hd, dtype):
    n = grid[0] * grid[1] * grid[2]
    split, scales = split_for(hd), (2.0, 1.0, 1.0)
    x = normal((n, heads, hd), "q_d", tdt(dtype), device=DEV)
    y = torch.empty_like(x)
    atlas.cube_reorder(x, y, grid, cube, atlas.make_rope(10000.0, split, scales))
    torch.cuda.synchronize()
    xd = f64(x)
    exact = orc().cube_reorder(orc().rope3d_grid(xd, grid, 10000.0, split, scales), grid, cube)
    assert_rope_close(f64(y), exact, orc().cube_reorder(xd, grid, cube), dtype)


@pytest.mark.parametrize("grid,cube,heads,hd,dtype", CASES)
def test_partial_cube_chain(grid, cube, heads, hd, dtype):
    """raster -> reorder(+RoPE) -> variable-window attention -> unorder,
    against the oracle's chain in raster order."""
    n = grid[0] * grid[1] * grid[2]
    G, split = 37, split_for(hd)
    rd = atlas.make_rope(10000.0, split, (1.0, 1.0, 1.0))
    mk = lambda rows, s: normal((rows, heads, hd), s, tdt(dtype), seed=1, device=DEV)
    x_q, x_k, x_v = mk(n, "q_d"), mk(n, "k_d"), mk(n, "v_d")
    q_g, k_g, v_g = mk(G, "q_g"), mk(G, "k_g"), mk(G, "v_g")
    q_d, k_d, v_d = torch.empty_like(x_q), torch.empty_like(x_k), torch.empty_like(x_v)
    atlas.cube_reorder(x_q, q_d, grid, cube, rd)
    atlas.cube_reorder(x_k, k_d, grid, cube, rd)
    atlas.cube_reorder(x_v, v_d, grid, cube)
    off = atlas.cube_window_offsets(grid, cube).to(DEV)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(q_g)
    lse = torch.empty(heads, n + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_windows(q_d, k_d, v_d, off, q_g, k_g, v_g, o_d, o_g, lse)
    o_r = torch.empty_like(o_d)
    atlas.cube_unorder(o_d, o_r, grid, cube)
    torch.cuda.synchronize()
    check_no_device_error()
    o = orc()
    rq = o.cube_reorder(o.rope3d_grid(f64(x_q), grid, 10000.0, split, (1, 1, 1)), grid, cube)
    rk = o.cube_reorder(o.rope3d_grid(f64(x_k), grid, 10000.0, split, (1, 1, 1)), grid, cube)
    rv = o.cube_reorder(f64(x_v), grid, cube)
    win = o.cube_windows(grid, cube)
    ref_d, ref_g, ref_lse = o.attention_full(rq, rk, rv, 1, f64(q_g), f64(k_g), f64(v_g),
                                             hd ** -0.5, n_threads(), win_off=win)
    got = np.concatenate([f64(o_r), f64(o_g)])
    ref = np.concatenate([o.cube_unorder(ref_d, grid, cube), ref_g])
    assert_attn_close(got, ref, dtype, f"{grid} {cube}")
    assert np.max(np.abs(f64(lse) - ref_lse)) <= (5e-3 if dtype == "bf16" else 1e-4)


def test_offsets_of_fixed_windows_match_fixed_path():
    """Offsets k*L select exactly the fixed-length path's result."""
    N, L, G, heads, hd = 3072, 768, 300, 2, 128
    mk = lambda rows, s: normal((rows, heads, hd), s, torch.bfloat16, seed=2, device=DEV)
    q_d, k_d, v_d, q_g, k_g, v_g = (mk(N, "q_d"), mk(N, "k_d"), mk(N, "v_d"), mk(G, "q_g"),
                                    mk(G, "k_g"), mk(G, "v_g"))
    a_d, a_g = torch.empty_like(q_d), torch.empty_like(q_g)
    b_d, b_g = torch.empty_like(q_d), torch.empty_like(q_g)
    atlas.local_global_attn(q_d, k_d, v_d, L, q_g, k_g, v_g, a_d, a_g)
    off = torch.arange(0, N + 1, L, dtype=torch.int32, device=DEV)
    atlas.local_global_attn_windows(q_d, k_d, v_d, off, q_g, k_g, v_g, b_d, b_g)
    torch.cuda.synchronize()
    assert torch.equal(a_d.view(torch.int16), b_d.view(torch.int16))
    assert torch.equal(a_g.view(torch.int16), b_g.view(torch.int16))


def test_partial_cubes_at_scale_sampled():
    """720p-like grid whose H the cube does not divide (partial cubes of 13
    rows), 8 heads; sampled windows (a full one, a partial one, the last) on
    the first and last head against the oracle."""
    grid, cube, G, heads, hd = (21, 45, 80), (3, 16, 16), 5040, 8, 128
    n = grid[0] * grid[1] * grid[2]
    mk = lambda rows, s: normal((rows, heads, hd), s, torch.bfloat16, seed=3, device=DEV)
    q_d, k_d, v_d = mk(n, "q_d"), mk(n, "k_d"), mk(n, "v_d")
    q_g, k_g, v_g = mk(G, "q_g"), mk(G, "k_g"), mk(G, "v_g")
    off_h = atlas.cube_window_offsets(grid, cube)
    off = off_h.to(DEV)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(q_g)
    atlas.local_global_attn_windows(q_d, k_d, v_d, off, q_g, k_g, v_g, o_d, o_g)
    torch.cuda.synchronize()
    check_no_device_error()
    offs = off_h.numpy().astype(np.int64)
    sizes = np.diff(offs)
    wins = [0, int(np.argmin(sizes)), len(sizes) - 1]
    assert sizes[wins[1]] < 768
    for head in (0, heads - 1):
        kg, vg = f64(k_g[:, head]), f64(v_g[:, head])
        for w in wins:
            lo, hi = int(offs[w]), int(offs[w + 1])
            rows = np.arange(lo, hi)
            ref, _ = orc().attention_head(n, 1, G, hd ** -0.5, f64(k_d[lo:hi, head]),
                                          f64(v_d[lo:hi, head]), lo, kg, vg, rows,
                                          f64(q_d[lo:hi, head]), n_threads(), win_off=offs)
            assert_attn_close(f64(o_d[lo:hi, head]), ref, "bf16", f"window {w} head {head}")


@pytest.mark.parametrize("name", ["8k29", "2k321"])
def test_long_shapes_full_size_sampled(name):
    """The 8K / 29-frame and 2K / 321-frame shapes at full size (40 heads,
    partial cubes) through the window-offset entry the benchmark times:
    sampled windows (first, smallest, last) and global rows on the first and
    last head against the oracle; V = 1 gives 1 on every row."""
    from video_dit_windowed_b200.workloads import WORKLOADS
    w = WORKLOADS[name]
    torch.cuda.empty_cache()
    N, G, heads, hd = w.n_detail, w.n_global, w.heads, w.head_dim
    mk = lambda rows, s: normal((rows, heads, hd), s, torch.bfloat16, seed=4, device=DEV)
    q_d, k_d, v_d = mk(N, "q_d"), mk(N, "k_d"), mk(N, "v_d")
    q_g, k_g, v_g = mk(G, "q_g"), mk(G, "k_g"), mk(G, "v_g")
    off_h = atlas.cube_window_offsets(w.grid, w.cube)
    off = off_h.to(DEV)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(q_g)
    lse = torch.empty(heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_windows(q_d, k_d, v_d, off, q_g, k_g, v_g, o_d, o_g, lse)
    torch.cuda.synchronize()
    check_no_device_error()
    offs = off_h.numpy().astype(np.int64)
    sizes = np.diff(offs)
    assert sizes.min() < w.window_len and offs.size - 1 == w.n_windows
    g_rows = np.array([0, 1, G // 2, G - 2, G - 1])
    for head in (0, heads - 1):
        kg, vg = f64(k_g[:, head]), f64(v_g[:, head])
        for win in (0, int(np.argmin(sizes)), len(sizes) - 1):
            lo, hi = int(offs[win]), int(offs[win + 1])
            ref, ref_l = orc().attention_head(N, 1, G, hd ** -0.5, f64(k_d[lo:hi, head]),
                                              f64(v_d[lo:hi, head]), lo, kg, vg,
                                              np.arange(lo, hi), f64(q_d[lo:hi, head]),
                                              n_threads(), win_off=offs)
            assert_attn_close(f64(o_d[lo:hi, head]), ref, "bf16", f"{name} window {win}")
            assert np.max(np.abs(f64(lse[head, lo:hi]) - ref_l)) <= 5e-3
        idx = torch.as_tensor(g_rows, device=DEV)
        ref, _ = orc().attention_head(N, 1, G, hd ** -0.5, None, None, 0, kg, vg, N + g_rows,
                                      f64(q_g[idx, head]), n_threads(), win_off=offs)
        assert_attn_close(f64(o_g[idx, head]), ref, "bf16", f"{name} global rows")
    del o_d, o_g, lse
    v_d.fill_(1.0)
    v_g.fill_(1.0)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(q_g)
    atlas.local_global_attn_windows(q_d, k_d, v_d, off, q_g, k_g, v_g, o_d, o_g)
    torch.cuda.synchronize()
    for t in (o_d, o_g):
        assert float((t.float() - 1).abs().max()) <= 8e-3
    del q_d, k_d, v_d, q_g, k_g, v_g, o_d, o_g
    torch.cuda.empty_cache()


# Window offsets that exercise both unit forms of the tensor-core forward:
# long windows of unequal lengths (own units, empty trailing slots, a
# 100-row window and a one-row window inside a long-window layout), and a
# layout whose slots would exceed three times the packed count (one long
# window among many short ones: packed units over the union of windows).
OFFSET_CASES = [
    [0, 700, 1212, 1213, 1313, 2081, 2336, 2592],
    [0, 1000] + list(range(1001, 1501)),
    [0, 128, 256, 384, 640, 900],
    [0, 384, 768, 1152],
]


@pytest.mark.parametrize("offsets", OFFSET_CASES)
@pytest.mark.parametrize("aligned", [False, True])
def test_window_units_match_oracle(offsets, aligned):
    """Variable windows against the oracle, all keys or per-window global
    ranges (some empty), bf16 on the tensor-core path."""
    off = torch.tensor(offsets, dtype=torch.int32)
    N, G, heads, hd = offsets[-1], 333, 2, 128
    nw = len(offsets) - 1
    t = {s: normal((N if s.endswith("_d") else G, heads, hd), s, torch.bfloat16, seed=31,
                   device=DEV) for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    gwin = None
    if aligned:
        rng = np.random.default_rng(5)
        cuts = np.sort(rng.integers(0, G + 1, size=nw - 1))
        cuts[nw // 2 - 1:nw // 2 + 1] = cuts[nw // 2 - 1]       # an empty range
        gwin = np.concatenate([[0], cuts, [G]]).astype(np.int32)
    o_d, o_g = torch.empty_like(t["q_d"]), torch.empty_like(t["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(
        t["q_d"], t["k_d"], t["v_d"], t["q_g"], t["k_g"], t["v_g"], o_d, o_g, lse,
        window_offsets=off.to(DEV),
        global_window_offsets=torch.from_numpy(gwin).to(DEV) if aligned else None)
    torch.cuda.synchronize()
    check_no_device_error()
    woff = np.asarray(offsets, dtype=np.int64)
    for h in range(heads):
        kd, vd = f64(t["k_d"][:, h]), f64(t["v_d"][:, h])
        kg, vg = f64(t["k_g"][:, h]), f64(t["v_g"][:, h])
        q = np.concatenate([f64(t["q_d"][:, h]), f64(t["q_g"][:, h])])
        if aligned:
            # window w alone, with its global range as the whole global set
            parts, lparts = [], []
            for w in range(nw):
                s0, e0, g0, g1 = int(woff[w]), int(woff[w + 1]), int(gwin[w]), int(gwin[w + 1])
                o_w, l_w = orc().attention_head(e0 - s0, e0 - s0, g1 - g0, hd ** -0.5,
                                                kd[s0:e0], vd[s0:e0], 0, kg[g0:g1], vg[g0:g1],
                                                np.arange(e0 - s0, dtype=np.int64), q[s0:e0],
                                                n_threads())
                parts.append(o_w)
                lparts.append(l_w)
            o_g_ref, l_g_ref = orc().attention_head(0, 1, G, hd ** -0.5, None, None, 0, kg, vg,
                                                    np.arange(G, dtype=np.int64), q[N:],
                                                    n_threads())
            ref = np.concatenate(parts + [o_g_ref])
            ref_l = np.concatenate(lparts + [l_g_ref])
        else:
            ref, ref_l = orc().attention_head(N, 1, G, hd ** -0.5, kd, vd, 0, kg, vg,
                                              np.arange(N + G, dtype=np.int64), q, n_threads(),
                                              woff)
        got = np.concatenate([f64(o_d[:, h]), f64(o_g[:, h])])
        assert_attn_close(got, ref, "bf16", f"{offsets[:4]} head {h}")
        assert np.max(np.abs(f64(lse[0, h]) - ref_l)) <= 5e-3
