"""GPU parity where every persistent CTA walks many work units.

The attention kernels run one CTA per SM and hand each CTA a sequence of work
units (a head and up to 256 query rows forward; a head and 128 query or key
rows backward). A CTA's second and later units reuse its tensor memory, its
shared-memory rings and the phases of its barriers, and the forward releases
a unit's Q tiles before its last P*V. Those paths are only reached when the
units outnumber the SMs several times over, so the cases here are sized for
that (the unit count is asserted against the device's SM count) and compare
EVERY row with the fp64 oracle:
  * the fixed-window form at the 720p geometry (21x48x80 grid, 3x16x16
    cubes, 21x12x20 proxy grid) with 4 heads, and on a smaller grid with a
    batch of two problems and with head_dim 64;
  * the NARROW form with partial cubes (variable windows from offsets) and
    with the "aligned proxy tokens only" ranges;
  * the backward, both unit forms (dQ with query rows resident, dK/dV with
    key rows resident), fixed and variable windows and the aligned ranges.

Then the indicator-V mask probe on every row of the full-size workloads (720p,
4k, 4k_long with fixed windows; 8k29 with partial cubes, all global keys and
the aligned ranges): V's column 3 + (window id mod m) is 1 on that window's
keys (m = 61, then 59), column 2 is 1 on global keys (in the aligned variant
column 66 + (window id mod m) marks each window's aligned global keys
instead). A detail row may put mass only on its own window's columns and the
global column(s); a global row only on global columns. Everything else must
be exactly 0, and the row's mass must sum to 1.

Passages: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie 1
Fase 2 (window attention over the cube-reordered sequence) and Methodologie 2
(asymmetric hierarchical attention; global -> detail is -inf; position
alignment). Bounds as the other parity tests: bf16 max-abs 2e-2, mean-abs
2e-3, LSE 5e-3; gradients rel-rms 6e-3, rel-max 1.5e-2.
"""
import numpy as np
import pytest
import torch

from helpers import (aligned_positions, assert_attn_close, assert_lse_close,
                     check_no_device_error, f64, n_threads, orc)
from test_gpu_backward import assert_grads_close
from test_gpu_backward import inputs as bwd_inputs
from test_gpu_backward import run_gpu as bwd_run_gpu
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import WORKLOADS, normal

pytestmark = pytest.mark.gpu
DEV = "cuda"
UNIT_ROWS_FWD = 256     # query rows per forward work unit
TILE_ROWS_BWD = 128     # rows per backward work unit


def n_sm():
    return torch.cuda.get_device_properties(0).multi_processor_count


def ceil_div(a, b):
    return -(-a // b)


def mk(rows, heads, hd, stream, seed):
    return normal((rows, heads, hd), stream, torch.bfloat16, seed=seed, device=DEV)


def window_offsets(grid, cube):
    """Window offsets from the oracle (cube-order position of every cube)."""
    return orc().cube_windows(grid, cube)


def fwd_units(window_lens, G, heads):
    """Forward work units when windows of 128+ rows get units of their own."""
    upw = ceil_div(max(window_lens), UNIT_ROWS_FWD)
    return (len(window_lens) * upw + ceil_div(G, UNIT_ROWS_FWD)) * heads


def compare_all_rows(o_d, o_g, lse, ref_d, ref_g, ref_l, what):
    got = np.concatenate([f64(o_d).ravel(), f64(o_g).ravel()])
    ref = np.concatenate([ref_d.ravel(), ref_g.ravel()])
    assert_attn_close(got, ref, "bf16", what)
    l_gpu = lse if isinstance(lse, np.ndarray) else f64(lse)
    assert_lse_close(l_gpu.reshape(ref_l.shape), ref_l, "bf16", what)


# ---------------------------------------------------------------------------
# Forward, every row
# ---------------------------------------------------------------------------

def test_every_row_fixed_windows_720p_geometry():
    """The benchmark's kernel form (fixed windows of 768 rows, every global
    key) on the 720p geometry with 4 heads: 1340 units."""
    w = WORKLOADS["720p"]
    N, L, G, heads, hd = w.n_detail, w.window_len, w.n_global, 4, w.head_dim
    assert fwd_units([L] * (N // L), G, heads) >= 8 * n_sm()
    x = {s: mk(N if s.endswith("_d") else G, heads, hd, s, seed=31)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    o_d, o_g = torch.empty_like(x["q_d"]), torch.empty_like(x["q_g"])
    lse = torch.empty(heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn(x["q_d"], x["k_d"], x["v_d"], L, x["q_g"], x["k_g"], x["v_g"], o_d,
                            o_g, lse)
    torch.cuda.synchronize()
    check_no_device_error()
    ref_d, ref_g, ref_l = orc().attention_full(
        f64(x["q_d"]), f64(x["k_d"]), f64(x["v_d"]), L, f64(x["q_g"]), f64(x["k_g"]),
        f64(x["v_g"]), w.softmax_scale, n_threads())
    compare_all_rows(o_d, o_g, lse, ref_d, ref_g, ref_l, "720p geometry, 4 heads")


@pytest.mark.parametrize("B,heads,hd", [(2, 4, 128), (1, 8, 64)])
def test_every_row_batch_and_head_dim_64(B, heads, hd):
    """Fixed windows on a 9x48x80 grid (3x16x16 cubes, 9x12x20 proxy grid):
    two problems stacked along the rows with 4 heads, and head_dim 64 with 8
    heads; 1152 units either way."""
    grid, gg, L = (9, 48, 80), (9, 12, 20), 768
    N, G = 9 * 48 * 80, 9 * 12 * 20
    assert fwd_units([L] * (N // L), G, heads) * B >= 7 * n_sm()
    x = {s: mk(B * (N if s.endswith("_d") else G), heads, hd, s, seed=38)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    o_d, o_g = torch.empty_like(x["q_d"]), torch.empty_like(x["q_g"])
    lse = torch.empty(B, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(x["q_d"], x["k_d"], x["v_d"], x["q_g"], x["k_g"], x["v_g"], o_d,
                               o_g, lse, batch=B, window_len=L)
    torch.cuda.synchronize()
    check_no_device_error()
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        ref_d, ref_g, ref_l = orc().attention_full(
            f64(x["q_d"][sd]), f64(x["k_d"][sd]), f64(x["v_d"][sd]), L, f64(x["q_g"][sg]),
            f64(x["k_g"][sg]), f64(x["v_g"][sg]), hd ** -0.5, n_threads())
        compare_all_rows(o_d[sd], o_g[sg], lse[b], ref_d, ref_g, ref_l,
                         f"problem {b}, {heads} heads, head_dim {hd}")


def test_every_row_partial_cubes_narrow_form():
    """Variable windows (9x45x80 grid, 3x16x16 cubes: 45 windows of 768 or
    624 rows) with a 9x9x16 proxy grid, 6 heads: 846 units of the NARROW
    form."""
    grid, cube, gg, heads, hd = (9, 45, 80), (3, 16, 16), (9, 9, 16), 6, 128
    N, G = 9 * 45 * 80, 9 * 9 * 16
    off = window_offsets(grid, cube)
    lens = np.diff(off)
    assert set(lens.tolist()) == {768, 624}
    assert fwd_units(lens.tolist(), G, heads) >= 5 * n_sm()
    x = {s: mk(N if s.endswith("_d") else G, heads, hd, s, seed=32)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    o_d, o_g = torch.empty_like(x["q_d"]), torch.empty_like(x["q_g"])
    lse = torch.empty(heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_windows(x["q_d"], x["k_d"], x["v_d"],
                                    torch.as_tensor(off, dtype=torch.int32, device=DEV),
                                    x["q_g"], x["k_g"], x["v_g"], o_d, o_g, lse)
    torch.cuda.synchronize()
    check_no_device_error()
    ref_d, ref_g, ref_l = orc().attention_full(
        f64(x["q_d"]), f64(x["k_d"]), f64(x["v_d"]), 1, f64(x["q_g"]), f64(x["k_g"]),
        f64(x["v_g"]), hd ** -0.5, n_threads(), win_off=off)
    compare_all_rows(o_d, o_g, lse, ref_d, ref_g, ref_l, "partial cubes, 6 heads")


def test_every_row_aligned_ranges_narrow_form():
    """Aligned proxy tokens only (9x48x80 grid, 3x16x16 cubes, 9x12x20 proxy
    grid: 48 aligned global keys per window), 8 heads: 1152 units of the
    NARROW form. The GPU takes the global tokens in the aligned order, the
    oracle in raster order with its coordinate-defined predicate."""
    grid, cube, gg, heads, hd = (9, 48, 80), (3, 16, 16), (9, 12, 20), 8, 128
    N, G = 9 * 48 * 80, 9 * 12 * 20
    assert fwd_units([768] * (N // 768), G, heads) >= 7 * n_sm()
    x = {s: mk(N if s.endswith("_d") else G, heads, hd, s, seed=33)
         for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    pos = aligned_positions(grid, cube, gg)     # aligned place of raster token g
    pos_t = torch.as_tensor(pos, device=DEV)
    y = {s: torch.empty_like(x[s]) for s in ("q_g", "k_g", "v_g")}
    for s in y:
        y[s][pos_t] = x[s]
    o_d, o_g = torch.empty_like(x["q_d"]), torch.empty_like(x["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(x["q_d"], x["k_d"], x["v_d"], y["q_g"], y["k_g"], y["v_g"], o_d,
                               o_g, lse,
                               window_offsets=atlas.cube_window_offsets(grid, cube).to(DEV),
                               global_window_offsets=atlas.aligned_global_offsets(
                                   grid, cube, gg).to(DEV))
    torch.cuda.synchronize()
    check_no_device_error()
    ref_d, ref_g, ref_l = orc().attention_full_aligned(
        f64(x["q_d"]), f64(x["k_d"]), f64(x["v_d"]), grid, cube, f64(x["q_g"]), f64(x["k_g"]),
        f64(x["v_g"]), gg, hd ** -0.5, n_threads())
    l_gpu = f64(lse[0])
    compare_all_rows(o_d, o_g[pos_t], np.concatenate([l_gpu[:, :N], l_gpu[:, N + pos]], axis=1),
                     ref_d, ref_g, ref_l, "aligned ranges, 8 heads")


# ---------------------------------------------------------------------------
# Backward, every row
# ---------------------------------------------------------------------------

def test_every_row_backward_fixed_windows():
    """15x32x48 grid, 3x16x16 cubes (30 windows of 768), 15x8x12 proxy
    grid, 4 heads: 768 units in each form."""
    grid, gg, heads, hd, L = (15, 32, 48), (15, 8, 12), 4, 128, 768
    N, G = 15 * 32 * 48, 15 * 8 * 12
    assert ceil_div(N + G, TILE_ROWS_BWD) * heads >= 5 * n_sm()
    t = bwd_inputs(1, N, G, heads, hd, "bf16", seed=34)
    got = bwd_run_gpu(t, 1, heads, N, G, window_len=L)
    ref = orc().attention_bwd_full(f64(t["q_d"]), f64(t["k_d"]), f64(t["v_d"]), L,
                                   f64(t["q_g"]), f64(t["k_g"]), f64(t["v_g"]), f64(t["do_d"]),
                                   f64(t["do_g"]), hd ** -0.5, n_threads())
    assert_grads_close([f64(g) for g in got], ref, "bf16", "backward, fixed windows")


def test_every_row_backward_partial_cubes():
    """9x45x80 grid, 3x16x16 cubes (768- and 624-row windows), 9x9x16
    proxy grid, 3 heads: 792 units in each form."""
    grid, cube, gg, heads, hd = (9, 45, 80), (3, 16, 16), (9, 9, 16), 3, 128
    N, G = 9 * 45 * 80, 9 * 9 * 16
    assert ceil_div(N + G, TILE_ROWS_BWD) * heads >= 5 * n_sm()
    off = window_offsets(grid, cube)
    t = bwd_inputs(1, N, G, heads, hd, "bf16", seed=35)
    got = bwd_run_gpu(t, 1, heads, N, G,
                      window_offsets=torch.as_tensor(off, dtype=torch.int32, device=DEV))
    ref = orc().attention_bwd_full(f64(t["q_d"]), f64(t["k_d"]), f64(t["v_d"]), 1,
                                   f64(t["q_g"]), f64(t["k_g"]), f64(t["v_g"]), f64(t["do_d"]),
                                   f64(t["do_g"]), hd ** -0.5, n_threads(), win_off=off)
    assert_grads_close([f64(g) for g in got], ref, "bf16", "backward, partial cubes")


def test_every_row_backward_aligned_ranges():
    """Aligned proxy tokens only (9x48x80 grid, 3x16x16 cubes, 9x12x20 proxy
    grid), 4 heads: 1148 units in each form. The GPU takes the global tokens
    in the aligned order, the oracle in raster order."""
    grid, cube, gg, heads, hd = (9, 48, 80), (3, 16, 16), (9, 12, 20), 4, 128
    N, G = 9 * 48 * 80, 9 * 12 * 20
    assert ceil_div(N + G, TILE_ROWS_BWD) * heads >= 7 * n_sm()
    t = bwd_inputs(1, N, G, heads, hd, "bf16", seed=37)
    pos_t = torch.as_tensor(aligned_positions(grid, cube, gg), device=DEV)
    y = dict(t)
    for s in ("q_g", "k_g", "v_g", "do_g"):      # raster -> aligned order
        y[s] = torch.empty_like(t[s])
        y[s][pos_t] = t[s]
    got = bwd_run_gpu(y, 1, heads, N, G,
                      window_offsets=atlas.cube_window_offsets(grid, cube).to(DEV),
                      global_window_offsets=atlas.aligned_global_offsets(grid, cube, gg).to(DEV))
    got = [f64(g) for g in got[:3]] + [f64(g[pos_t]) for g in got[3:]]   # back to raster
    ref = orc().attention_bwd_full_aligned(
        f64(t["q_d"]), f64(t["k_d"]), f64(t["v_d"]), grid, cube, f64(t["q_g"]), f64(t["k_g"]),
        f64(t["v_g"]), gg, f64(t["do_d"]), f64(t["do_g"]), hd ** -0.5, n_threads())
    assert_grads_close(got, ref, "bf16", "backward, aligned ranges")


# ---------------------------------------------------------------------------
# Mask probe on every row of the full-size workloads
# ---------------------------------------------------------------------------

CHUNK = 1 << 16   # rows checked per step (bounded host-side memory)


def check_probe_rows(o, cls, m, own_col0, glob_cols, glob_cls=None):
    """o: [rows, heads, D] output of indicator-V attention. For every row,
    the mass must lie only on column own_col0 + cls[row] and on the global
    columns (glob_cols, or glob_col0 + glob_cls[row] when glob_cls is given:
    the aligned variant), be > 0 on the own column and sum to 1 (8e-3)."""
    rows, heads, D = o.shape
    for c0 in range(0, rows, CHUNK):
        c1 = min(rows, c0 + CHUNK)
        blk = o[c0:c1].float()                                   # [r, heads, D]
        allowed = torch.zeros(c1 - c0, D, dtype=torch.bool, device=DEV)
        r = torch.arange(c1 - c0, device=DEV)
        if cls is not None:
            allowed[r, own_col0 + cls[c0:c1]] = True
        if glob_cls is not None:
            allowed[r, glob_cols + glob_cls[c0:c1]] = True
        else:
            allowed[:, glob_cols] = True
        outside = blk.masked_fill(allowed[:, None, :], 0.0)
        assert torch.count_nonzero(outside) == 0, f"mass outside the allowed set (mod {m})"
        if cls is not None:
            own = blk[r, :, own_col0 + cls[c0:c1]]
            assert torch.all(own > 0), f"no mass on the own window (mod {m})"
        total = blk.sum(dim=2)
        assert float((total - 1).abs().max()) <= 8e-3, f"row mass != 1 (mod {m})"


def probe(name, variant):
    w = WORKLOADS[name]
    N, G, heads, hd = w.n_detail, w.n_global, w.heads, w.head_dim
    torch.cuda.empty_cache()
    q_d, k_d = mk(N, heads, hd, "q_d", 36), mk(N, heads, hd, "k_d", 36)
    q_g, k_g = mk(G, heads, hd, "q_g", 36), mk(G, heads, hd, "k_g", 36)
    if w.partial or variant == "aligned":
        off = torch.as_tensor(window_offsets(w.grid, w.cube), dtype=torch.int64, device=DEV)
    else:
        off = torch.arange(0, N + 1, w.window_len, device=DEV)
    n_win = off.numel() - 1
    win_of_row = torch.repeat_interleave(torch.arange(n_win, device=DEV), off.diff())
    layout = {}
    if w.partial or variant == "aligned":
        layout["window_offsets"] = off.to(torch.int32)
    else:
        layout["window_len"] = w.window_len
    gwin_of_row = None
    if variant == "aligned":
        gwin = atlas.aligned_global_offsets(w.grid, w.cube, w.global_grid).to(DEV)
        layout["global_window_offsets"] = gwin
        gwin_of_row = torch.repeat_interleave(torch.arange(n_win, device=DEV),
                                              gwin.to(torch.int64).diff())
    v_d = torch.empty(N, heads, hd, dtype=torch.bfloat16, device=DEV)
    v_g = torch.empty(G, heads, hd, dtype=torch.bfloat16, device=DEV)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(q_g)
    for m in (61, 59):
        assert 3 + m <= 66 and 66 + m <= hd
        cls = win_of_row % m
        v_d.zero_()
        v_d[torch.arange(N, device=DEV), :, 3 + cls] = 1.0
        v_g.zero_()
        if variant == "aligned":
            v_g[torch.arange(G, device=DEV), :, 66 + gwin_of_row % m] = 1.0
        else:
            v_g[:, :, 2] = 1.0
        o_d.fill_(float("nan"))
        o_g.fill_(float("nan"))
        atlas.local_global_attn_ex(q_d, k_d, v_d, q_g, k_g, v_g, o_d, o_g, None, **layout)
        torch.cuda.synchronize()
        check_no_device_error()
        if variant == "aligned":
            # a detail row: own window column, and its window's aligned global
            # keys' column (the same class); a global row: any global column
            check_probe_rows(o_d, cls, m, 3, 66, glob_cls=cls)
            gcols = torch.arange(66, 66 + m, device=DEV)
            check_probe_rows(o_g, None, m, 0, gcols)
        else:
            check_probe_rows(o_d, cls, m, 3, 2)
            check_probe_rows(o_g, None, m, 0, 2)
            assert torch.all(o_d[:, :, 2].float() > 0), "a detail row missed the global keys"
    del q_d, k_d, q_g, k_g, v_d, v_g, o_d, o_g
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,variant", [("720p", "all"), ("4k", "all"), ("4k_long", "all"),
                                          ("8k29", "all"), ("8k29", "aligned")])
def test_full_size_mask_probe_every_row(name, variant):
    probe(name, variant)
