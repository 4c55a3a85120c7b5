"""GPU parity of the attention backward (dQ, dK, dV) against the fp64 oracle,
through the C-ABI.

The GPU forward gives O and the LSE; dO is seeded N(0,1); the GPU backward
and the oracle's (softmax-Jacobian definition, fp64, on the same bf16/fp32
inputs) are compared per gradient tensor, relative to the reference's scale:
  rel_max = max|g - ref| / max|ref|,  rel_rms = rms(g - ref) / rms(ref).
Bounds (derived from the arithmetic): bf16 keeps 8 significant bits, so each
of P, dS, O (inside delta) and the output is rounded with relative error up
to 2^-9 ~ 2e-3; rounding the output alone gives rel_rms ~ 2^-9/sqrt(3) ~
1.1e-3, and the rounded P and dS add about as much again. bf16: rel_rms <=
6e-3, rel_max <= 1.5e-2 (measured on B200: rel_rms 2.4e-3, rel_max <= 4.5e-3
over the cases below). fp32 (exact fp32 products, expf, accumulation over up
to ~1e3 terms): rel_rms <= 2e-6, rel_max <= 5e-6 (measured <= 4e-7 / 7e-7).
"""
import numpy as np
import pytest
import torch

from helpers import check_no_device_error, f64, n_threads, orc
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import normal

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = {"bf16": (6e-3, 1.5e-2), "fp32": (2e-6, 5e-6)}
NAMES = ("dq_d", "dk_d", "dv_d", "dq_g", "dk_g", "dv_g")


def tdt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def assert_grads_close(got, ref, dtype, what=""):
    rms_tol, max_tol = TOL[dtype]
    for name, g, r in zip(NAMES, got, ref):
        if r.size == 0:
            continue
        scale_max = float(np.max(np.abs(r)))
        scale_rms = float(np.sqrt(np.mean(r * r)))
        err = np.abs(g - r)
        rel_max = float(err.max()) / max(scale_max, 1e-30)
        rel_rms = float(np.sqrt(np.mean(err * err))) / max(scale_rms, 1e-30)
        assert rel_rms <= rms_tol and rel_max <= max_tol, (
            f"{what} {name}: rel_rms {rel_rms:.2e} rel_max {rel_max:.2e}")


def run_gpu(t, B, heads, N, G, **layout):
    """Forward then backward on the GPU; returns the six gradients."""
    o_d, o_g = torch.empty_like(t["q_d"]), torch.empty_like(t["q_g"])
    lse = torch.empty(B, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(t["q_d"], t["k_d"], t["v_d"], t["q_g"], t["k_g"], t["v_g"], o_d,
                               o_g, lse, batch=B, **layout)
    grads = [torch.empty_like(t[s]) for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")]
    atlas.local_global_attn_bwd(t["q_d"], t["k_d"], t["v_d"], o_d, t["do_d"], t["q_g"],
                                t["k_g"], t["v_g"], o_g, t["do_g"], lse, *grads, batch=B,
                                **layout)
    torch.cuda.synchronize()
    check_no_device_error()
    return grads


def inputs(B, N, G, heads, hd, dtype, seed):
    streams = {"q_d": "q_d", "k_d": "k_d", "v_d": "v_d", "q_g": "q_g", "k_g": "k_g",
               "v_g": "v_g", "do_d": 0, "do_g": 3}
    out = {}
    for name, st in streams.items():
        rows = B * (N if name.endswith("_d") else G)
        s = seed + (100 if name.startswith("do") else 0)
        out[name] = normal((rows, heads, hd), st, tdt(dtype), seed=s, device=DEV)
    return out


# N, L, G, heads, hd, dtype
FIXED = [
    (1536, 768, 300, 2, 128, "bf16"),
    (960, 48, 130, 2, 64, "bf16"),
    (512, 256, 0, 2, 128, "bf16"),
    (0, 1, 300, 2, 128, "bf16"),
    (640, 128, 77, 1, 64, "bf16"),
    (256, 32, 32, 2, 64, "fp32"),
    (384, 96, 45, 2, 128, "fp32"),
]


@pytest.mark.parametrize("N,L,G,heads,hd,dtype", FIXED)
def test_backward_fixed_windows(N, L, G, heads, hd, dtype):
    t = inputs(1, N, G, heads, hd, dtype, seed=21)
    got = run_gpu(t, 1, heads, N, G, window_len=L if N else 0)
    ref = orc().attention_bwd_full(f64(t["q_d"]), f64(t["k_d"]), f64(t["v_d"]), max(L, 1),
                                   f64(t["q_g"]), f64(t["k_g"]), f64(t["v_g"]), f64(t["do_d"]),
                                   f64(t["do_g"]), hd ** -0.5, n_threads())
    assert_grads_close([f64(g) for g in got], ref, dtype, f"N={N} L={L} G={G}")


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_backward_partial_cubes_batched(dtype):
    grid, cube, G, B, heads, hd = (5, 7, 9), (2, 3, 4), 29, 2, 2, 64
    N = 315
    off = atlas.cube_window_offsets(grid, cube)
    t = inputs(B, N, G, heads, hd, dtype, seed=22)
    got = run_gpu(t, B, heads, N, G, window_offsets=off.to(DEV))
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        ref = orc().attention_bwd_full(
            f64(t["q_d"][sd]), f64(t["k_d"][sd]), f64(t["v_d"][sd]), 1, f64(t["q_g"][sg]),
            f64(t["k_g"][sg]), f64(t["v_g"][sg]), f64(t["do_d"][sd]), f64(t["do_g"][sg]),
            hd ** -0.5, n_threads(), win_off=off.numpy().astype(np.int64))
        part = [f64(g[sd if i < 3 else sg]) for i, g in enumerate(got)]
        assert_grads_close(part, ref, dtype, f"problem {b}")


@pytest.mark.parametrize("dtype,B", [("bf16", 1), ("bf16", 2), ("fp32", 1)])
def test_backward_aligned(dtype, B):
    """Aligned variant; the global tokens go to the GPU in global cube order
    and the oracle takes them in raster order."""
    grid, cube, gg, heads, hd = (6, 16, 16), (3, 8, 8), (6, 4, 4), 2, 128
    N, G = 1536, 96
    gcube = atlas.aligned_global_cube(grid, cube, gg)
    t = inputs(B, N, G, heads, hd, dtype, seed=23)
    tg = dict(t)
    for s in ("q_g", "k_g", "v_g", "do_g"):
        tg[s] = torch.empty_like(t[s])
        atlas.cube_reorder_batched(t[s], tg[s], B, gg, gcube)
    gwin = atlas.cube_window_offsets(gg, gcube).to(DEV)
    got = run_gpu(tg, B, heads, N, G, window_len=192, global_window_offsets=gwin)
    # global gradients back to raster order
    for i in (3, 4, 5):
        r = torch.empty_like(got[i])
        atlas.cube_unorder_batched(got[i], r, B, gg, gcube)
        got[i] = r
    torch.cuda.synchronize()
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        ref = orc().attention_bwd_full_aligned(
            f64(t["q_d"][sd]), f64(t["k_d"][sd]), f64(t["v_d"][sd]), grid, cube,
            f64(t["q_g"][sg]), f64(t["k_g"][sg]), f64(t["v_g"][sg]), gg, f64(t["do_d"][sd]),
            f64(t["do_g"][sg]), hd ** -0.5, n_threads())
        part = [f64(g[sd if i < 3 else sg]) for i, g in enumerate(got)]
        assert_grads_close(part, ref, dtype, f"aligned problem {b}")


@pytest.mark.parametrize("dtype,B", [("bf16", 1), ("fp32", 2)])
def test_backward_aligned_order_general(dtype, B):
    """Aligned variant at ratios that are not integers (detail 6x20x30 with
    cubes 3x8x8 and partial cubes, global 4x6x7): global tokens in the
    aligned order on the GPU, raster order in the oracle."""
    grid, cube, gg, heads, hd = (6, 20, 30), (3, 8, 8), (4, 6, 7), 2, 128
    N, G = 3600, 168
    win = atlas.cube_window_offsets(grid, cube)
    gwin = atlas.aligned_global_offsets(grid, cube, gg)
    t = inputs(B, N, G, heads, hd, dtype, seed=24)
    tg = dict(t)
    for s in ("q_d", "k_d", "v_d", "do_d"):
        tg[s] = torch.empty_like(t[s])
        atlas.cube_reorder_batched(t[s], tg[s], B, grid, cube)
    for s in ("q_g", "k_g", "v_g", "do_g"):
        tg[s] = torch.empty_like(t[s])
        atlas.aligned_global_reorder(t[s], tg[s], grid, cube, gg, batch=B)
    got = run_gpu(tg, B, heads, N, G, window_offsets=win.to(DEV),
                  global_window_offsets=gwin.to(DEV))
    for i in range(6):
        r = torch.empty_like(got[i])
        if i < 3:
            atlas.cube_unorder_batched(got[i], r, B, grid, cube)
        else:
            atlas.aligned_global_unorder(got[i], r, grid, cube, gg, batch=B)
        got[i] = r
    torch.cuda.synchronize()
    o = orc()
    for b in range(B):
        sd, sg = slice(b * N, (b + 1) * N), slice(b * G, (b + 1) * G)
        cu = lambda s: o.cube_reorder(f64(t[s][sd]), grid, cube)
        ref = o.attention_bwd_full_aligned(
            cu("q_d"), cu("k_d"), cu("v_d"), grid, cube, f64(t["q_g"][sg]), f64(t["k_g"][sg]),
            f64(t["v_g"][sg]), gg, cu("do_d"), f64(t["do_g"][sg]), hd ** -0.5, n_threads())
        ref = [o.cube_unorder(r, grid, cube) if i < 3 else r for i, r in enumerate(ref)]
        part = [f64(g[sd if i < 3 else sg]) for i, g in enumerate(got)]
        assert_grads_close(part, ref, dtype, f"aligned order problem {b}")


def test_backward_dv_of_constant_do():
    """dO = 1 on every row: dV_j = sum_i P_ij, so the detail and global dV
    columns sum, over all keys, to the number of query rows (each row's P
    sums to 1); a property that holds at any size."""
    N, L, G, heads, hd = 4608, 768, 1000, 2, 128
    t = inputs(1, N, G, heads, hd, "bf16", seed=24)
    t["do_d"].fill_(1.0)
    t["do_g"].fill_(1.0)
    got = run_gpu(t, 1, heads, N, G, window_len=L)
    total = got[2][:, :, 0].float().sum(0) + got[5][:, :, 0].float().sum(0)
    assert torch.allclose(total, torch.full_like(total, N + G), rtol=1e-2)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_chain_backward_raster(dtype):
    """The whole path's gradient w.r.t. its raster inputs: forward reorder +
    RoPE -> attention -> unorder; backward reorder of dO -> attention
    backward -> unorder with the transposed RoPE (negated scales) for dQ and
    dK, plain unorder for dV, transposed RoPE for the global dQ and dK."""
    grid, cube, gg, heads = (4, 8, 8), (2, 4, 4), (2, 4, 4), 2
    hd = 64 if dtype == "fp32" else 128
    split = (16, 24, 24) if hd == 64 else (44, 42, 42)
    N, G, L = 256, 32, 32
    rd = atlas.make_rope(10000.0, split, (1.0, 1.0, 1.0))
    rg = atlas.make_rope(10000.0, split, (2.0, 2.0, 2.0))
    x = inputs(1, N, G, heads, hd, dtype, seed=25)
    y = {s: torch.empty_like(x[s]) for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "do_d")}
    for s in ("q_d", "k_d"):
        atlas.cube_reorder(x[s], y[s], grid, cube, rd)
    atlas.cube_reorder(x["v_d"], y["v_d"], grid, cube)
    for s in ("q_g", "k_g"):
        atlas.rope3d(x[s], y[s], gg, rg)
    o_d, o_g = torch.empty_like(y["q_d"]), torch.empty_like(y["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(y["q_d"], y["k_d"], y["v_d"], y["q_g"], y["k_g"], x["v_g"], o_d,
                               o_g, lse, window_len=L)
    # backward: dO arrives in raster order
    atlas.cube_reorder(x["do_d"], y["do_d"], grid, cube)
    g = [torch.empty_like(y[s]) for s in ("q_d", "k_d", "v_d", "q_g", "k_g")] + \
        [torch.empty_like(x["v_g"])]
    atlas.local_global_attn_bwd(y["q_d"], y["k_d"], y["v_d"], o_d, y["do_d"], y["q_g"], y["k_g"],
                                x["v_g"], o_g, x["do_g"], lse, *g, window_len=L)
    r = [torch.empty_like(t) for t in g]
    atlas.cube_unorder_rope(g[0], r[0], grid, cube, atlas.transpose_rope(rd))
    atlas.cube_unorder_rope(g[1], r[1], grid, cube, atlas.transpose_rope(rd))
    atlas.cube_unorder(g[2], r[2], grid, cube)
    atlas.rope3d(g[3], r[3], gg, atlas.transpose_rope(rg))
    atlas.rope3d(g[4], r[4], gg, atlas.transpose_rope(rg))
    r[5] = g[5]
    torch.cuda.synchronize()
    check_no_device_error()
    o = orc()
    rope = lambda t, grd, sc: o.rope3d_grid(t, grd, 10000.0, split, sc)
    qd = o.cube_reorder(rope(f64(x["q_d"]), grid, (1, 1, 1)), grid, cube)
    kd = o.cube_reorder(rope(f64(x["k_d"]), grid, (1, 1, 1)), grid, cube)
    vd = o.cube_reorder(f64(x["v_d"]), grid, cube)
    qg, kg = rope(f64(x["q_g"]), gg, (2, 2, 2)), rope(f64(x["k_g"]), gg, (2, 2, 2))
    ref = o.attention_bwd_full(qd, kd, vd, L, qg, kg, f64(x["v_g"]),
                               o.cube_reorder(f64(x["do_d"]), grid, cube), f64(x["do_g"]),
                               hd ** -0.5, n_threads())
    ref = [rope(o.cube_unorder(ref[0], grid, cube), grid, (-1, -1, -1)),
           rope(o.cube_unorder(ref[1], grid, cube), grid, (-1, -1, -1)),
           o.cube_unorder(ref[2], grid, cube),
           rope(ref[3], gg, (-2, -2, -2)), rope(ref[4], gg, (-2, -2, -2)), ref[5]]
    assert_grads_close([f64(t) for t in r], ref, dtype, "chain")


def test_backward_full_size_sampled():
    """720p workload at full size (80,640 detail and 5,040 global tokens, 40
    heads), the configuration bench.py --backward times: dQ of sampled query
    rows and dK, dV of sampled key rows (detail keys of two windows, global
    keys, whose gradients sum over every query) on the first and last head
    against the oracle."""
    from video_dit_windowed_b200.workloads import WORKLOADS
    w = WORKLOADS["720p"]
    torch.cuda.empty_cache()
    N, L, G, heads, hd = w.n_detail, w.window_len, w.n_global, w.heads, w.head_dim
    t = inputs(1, N, G, heads, hd, "bf16", seed=26)
    got = run_gpu(t, 1, heads, N, G, window_len=L)
    q_rows = np.concatenate([np.arange(0, 128), 57 * L + np.arange(300, 428), [N - 1],
                             N + np.array([0, 1, 2500, G - 1])])
    k_rows = np.concatenate([np.arange(0, 32), 104 * L + np.arange(700, 768),
                             N + np.array([0, 77, 2500, G - 2, G - 1])])
    for head in (0, heads - 1):
        cat = lambda a, b: np.concatenate([f64(a[:, head]), f64(b[:, head])])
        dq, dk, dv = orc().attention_bwd_sampled(
            cat(t["q_d"], t["q_g"]), cat(t["k_d"], t["k_g"]), cat(t["v_d"], t["v_g"]),
            cat(t["do_d"], t["do_g"]), N, L, hd ** -0.5, q_rows, k_rows, n_threads())
        g_q = cat(got[0], got[3])[q_rows]
        g_k = cat(got[1], got[4])[k_rows]
        g_v = cat(got[2], got[5])[k_rows]
        assert_grads_close([g_q, g_k, g_v], [dq, dk, dv], "bf16", f"720p head {head}")
    del got, t
    torch.cuda.empty_cache()


# Window offsets for both unit forms of the backward (as the forward's
# parity cases): unequal long windows with empty slots and a one-row window,
# and one long window among many short ones (packed tiles).
BWD_OFFSETS = [
    [0, 700, 1212, 1213, 1313, 2081, 2336, 2592],
    [0, 1000] + list(range(1001, 1501)),
]


@pytest.mark.parametrize("offsets", BWD_OFFSETS)
def test_backward_window_forms(offsets):
    N, G, heads, hd = offsets[-1], 150, 2, 128
    off = torch.tensor(offsets, dtype=torch.int32)
    t = inputs(1, N, G, heads, hd, "bf16", seed=25)
    got = run_gpu(t, 1, heads, N, G, window_offsets=off.to(DEV))
    ref = orc().attention_bwd_full(f64(t["q_d"]), f64(t["k_d"]), f64(t["v_d"]), 1,
                                   f64(t["q_g"]), f64(t["k_g"]), f64(t["v_g"]), f64(t["do_d"]),
                                   f64(t["do_g"]), hd ** -0.5, n_threads(),
                                   win_off=np.asarray(offsets, dtype=np.int64))
    assert_grads_close([f64(g) for g in got], ref, "bf16", f"offsets {offsets[:4]}")


def test_gradients_only_16_byte_aligned():
    """Gradient outputs that start 16 bytes into a buffer (the C-ABI's
    minimum alignment) take the 16-byte store path: same bits as aligned
    outputs."""
    N, L, G, heads, hd = 1536, 768, 300, 2, 128
    t = inputs(1, N, G, heads, hd, "bf16", seed=24)
    ref = run_gpu(t, 1, heads, N, G, window_len=L)
    o_d, o_g = torch.empty_like(t["q_d"]), torch.empty_like(t["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    atlas.local_global_attn_ex(t["q_d"], t["k_d"], t["v_d"], t["q_g"], t["k_g"], t["v_g"], o_d,
                               o_g, lse, window_len=L)
    grads = []
    for name in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g"):
        buf = torch.zeros(t[name].numel() + 8, dtype=torch.bfloat16, device=DEV)
        g = buf[8:].view(t[name].shape)
        assert g.data_ptr() % 32 == 16
        grads.append(g)
    atlas.local_global_attn_bwd(t["q_d"], t["k_d"], t["v_d"], o_d, t["do_d"], t["q_g"],
                                t["k_g"], t["v_g"], o_g, t["do_g"], lse, *grads, window_len=L)
    torch.cuda.synchronize()
    check_no_device_error()
    for a, b in zip(grads, ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
