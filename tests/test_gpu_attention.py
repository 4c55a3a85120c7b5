"""GPU parity of the asymmetric local-global attention (steps 3 and 4) and of
the whole chain against the fp64 oracle, through the C-ABI.

Passages: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie 1
Fase 2 (window attention on the reordered sequence) and Methodologie 2
(asymmetric hierarchical attention: detail rows see their own cube and every
global token; global rows see only global tokens).

Bounds (tests/helpers.py): bf16 max-abs 2e-2, mean-abs 2e-3, LSE 5e-3 against
the fp64 oracle; structural checks (exact zeros outside the allowed set,
V = 1 rows) on every row.
"""
import math

import numpy as np
import pytest
import torch

from helpers import (assert_attn_close, assert_lse_close, attention_gpu, check_no_device_error,
                     f64, n_threads, orc, oracle_attention_rows)
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import WORKLOADS, make_inputs, normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def tdt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def inputs(N, G, heads, hd, dtype, seed=0):
    mk = lambda n, s: normal((n, heads, hd), s, tdt(dtype), seed=seed, device=DEV)
    return mk(N, "q_d"), mk(N, "k_d"), mk(N, "v_d"), mk(G, "q_g"), mk(G, "k_g"), mk(G, "v_g")


def full_oracle(q_d, k_d, v_d, L, q_g, k_g, v_g, scale):
    return orc().attention_full(f64(q_d), f64(k_d), f64(v_d), L, f64(q_g), f64(k_g),
                                f64(v_g), scale, n_threads())


# N (detail rows, cube order), L (window), G, heads, head_dim, dtype
SMALL = [
    (256, 32, 32, 2, 64, "bf16"),       # tiny workload's shape, bf16
    (256, 32, 32, 2, 64, "fp32"),       # tiny workload as given (fp32)
    (1536, 768, 1, 2, 128, "bf16"),     # G = 1
    (1536, 768, 127, 1, 128, "bf16"),   # G one short of a tile
    (1536, 768, 128, 1, 128, "bf16"),   # G exactly one tile
    (1536, 768, 129, 1, 128, "bf16"),   # G one past a tile
    (1024, 128, 200, 3, 128, "bf16"),   # windows of exactly one tile
    (960, 48, 77, 2, 128, "bf16"),      # windows not aligned to tiles
    (512, 1, 64, 2, 128, "bf16"),       # 1x1x1 cubes: each row sees itself and the globals
    (2048, 512, 300, 2, 64, "bf16"),    # head_dim 64
    (3072, 1536, 500, 1, 128, "bf16"),  # long windows
    (1920, 384, 65, 2, 128, "bf16"),    # 1.5 units per window: a half-empty second unit
    (2560, 640, 33, 2, 128, "bf16"),    # 2.5 units per window; a 64-key global tile
    (1280, 640, 20, 1, 64, "bf16"),     # a 32-key global tile at head_dim 64
    (768, 768, 0, 2, 128, "bf16"),      # no global tokens (pure window attention)
    (0, 1, 1000, 2, 128, "bf16"),       # global tokens only
    (600, 100, 50, 2, 128, "fp32"),
    (0, 1, 70, 3, 64, "fp32"),
]


@pytest.mark.parametrize("N,L,G,heads,hd,dtype", SMALL)
def test_attention_matches_oracle(N, L, G, heads, hd, dtype):
    q_d, k_d, v_d, q_g, k_g, v_g = inputs(N, G, heads, hd, dtype)
    o_d, o_g, lse = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g)
    torch.cuda.synchronize()
    check_no_device_error()
    ref_d, ref_g, ref_lse = full_oracle(q_d, k_d, v_d, L, q_g, k_g, v_g, 1 / math.sqrt(hd))
    got = np.concatenate([f64(o_d), f64(o_g)])
    ref = np.concatenate([ref_d, ref_g])
    assert_attn_close(got, ref, dtype, f"N={N} L={L} G={G}")
    assert_lse_close(f64(lse), ref_lse, dtype)


def test_softmax_scale_argument():
    N, L, G, heads, hd = 512, 256, 64, 2, 128
    q_d, k_d, v_d, q_g, k_g, v_g = inputs(N, G, heads, hd, "bf16", seed=1)
    o_d, o_g = torch.empty_like(q_d), torch.empty_like(q_g)
    atlas.local_global_attn(q_d, k_d, v_d, L, q_g, k_g, v_g, o_d, o_g, None, softmax_scale=0.05)
    torch.cuda.synchronize()
    ref_d, ref_g, _ = full_oracle(q_d, k_d, v_d, L, q_g, k_g, v_g, 0.05)
    assert_attn_close(np.concatenate([f64(o_d), f64(o_g)]), np.concatenate([ref_d, ref_g]),
                      "bf16")


@pytest.mark.parametrize("N,L,G,hd", [(2304, 768, 300, 128), (960, 48, 130, 64),
                                      (256, 32, 32, 64), (4096, 128, 0, 128)])
def test_mask_probe_exact_zeros(N, L, G, hd):
    """V = indicators: column 3 + (window id mod m) is 1 on that window's
    keys, column 2 is 1 on global keys. A detail row may only put mass on its
    own window's column and column 2; every other class column must be
    exactly 0. A global row must have exactly 0 in every class column."""
    heads = 2
    q_d, k_d, _, q_g, k_g, _ = inputs(N, G, heads, hd, "bf16", seed=2)
    rows = torch.arange(N, device=DEV)
    for modulus in (61, 59):
        cls = (rows // L) % modulus
        v_d = torch.zeros(N, heads, hd, dtype=torch.bfloat16, device=DEV)
        v_g = torch.zeros(G, heads, hd, dtype=torch.bfloat16, device=DEV)
        v_d[rows, :, 3 + cls] = 1.0
        v_g[:, :, 2] = 1.0
        o_d, o_g, _ = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g, with_lse=False)
        torch.cuda.synchronize()
        check_no_device_error()
        od = o_d.float()[:, :, 3:3 + modulus].clone()
        own = od[rows, :, cls].clone()
        od[rows, :, cls] = 0.0
        assert torch.all(od == 0), f"mass outside the own window (mod {modulus})"
        assert torch.all(own > 0)
        if G:
            assert torch.all(o_d.float()[:, :, 2] > 0)
            assert torch.all(o_g.float()[:, :, 3:3 + modulus] == 0)
            assert float((o_g.float()[:, :, 2] - 1).abs().max()) <= 8e-3
        else:
            assert torch.all(o_d.float()[:, :, 2] == 0)


@pytest.mark.parametrize("N,L,G", [(1536, 768, 129), (960, 48, 77), (0, 1, 300)])
def test_constant_v_rows_sum_to_one(N, L, G):
    heads, hd = 2, 128
    q_d, k_d, _, q_g, k_g, _ = inputs(N, G, heads, hd, "bf16", seed=3)
    v_d = torch.ones(N, heads, hd, dtype=torch.bfloat16, device=DEV)
    v_g = torch.ones(G, heads, hd, dtype=torch.bfloat16, device=DEV)
    o_d, o_g, _ = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g, with_lse=False)
    torch.cuda.synchronize()
    o = torch.cat([o_d.float().flatten(), o_g.float().flatten()])
    assert float((o - 1).abs().max()) <= 8e-3


def test_outputs_untouched_beyond_rows():
    """Rows past the end of a ragged last tile are never written."""
    N, L, G, heads, hd = 384, 128, 130, 1, 128
    q_d, k_d, v_d, q_g, k_g, v_g = inputs(N, G, heads, hd, "bf16", seed=4)
    store_d = torch.full((N + 256, heads, hd), 7.0, dtype=torch.bfloat16, device=DEV)
    store_g = torch.full((G + 256, heads, hd), 7.0, dtype=torch.bfloat16, device=DEV)
    o_d, o_g = store_d[:N], store_g[:G]
    atlas.local_global_attn(q_d, k_d, v_d, L, q_g, k_g, v_g, o_d, o_g, None)
    torch.cuda.synchronize()
    assert torch.all(store_d[N:] == 7.0) and torch.all(store_g[G:] == 7.0)


def test_whole_chain_tiny():
    """reorder+RoPE -> attention -> unorder on the tiny workload (fp32 and a
    bf16 copy) against the oracle's chain in raster order."""
    w = WORKLOADS["tiny"]
    for dtype in ("fp32", "bf16"):
        x = {k: v.to(DEV).to(tdt(dtype)) for k, v in make_inputs(w, device="cpu").items()}
        ro_d = atlas.make_rope(w.theta, w.split, w.detail_scales)
        ro_g = atlas.make_rope(w.theta, w.split, w.global_scales)
        q_d, k_d, v_d = (torch.empty_like(x[k]) for k in ("q_d", "k_d", "v_d"))
        atlas.cube_reorder(x["q_d"], q_d, w.grid, w.cube, ro_d)
        atlas.cube_reorder(x["k_d"], k_d, w.grid, w.cube, ro_d)
        atlas.cube_reorder(x["v_d"], v_d, w.grid, w.cube)
        q_g, k_g = torch.empty_like(x["q_g"]), torch.empty_like(x["k_g"])
        atlas.rope3d(x["q_g"], q_g, w.global_grid, ro_g)
        atlas.rope3d(x["k_g"], k_g, w.global_grid, ro_g)
        o_d, o_g, _ = attention_gpu(q_d, k_d, v_d, w.window_len, q_g, k_g, x["v_g"])
        o_raster = torch.empty_like(o_d)
        atlas.cube_unorder(o_d, o_raster, w.grid, w.cube)
        torch.cuda.synchronize()
        check_no_device_error()
        # oracle chain, fp64 throughout
        o = orc()
        rq = o.cube_reorder(o.rope3d_grid(f64(x["q_d"]), w.grid, w.theta, w.split,
                                          w.detail_scales), w.grid, w.cube)
        rk = o.cube_reorder(o.rope3d_grid(f64(x["k_d"]), w.grid, w.theta, w.split,
                                          w.detail_scales), w.grid, w.cube)
        rv = o.cube_reorder(f64(x["v_d"]), w.grid, w.cube)
        gq = o.rope3d_grid(f64(x["q_g"]), w.global_grid, w.theta, w.split, w.global_scales)
        gk = o.rope3d_grid(f64(x["k_g"]), w.global_grid, w.theta, w.split, w.global_scales)
        ref_d, ref_g, _ = o.attention_full(rq, rk, rv, w.window_len, gq, gk, f64(x["v_g"]),
                                           w.softmax_scale)
        ref_raster = o.cube_unorder(ref_d, w.grid, w.cube)
        assert_attn_close(np.concatenate([f64(o_raster), f64(o_g)]),
                          np.concatenate([ref_raster, ref_g]), dtype, f"chain {dtype}")


@pytest.mark.parametrize("name", ["720p", "global_only", "4k", "4k_long"])
def test_full_size_sampled_rows(name):
    """Full-size workloads, in the configuration the benchmark times: sampled
    rows (first, last and one random window; first, last-tile and random
    global rows) on the first and last head against the oracle, plus V = 1
    and mask-probe properties on every row."""
    w = WORKLOADS[name]
    torch.cuda.empty_cache()
    N, L, G, heads = w.n_detail, w.window_len, w.n_global, w.heads
    q_d, k_d, v_d, q_g, k_g, v_g = inputs(N, G, heads, w.head_dim, "bf16")
    o_d, o_g, lse = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g)
    torch.cuda.synchronize()
    check_no_device_error()
    rng = np.random.default_rng(0)
    nwin = N // L if N else 0
    wins = sorted({0, nwin - 1, int(rng.integers(0, max(nwin, 1)))}) if N else []
    det_rows = np.concatenate([np.arange(wi * L, (wi + 1) * L) for wi in wins]) if N else []
    g_rows = np.unique(np.concatenate([np.arange(min(128, G)), np.arange(max(0, G - 128), G),
                                       rng.integers(0, G, 128)]))
    for head in (0, heads - 1):
        outs, lses = oracle_attention_rows(q_d, k_d, v_d, L, q_g, k_g, v_g, head, det_rows,
                                           g_rows, w.softmax_scale)
        got, got_l = [], []
        if N:
            idx = torch.as_tensor(det_rows, device=DEV)
            got.append(f64(o_d[idx, head]))
            got_l.append(f64(lse[head, idx]))
        idx = torch.as_tensor(g_rows, device=DEV)
        got.append(f64(o_g[idx, head]))
        got_l.append(f64(lse[head, N + idx]))
        assert_attn_close(np.concatenate(got), np.concatenate(outs), "bf16", f"{name} h{head}")
        assert_lse_close(np.concatenate(got_l), np.concatenate(lses), "bf16", f"{name} h{head}")
    # every row: V = 1 gives 1
    del o_d, o_g, lse
    v_d.fill_(1.0)
    v_g.fill_(1.0)
    o_d, o_g, _ = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g, with_lse=False)
    torch.cuda.synchronize()
    for t in (o_d, o_g):
        if t.numel():
            assert float((t.float() - 1).abs().max()) <= 8e-3
    del q_d, k_d, v_d, q_g, k_g, v_g, o_d, o_g
    torch.cuda.empty_cache()


def test_head_shards_equal_the_full_call():
    """Head-parallel sharding: heads are independent end to end, so the
    reorder+RoPE and the attention of a slice of the heads (as one rank of a
    head-parallel run holds them) give the full call's bits for those heads."""
    grid, cube, gg, heads, hd = (6, 16, 16), (3, 8, 8), (6, 4, 4), 4, 128
    N, G, L = 1536, 96, 192
    rope = atlas.make_rope(10000.0, (44, 42, 42), (1.0, 1.0, 1.0))
    x = {s: normal((N if s.endswith("_d") else G, heads, hd), s, torch.bfloat16, seed=41,
                   device="cuda") for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}

    def run(t, nh):
        q, k = torch.empty_like(t["q_d"]), torch.empty_like(t["k_d"])
        atlas.cube_reorder(t["q_d"], q, grid, cube, rope)
        atlas.cube_reorder(t["k_d"], k, grid, cube, rope)
        o_d, o_g = torch.empty_like(q), torch.empty_like(t["q_g"])
        lse = torch.empty(nh, N + G, dtype=torch.float32, device="cuda")
        atlas.local_global_attn(q, k, t["v_d"], L, t["q_g"], t["k_g"], t["v_g"], o_d, o_g, lse)
        return q, o_d, o_g, lse

    full = run(x, heads)
    for h0, h1 in ((0, 2), (2, 4), (1, 2)):
        part = run({s: v[:, h0:h1].contiguous() for s, v in x.items()}, h1 - h0)
        torch.cuda.synchronize()
        check_no_device_error()
        for a, b in zip(full[:3], part[:3]):
            assert torch.equal(a[:, h0:h1].contiguous().view(torch.int16), b.view(torch.int16))
        assert torch.equal(full[3][h0:h1], part[3])


def test_outputs_only_16_byte_aligned():
    """The C-ABI promises outputs 16-byte alignment only; with both outputs
    32-byte aligned the epilogue stores 32 bytes at a time, otherwise 16.
    Outputs that start 16 bytes into a buffer take the 16-byte path and
    must give the same bits."""
    N, L, G, heads, hd = 1536, 768, 300, 2, 128
    q_d, k_d, v_d, q_g, k_g, v_g = inputs(N, G, heads, hd, "bf16", seed=6)
    ref_d, ref_g, ref_l = attention_gpu(q_d, k_d, v_d, L, q_g, k_g, v_g)
    buf_d = torch.zeros(N * heads * hd + 8, dtype=torch.bfloat16, device=DEV)
    buf_g = torch.zeros(G * heads * hd + 8, dtype=torch.bfloat16, device=DEV)
    o_d = buf_d[8:].view(N, heads, hd)          # 16 bytes past a 512-byte boundary
    o_g = buf_g[8:].view(G, heads, hd)
    assert o_d.data_ptr() % 32 == 16 and o_g.data_ptr() % 32 == 16
    lse = torch.empty_like(ref_l)
    atlas.local_global_attn(q_d, k_d, v_d, L, q_g, k_g, v_g, o_d, o_g, lse)
    torch.cuda.synchronize()
    check_no_device_error()
    assert torch.equal(o_d.view(torch.int16), ref_d.view(torch.int16))
    assert torch.equal(o_g.view(torch.int16), ref_g.view(torch.int16))
    assert torch.equal(lse, ref_l)
