"""Host-side checks of the C-ABI library (no GPU needed).

The library must build, load, export exactly the symbols ``include/atlas.h``
declares, and reject bad arguments on the host before any CUDA call. Fake
pointer values are never dereferenced: every case below fails validation
first.
"""
import ctypes
import os
import re
import subprocess

import pytest

from video_dit_windowed_b200 import atlas, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "atlas.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return atlas.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(atlas_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for want in ("atlas_cube_reorder", "atlas_cube_unorder", "atlas_rope3d",
                 "atlas_local_global_attn", "atlas_status_string"):
        assert want in names


def test_exports_match_header(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", atlas.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = sorted({l.split()[-1] for l in out.splitlines()
                       if l.split()[-2:-1] == ["T"] and l.split()[-1].startswith("atlas_")})
    assert exported == declared_functions()


def test_status_strings(lib):
    for code in range(9):
        s = atlas.status_string(code)
        assert s.startswith("ATLAS_")
    assert "UNKNOWN" in atlas.status_string(99)
    assert atlas.version() >= 100


FAKE = 0x7F0000000000  # 16-byte aligned, never dereferenced
G = atlas.Grid3(4, 8, 8)
C = atlas.Cube3(2, 4, 4)


def reorder(lib, src, dst, grid=G, cube=C, heads=2, hd=64, dt=atlas.FP32, rope=None):
    return lib.atlas_cube_reorder(src, dst, grid, cube, heads, hd, dt,
                                  ctypes.byref(rope) if rope else None, None)


def test_reorder_validation(lib):
    big = FAKE + (1 << 30)
    assert reorder(lib, None, big) == atlas.ERR_NULL
    assert reorder(lib, FAKE, None) == atlas.ERR_NULL
    assert reorder(lib, FAKE, big, cube=atlas.Cube3(0, 4, 4)) == atlas.ERR_SHAPE
    assert reorder(lib, FAKE, big, grid=atlas.Grid3(0, 8, 8)) == atlas.ERR_SHAPE
    assert reorder(lib, FAKE + 8, big) == atlas.ERR_ALIGN
    assert reorder(lib, FAKE, big, hd=6, dt=atlas.BF16) == atlas.ERR_ALIGN
    assert reorder(lib, FAKE, FAKE + 64) == atlas.ERR_ALIAS
    assert reorder(lib, FAKE, FAKE) == atlas.ERR_ALIAS
    assert reorder(lib, FAKE, big, dt=7) == atlas.ERR_UNSUPPORTED
    bad_split = atlas.make_rope(10000, (16, 24, 22), (1, 1, 1))
    assert reorder(lib, FAKE, big, rope=bad_split) == atlas.ERR_UNSUPPORTED
    odd_split = atlas.make_rope(10000, (15, 25, 24), (1, 1, 1))
    assert reorder(lib, FAKE, big, rope=odd_split) == atlas.ERR_UNSUPPORTED
    bad_theta = atlas.make_rope(0.0, (16, 24, 24), (1, 1, 1))
    assert reorder(lib, FAKE, big, rope=bad_theta) == atlas.ERR_UNSUPPORTED
    huge = atlas.Grid3(1 << 16, 1 << 16, 1)
    assert reorder(lib, FAKE, big, grid=huge, cube=atlas.Cube3(1, 1, 1)) == atlas.ERR_SHAPE


def test_unorder_and_rope_validation(lib):
    big = FAKE + (1 << 30)
    assert lib.atlas_cube_unorder(None, big, G, C, 2, 64, atlas.FP32, None) == atlas.ERR_NULL
    assert lib.atlas_cube_unorder(FAKE, big, G, atlas.Cube3(2, 0, 4), 2, 64, atlas.FP32,
                                  None) == atlas.ERR_SHAPE
    assert lib.atlas_cube_unorder(FAKE, FAKE + 16, G, C, 2, 64, atlas.FP32,
                                  None) == atlas.ERR_ALIAS
    rope = atlas.make_rope(10000, (16, 24, 24), (1, 1, 1))
    assert lib.atlas_rope3d(FAKE, big, G, 2, 64, atlas.FP32, None, None) == atlas.ERR_NULL
    assert lib.atlas_rope3d(FAKE, FAKE + 16, G, 2, 64, atlas.FP32, ctypes.byref(rope),
                            None) == atlas.ERR_ALIAS
    assert lib.atlas_rope3d(FAKE + 4, FAKE + 4, G, 2, 64, atlas.FP32, ctypes.byref(rope),
                            None) == atlas.ERR_ALIGN


def attn(lib, q_d=FAKE, k_d=FAKE + (1 << 28), v_d=FAKE + (2 << 28), n_d=256, L=32,
         q_g=FAKE + (3 << 28), k_g=FAKE + (4 << 28), v_g=FAKE + (5 << 28), n_g=32, heads=2,
         hd=64, dt=atlas.BF16, o_d=FAKE + (6 << 28), o_g=FAKE + (7 << 28), lse=None):
    return lib.atlas_local_global_attn(q_d, k_d, v_d, n_d, L, q_g, k_g, v_g, n_g, heads, hd,
                                       0.0, dt, o_d, o_g, lse, None)


def test_attention_validation(lib):
    assert attn(lib, q_d=None) == atlas.ERR_NULL
    assert attn(lib, o_g=None) == atlas.ERR_NULL
    assert attn(lib, n_d=250) == atlas.ERR_SHAPE          # not a multiple of L
    assert attn(lib, L=0) == atlas.ERR_SHAPE
    assert attn(lib, n_d=-1) == atlas.ERR_SHAPE
    assert attn(lib, heads=0) == atlas.ERR_SHAPE
    assert attn(lib, hd=96) == atlas.ERR_UNSUPPORTED
    assert attn(lib, dt=5) == atlas.ERR_UNSUPPORTED
    assert attn(lib, k_g=FAKE + (4 << 28) + 8) == atlas.ERR_ALIGN
    assert attn(lib, lse=FAKE + 2) == atlas.ERR_ALIGN
    assert attn(lib, o_d=FAKE + (1 << 28)) == atlas.ERR_ALIAS   # o_d over k_d
    assert attn(lib, o_g=FAKE + (6 << 28)) == atlas.ERR_ALIAS   # o_g over o_d
    # Absent sides: their pointers are not required.
    assert attn(lib, n_d=0, q_d=None, k_d=None, v_d=None, o_d=None, n_g=0,
                q_g=None, k_g=None, v_g=None, o_g=None) == atlas.OK


def test_valid_call_without_gpu_reports_device(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert attn(lib) == atlas.ERR_DEVICE
    big = FAKE + (1 << 30)
    assert reorder(lib, FAKE, big) == atlas.ERR_DEVICE


def test_cube_window_offsets_host(lib):
    import numpy as np
    import oracle
    orc = oracle.Oracle()
    for grid, cube in (((5, 7, 9), (2, 3, 4)), ((4, 8, 8), (2, 4, 4)), ((21, 48, 80), (3, 16, 16))):
        got = atlas.cube_window_offsets(grid, cube).numpy()
        assert np.array_equal(got, orc.cube_windows(grid, cube))
    n = ctypes.c_int64(0)
    small = (ctypes.c_int32 * 3)()
    assert lib.atlas_cube_window_offsets(atlas.Grid3(5, 7, 9), atlas.Cube3(2, 3, 4), small, 3,
                                         ctypes.byref(n)) == atlas.ERR_CAPACITY
    assert lib.atlas_cube_window_offsets(atlas.Grid3(5, 7, 9), atlas.Cube3(0, 3, 4), None, 0,
                                         ctypes.byref(n)) == atlas.ERR_SHAPE
    assert lib.atlas_cube_window_offsets(atlas.Grid3(5, 7, 9), atlas.Cube3(2, 3, 4), None, 0,
                                         None) == atlas.ERR_NULL


def test_windows_attention_validation(lib):
    base = dict(q_d=FAKE, k_d=FAKE + (1 << 28), v_d=FAKE + (2 << 28), q_g=FAKE + (3 << 28),
                k_g=FAKE + (4 << 28), v_g=FAKE + (5 << 28), o_d=FAKE + (6 << 28),
                o_g=FAKE + (7 << 28))
    def call(off=FAKE + (8 << 28), n_win=8, n_d=256, **kw):
        a = dict(base, **kw)
        return lib.atlas_local_global_attn_windows(a["q_d"], a["k_d"], a["v_d"], n_d, off, n_win,
                                                   a["q_g"], a["k_g"], a["v_g"], 32, 2, 64, 0.0,
                                                   atlas.BF16, a["o_d"], a["o_g"], None, None)
    assert call(off=None) == atlas.ERR_NULL
    assert call(n_win=0) == atlas.ERR_SHAPE
    assert call(n_win=300) == atlas.ERR_SHAPE
    assert call(off=FAKE + (8 << 28) + 2) == atlas.ERR_ALIGN


def test_attention_ex_validation(lib):
    base = [FAKE, FAKE + (1 << 28), FAKE + (2 << 28), 256, FAKE + (3 << 28), FAKE + (4 << 28),
            FAKE + (5 << 28), 32]
    outs = [FAKE + (6 << 28), FAKE + (7 << 28)]

    def call(ly, n_d=256, heads=2, lse=None):
        args = list(base)
        args[3] = n_d
        return lib.atlas_local_global_attn_ex(*args, ctypes.byref(ly) if ly else None, heads, 64,
                                              0.0, atlas.BF16, *outs, lse, None)
    L = atlas.AttnLayout
    assert call(None) == atlas.ERR_NULL
    assert call(L(0, 32, None, 0, None)) == atlas.ERR_SHAPE            # batch < 1
    assert call(L(1, 30, None, 0, None)) == atlas.ERR_SHAPE            # 256 % 30
    assert call(L(1, 32, None, 7, FAKE + (8 << 28))) == atlas.ERR_SHAPE  # 8 windows, not 7
    assert call(L(1, 32, None, 8, FAKE + (8 << 28) + 2)) == atlas.ERR_ALIGN
    assert call(L(1, 0, FAKE + (8 << 28), 0, None)) == atlas.ERR_SHAPE   # no windows
    assert call(L(1 << 30, 32, None, 0, None)) == atlas.ERR_SHAPE      # too many rows
    # batch 2: the tensors hold 512 detail rows; the outputs overlap k_d's second half
    assert lib.atlas_local_global_attn_ex(
        FAKE, FAKE + 256 * 256, FAKE + (2 << 28), 256, FAKE + (3 << 28), FAKE + (4 << 28),
        FAKE + (5 << 28), 32, ctypes.byref(L(2, 32, None, 0, None)), 1, 64, 0.0, atlas.BF16,
        FAKE + 384 * 256, FAKE + (7 << 28), None, None) == atlas.ERR_ALIAS
    import torch
    if not torch.cuda.is_available():
        assert call(L(2, 32, None, 8, FAKE + (8 << 28))) == atlas.ERR_DEVICE


def test_aligned_global_cube_host(lib):
    assert atlas.aligned_global_cube((21, 48, 80), (3, 16, 16), (21, 12, 20)) == (3, 4, 4)
    assert atlas.aligned_global_cube((42, 144, 240), (6, 16, 16), (21, 18, 30)) == (3, 2, 2)
    out = atlas.Cube3()
    G3, C3 = atlas.Grid3, atlas.Cube3
    assert lib.atlas_aligned_global_cube(G3(5, 7, 9), C3(2, 3, 4), G3(2, 3, 4),
                                         ctypes.byref(out)) == atlas.ERR_UNSUPPORTED
    assert lib.atlas_aligned_global_cube(G3(4, 8, 8), C3(2, 4, 3), G3(2, 4, 4),
                                         ctypes.byref(out)) == atlas.ERR_UNSUPPORTED
    assert lib.atlas_aligned_global_cube(G3(4, 8, 8), C3(2, 4, 4), G3(0, 4, 4),
                                         ctypes.byref(out)) == atlas.ERR_SHAPE
    assert lib.atlas_aligned_global_cube(G3(4, 8, 8), C3(2, 4, 4), G3(2, 4, 4),
                                         None) == atlas.ERR_NULL


def test_aligned_global_cube_matches_oracle(lib):
    """For integral ratios, cube c of the global grid cut into the returned
    cube holds exactly the global tokens the oracle's aligned predicate
    gives detail cube c (K = 0 makes the oracle's LSE a key count, and the
    probe below names the keys)."""
    import numpy as np
    import oracle
    orc = oracle.Oracle()
    for grid, cube, gg in (((4, 8, 8), (2, 4, 4), (2, 4, 4)), ((5, 12, 20), (2, 8, 8), (5, 3, 5)),
                           ((6, 16, 16), (3, 8, 8), (6, 4, 4))):
        gcube = atlas.aligned_global_cube(grid, cube, gg)
        goff = atlas.cube_window_offsets(gg, gcube).numpy()
        doff = atlas.cube_window_offsets(grid, cube).numpy()
        assert goff.size == doff.size
        gpos = orc.cube_positions(gg, gcube)   # raster -> global cube order
        G = gg[0] * gg[1] * gg[2]
        D = 8
        # V_g = one-hot of the raster index (first D rows only carry mass
        # visibility): use indicator of "global cube order position in window w"
        for w in range(doff.size - 1):
            lo, hi = int(doff[w]), int(doff[w + 1])
            vg = np.zeros((G, D))
            inside = (gpos >= goff[w]) & (gpos < goff[w + 1])
            vg[inside, 0] = 1.0
            vg[~inside, 1] = 1.0
            kd = np.zeros((hi - lo, D))
            o, _ = orc.attention_head_aligned(grid, cube, gg, 1.0, kd, kd, lo, np.zeros((G, D)),
                                              vg, np.arange(lo, hi), np.zeros((hi - lo, D)))
            assert np.all(o[:, 1] == 0.0), (grid, w)
            n_in = int(inside.sum())
            assert np.allclose(o[:, 0], n_in / (hi - lo + n_in)), (grid, w)


def test_attention_bwd_validation(lib):
    ins_d = [FAKE + (i << 27) for i in range(5)]          # q, k, v, o, do (detail)
    ins_g = [FAKE + ((8 + i) << 27) for i in range(5)]    # global
    grads = [FAKE + ((16 + i) << 27) for i in range(6)]
    lse, delta = FAKE + (24 << 27), FAKE + (25 << 27)
    L = atlas.AttnLayout

    def call(ly=L(1, 32, None, 0, None), i_d=None, i_g=None, g=None, lse_=lse, delta_=delta,
             hd=64):
        i_d = i_d or ins_d
        i_g = i_g or ins_g
        g = g or grads
        return lib.atlas_local_global_attn_bwd(*i_d, 256, *i_g, 32,
                                               ctypes.byref(ly) if ly else None, 2, hd, 0.0,
                                               atlas.BF16, lse_, delta_, *g, None)
    assert call(ly=None) == atlas.ERR_NULL
    assert call(lse_=None) == atlas.ERR_NULL
    assert call(delta_=None) == atlas.ERR_NULL
    assert call(delta_=delta + 2) == atlas.ERR_ALIGN
    assert call(hd=96) == atlas.ERR_UNSUPPORTED
    assert call(i_d=ins_d[:4] + [None]) == atlas.ERR_NULL             # dO_d missing
    assert call(g=grads[:5] + [None]) == atlas.ERR_NULL               # dv_g missing
    assert call(g=[grads[0] + 8] + grads[1:]) == atlas.ERR_ALIGN
    assert call(g=[ins_d[0]] + grads[1:]) == atlas.ERR_ALIAS          # dq_d over q_d
    assert call(g=grads[:2] + [grads[1]] + grads[3:]) == atlas.ERR_ALIAS   # dv_d over dk_d
    assert call(delta_=ins_g[4]) == atlas.ERR_ALIAS                   # delta over dO_g
    assert call(ly=L(1, 30, None, 0, None)) == atlas.ERR_SHAPE
    import torch
    if not torch.cuda.is_available():
        assert call() == atlas.ERR_DEVICE


def test_projection_validation(lib):
    G3, C3 = atlas.Grid3, atlas.Cube3
    x, w = FAKE, FAKE + (1 << 30)
    q, k, v = FAKE + (2 << 30), FAKE + (3 << 30), FAKE + (4 << 30)

    def qkv(x=x, w=w, batch=1, grid=G3(4, 8, 8), c_in=256, heads=2, hd=128, dt=atlas.BF16,
            q=q, k=k, v=v, rope=None):
        return lib.atlas_qkv_proj_reorder(x, w, batch, grid, C3(2, 4, 4), c_in, heads, hd, dt,
                                          ctypes.byref(rope) if rope else None, q, k, v, None)
    assert qkv(x=None) == atlas.ERR_NULL
    assert qkv(v=None) == atlas.ERR_NULL
    assert qkv(batch=0) == atlas.ERR_SHAPE
    assert qkv(dt=atlas.FP32) == atlas.ERR_UNSUPPORTED
    assert qkv(c_in=96) == atlas.ERR_UNSUPPORTED            # not a multiple of 64
    assert qkv(heads=3, hd=64) == atlas.ERR_UNSUPPORTED     # 192 not a multiple of 256
    assert qkv(q=q + 8) == atlas.ERR_ALIGN
    assert qkv(k=q + 64) == atlas.ERR_ALIAS                 # k over q
    assert qkv(q=x) == atlas.ERR_ALIAS                      # q over x
    assert qkv(rope=atlas.make_rope(10000, (44, 42, 40), (1, 1, 1))) == atlas.ERR_UNSUPPORTED

    def out(o=x, w=w, c_in=256, c_out=512, y=q, dt=atlas.BF16):
        return lib.atlas_out_proj_unorder(o, w, 1, G3(4, 8, 8), C3(2, 4, 4), c_in, c_out, dt, y,
                                          None)
    assert out(y=None) == atlas.ERR_NULL
    assert out(c_out=300) == atlas.ERR_UNSUPPORTED
    assert out(y=w) == atlas.ERR_ALIAS
    import torch
    if not torch.cuda.is_available():
        assert qkv() == atlas.ERR_DEVICE
        assert out() == atlas.ERR_DEVICE


def test_aligned_global_offsets_host(lib):
    """Window ranges of the aligned order: validation, and for ratios that
    are not integers the range of window w holds exactly the global tokens
    the oracle's aligned predicate gives detail cube w (probe as above, with
    the aligned order's positions from their definition)."""
    import numpy as np
    import oracle
    from helpers import aligned_positions
    G3, C3 = atlas.Grid3, atlas.Cube3
    n = ctypes.c_int64(0)
    assert lib.atlas_aligned_global_offsets(G3(4, 8, 8), C3(2, 4, 4), G3(2, 4, 4), None, 0,
                                            None) == atlas.ERR_NULL
    assert lib.atlas_aligned_global_offsets(G3(4, 8, 8), C3(2, 4, 4), G3(2, 0, 4), None, 0,
                                            ctypes.byref(n)) == atlas.ERR_SHAPE
    assert lib.atlas_aligned_global_offsets(G3(4, 8, 8), C3(0, 4, 4), G3(2, 4, 4), None, 0,
                                            ctypes.byref(n)) == atlas.ERR_SHAPE
    assert lib.atlas_aligned_global_offsets(G3(4, 8, 8), C3(2, 4, 4), G3(2, 4, 4), None, 0,
                                            ctypes.byref(n)) == atlas.OK
    assert n.value == 8
    buf = (ctypes.c_int32 * 8)()
    assert lib.atlas_aligned_global_offsets(G3(4, 8, 8), C3(2, 4, 4), G3(2, 4, 4), buf, 8,
                                            ctypes.byref(n)) == atlas.ERR_CAPACITY
    orc = oracle.Oracle()
    for grid, cube, gg in (((5, 7, 9), (2, 3, 4), (2, 3, 4)), ((6, 20, 30), (3, 8, 8), (4, 6, 7)),
                           ((4, 8, 8), (2, 4, 4), (3, 10, 5))):
        goff = atlas.aligned_global_offsets(grid, cube, gg).numpy()
        doff = atlas.cube_window_offsets(grid, cube).numpy()
        G = gg[0] * gg[1] * gg[2]
        assert goff.size == doff.size and goff[0] == 0 and goff[-1] == G
        assert np.all(np.diff(goff) >= 0)
        pos = aligned_positions(grid, cube, gg)
        assert sorted(pos.tolist()) == list(range(G))
        D = 8
        for w in range(doff.size - 1):
            lo, hi = int(doff[w]), int(doff[w + 1])
            vg = np.zeros((G, D))
            inside = (pos >= goff[w]) & (pos < goff[w + 1])
            vg[inside, 0] = 1.0
            vg[~inside, 1] = 1.0
            kd = np.zeros((hi - lo, D))
            o, _ = orc.attention_head_aligned(grid, cube, gg, 1.0, kd, kd, lo, np.zeros((G, D)),
                                              vg, np.arange(lo, hi), np.zeros((hi - lo, D)))
            assert np.all(o[:, 1] == 0.0), (grid, w)
            n_in = int(inside.sum())
            assert np.allclose(o[:, 0], n_in / (hi - lo + n_in)), (grid, w)
        if grid == (5, 7, 9):
            assert int(np.sum(np.diff(goff) == 0)) > 0   # windows with no aligned token


def test_aligned_global_permute_validation(lib):
    big = FAKE + (1 << 30)
    G3, C3 = atlas.Grid3, atlas.Cube3
    for fn in (lib.atlas_aligned_global_reorder, lib.atlas_aligned_global_unorder):
        call = lambda src=FAKE, dst=big, b=1, grid=G3(4, 8, 8), cube=C3(2, 4, 4), \
            gg=G3(2, 4, 4), hd=64, dt=atlas.FP32: fn(src, dst, b, grid, cube, gg, 2, hd, dt,
                                                      None, None)
        assert call(src=None) == atlas.ERR_NULL
        assert call(dst=None) == atlas.ERR_NULL
        assert call(gg=G3(2, 0, 4)) == atlas.ERR_SHAPE
        assert call(cube=C3(2, 4, 0)) == atlas.ERR_SHAPE
        assert call(grid=G3(-1, 8, 8)) == atlas.ERR_SHAPE
        assert call(b=-1) == atlas.ERR_SHAPE
        assert call(src=FAKE + 8) == atlas.ERR_ALIGN
        assert call(dst=FAKE + 64) == atlas.ERR_ALIAS
        assert call(dt=7) == atlas.ERR_UNSUPPORTED


def test_aligned_global_offsets_property(lib):
    """Many random shapes: the range lengths of the aligned order equal the
    number of global tokens whose alignment point floor(x*E/(c*e)) falls in
    each detail cube, counted token by token; the ranges are the prefix sums
    of those counts in the cube grid's raster order."""
    import numpy as np
    rng = np.random.default_rng(2026)
    for _ in range(300):
        grid = tuple(int(v) for v in rng.integers(1, 40, size=3))
        cube = tuple(int(min(g, v)) for g, v in zip(grid, rng.integers(1, 17, size=3)))
        gg = tuple(int(v) for v in rng.integers(1, 25, size=3))
        nb = [-(-E // c) for E, c in zip(grid, cube)]
        counts = np.zeros(nb[0] * nb[1] * nb[2], dtype=np.int64)
        bt = [x * grid[0] // (cube[0] * gg[0]) for x in range(gg[0])]
        bh = [x * grid[1] // (cube[1] * gg[1]) for x in range(gg[1])]
        bw = [x * grid[2] // (cube[2] * gg[2]) for x in range(gg[2])]
        for a in bt:
            for b in bh:
                for c in bw:
                    counts[(a * nb[1] + b) * nb[2] + c] += 1
        want = np.concatenate([[0], np.cumsum(counts)])
        got = atlas.aligned_global_offsets(grid, cube, gg).numpy()
        assert np.array_equal(got, want), (grid, cube, gg)


def test_plain_c_program_against_the_header(lib, tmp_path):
    """The boundary from C: tests/c_abi/host_calls.c, compiled with gcc
    against include/atlas.h and linked to libatlas.so, runs its host-only
    checks (window offsets of the cube and aligned orders against counts from
    the definitions, status names, an argument error) and prints ok."""
    src = os.path.join(ROOT, "tests", "c_abi", "host_calls.c")
    exe = str(tmp_path / "host_calls")
    libdir = os.path.dirname(atlas.LIB_PATH)
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-O1", src, "-I", os.path.join(ROOT, "include"),
           "-L", libdir, "-l:libatlas.so", f"-Wl,-rpath,{libdir}", "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
