"""The entry point that allocates no device memory.

Some callers cannot let a library call cudaMalloc: a serving process whose
device memory is reserved up front by its own allocator and budget, or a
latency-critical loop that cannot take cudaMalloc's implicit device-wide
synchronisation. For them, ``atlas_cube_reorder_noalloc`` keeps the RoPE
cos/sin table in a fixed array compiled into the library instead of the
buffer ``atlas_cube_reorder`` allocates and caches. Its results must be those
of ``atlas_cube_reorder``, call after call, since every call rewrites the
shared array.

This file is collected last on purpose (it is named so): if it fails, a run
that stops at the first failure has already run every other test.
"""
import ctypes
import os
import subprocess
import sys
import textwrap

import pytest
import torch

from helpers import assert_rope_close, check_no_device_error, f64, orc
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import normal

pytestmark = pytest.mark.gpu
DEV = "cuda"

# Two calls in a row with different grids, RoPE scales and dtypes, so the
# second call must fully replace the table the first one left behind.
CALLS = [
    dict(grid=(21, 48, 80), cube=(3, 16, 16), heads=40, hd=128, dtype=torch.bfloat16,
         split=(44, 42, 42), scales=(1.0, 1.0, 1.0)),
    dict(grid=(4, 8, 8), cube=(2, 4, 4), heads=2, hd=64, dtype=torch.float32,
         split=(16, 24, 24), scales=(4.0, 2.0, 2.0)),
]


def _compare(call, seed):
    n = call["grid"][0] * call["grid"][1] * call["grid"][2]
    x = normal((n, call["heads"], call["hd"]), "q_d", call["dtype"], seed=seed, device=DEV)
    rope = atlas.make_rope(10000.0, call["split"], call["scales"])
    ref = torch.empty_like(x)
    got = torch.empty_like(x)
    atlas.cube_reorder(x, ref, call["grid"], call["cube"], rope)
    atlas.cube_reorder_noalloc(x, got, call["grid"], call["cube"], rope)
    torch.cuda.synchronize()
    check_no_device_error()
    dtype = "bf16" if call["dtype"] == torch.bfloat16 else "fp32"
    # within the RoPE tolerance of the other tests, measured against the
    # existing entry point's output (same table, same kernel: equal in fact)
    assert_rope_close(f64(got), f64(ref), f64(ref), dtype)
    assert torch.equal(got.view(torch.uint8), ref.view(torch.uint8))
    # and against the fp64 oracle's RoPE then reorder, on the first and last
    # head (the rotation is the same for every head)
    heads = [0, call["heads"] - 1]
    xs = f64(x[:, heads])
    exact = orc().cube_reorder(orc().rope3d_grid(xs, call["grid"], 10000.0, call["split"],
                                                 call["scales"]), call["grid"], call["cube"])
    assert_rope_close(f64(got[:, heads]), exact, orc().cube_reorder(xs, call["grid"],
                                                                    call["cube"]), dtype)


def test_noalloc_matches_reorder_twice():
    for i, call in enumerate(CALLS):
        _compare(call, seed=i)
    # and the first configuration once more, after the second overwrote it
    # (refilled), then again with the same grid and RoPE (the fill skipped)
    _compare(CALLS[0], seed=7)
    _compare(CALLS[0], seed=8)


def test_noalloc_pure_permutation():
    grid, cube = (3, 6, 10), (3, 2, 5)
    x = normal((180, 3, 128), "k_d", torch.bfloat16, device=DEV)
    ref, got = torch.empty_like(x), torch.empty_like(x)
    atlas.cube_reorder(x, ref, grid, cube)
    atlas.cube_reorder_noalloc(x, got, grid, cube)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.uint8), ref.view(torch.uint8))


def test_noalloc_rejects_tables_beyond_capacity():
    # T*(d_t/2) + H*(d_h/2) + W*(d_w/2) = 1*22 + 1*21 + 2048*21 > 32768 pairs
    grid, cube = (1, 1, 2048), (1, 1, 1)
    x = torch.zeros((2048, 1, 128), dtype=torch.bfloat16, device=DEV)
    y = torch.empty_like(x)
    rope = atlas.make_rope(10000.0, (44, 42, 42), (1.0, 1.0, 1.0))
    st = atlas.lib().atlas_cube_reorder_noalloc(
        ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()), atlas.Grid3(*grid),
        atlas.Cube3(*cube), 1, 128, atlas.BF16, ctypes.byref(rope),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == atlas.ERR_CAPACITY
    assert "CAPACITY" in atlas.status_string(st)


def test_noalloc_first_call_leaves_the_allocating_cache_empty():
    """In a fresh process, the no-alloc entry point (with RoPE, two grids)
    is the library's first call: afterwards the library holds no table in
    memory it allocated. The allocating entry point then adds one, so the
    count does see allocations."""
    script = textwrap.dedent("""
        import torch
        from video_dit_windowed_b200 import atlas
        x = torch.randn(8 * 16 * 16, 2, 128, device="cuda").to(torch.bfloat16)
        y = torch.empty_like(x)
        rope = atlas.make_rope(10000.0, (44, 42, 42), (1.0, 1.0, 1.0))
        atlas.cube_reorder_noalloc(x, y, (8, 16, 16), (2, 8, 8), rope)
        atlas.cube_reorder_noalloc(x, y, (4, 32, 16), (2, 8, 8), rope)
        torch.cuda.synchronize()
        assert atlas.last_device_error() == 0
        assert atlas.cached_rope_tables() == 0, atlas.cached_rope_tables()
        atlas.cube_reorder(x, y, (8, 16, 16), (2, 8, 8), rope)
        torch.cuda.synchronize()
        assert atlas.cached_rope_tables() == 1, atlas.cached_rope_tables()
        print("fresh process ok")
    """)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root + os.pathsep + os.environ.get("PYTHONPATH", ""))
    res = subprocess.run([sys.executable, "-c", script], cwd=root, env=env,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "fresh process ok" in res.stdout
