"""GPU parity of the cube reorder / unorder and the 3D RoPE pass against the
fp64 oracle, through the C-ABI (steps 1 and 2 of the path).

Passages: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie 1
Fase 2 (cube reorder), Fase 1 (temporal RoPE scale r_t) and Methodologie 2
(position alignment of the global proxy).

Reorder and unorder are compared bit for bit; RoPE within 1 ulp of the I/O
type plus 2^-20 of the pair magnitude (tests/helpers.py).
"""
import numpy as np
import pytest
import torch

from helpers import assert_rope_close, check_no_device_error, f64, orc
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import WORKLOADS, normal

pytestmark = pytest.mark.gpu

DEV = "cuda"

# grid, cube, heads, head_dim, dtype
CASES = [
    ((4, 8, 8), (2, 4, 4), 2, 64, "fp32"),
    ((4, 8, 8), (2, 4, 4), 2, 64, "bf16"),
    ((3, 6, 10), (3, 2, 5), 3, 128, "bf16"),
    ((2, 4, 6), (1, 2, 3), 5, 64, "bf16"),
    ((6, 4, 4), (2, 4, 2), 1, 128, "fp32"),
    ((5, 3, 7), (1, 1, 1), 7, 64, "bf16"),
    ((2, 3, 4), (2, 3, 4), 40, 128, "bf16"),
    ((7, 9, 11), (7, 3, 11), 4, 64, "bf16"),
]
ROPES = [
    (10000.0, (16, 24, 24), (1.0, 1.0, 1.0)),
    (10000.0, (16, 24, 24), (4.0, 2.0, 2.0)),
]


def tdt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


def split_for(hd):
    return (16, 24, 24) if hd == 64 else (44, 42, 42)


def rand(n, heads, hd, dtype, stream):
    return normal((n, heads, hd), stream, tdt(dtype), seed=0, device=DEV)


@pytest.mark.parametrize("grid,cube,heads,hd,dtype", CASES)
def test_reorder_unorder_bit_exact(grid, cube, heads, hd, dtype):
    n = grid[0] * grid[1] * grid[2]
    x = rand(n, heads, hd, dtype, 1)
    y = torch.empty_like(x)
    z = torch.empty_like(x)
    atlas.cube_reorder(x, y, grid, cube)
    atlas.cube_unorder(y, z, grid, cube)
    torch.cuda.synchronize()
    check_no_device_error()
    xh = x.cpu().view(torch.uint8).numpy()
    expect = orc().cube_reorder(xh.reshape(n, -1), grid, cube)
    assert y.cpu().view(torch.uint8).numpy().reshape(n, -1).tobytes() == expect.tobytes()
    assert torch.equal(z.view(torch.uint8), x.view(torch.uint8))


def test_reorder_preserves_every_bit_pattern():
    grid, cube = (2, 4, 8), (1, 2, 4)
    n = 64
    raw = torch.randint(0, 1 << 16, (n, 3, 64), dtype=torch.int32,
                        generator=torch.Generator().manual_seed(3)).to(torch.int16)
    raw[::5, 0, :8] = 0x7FC1   # NaN payloads
    raw[::7, 1, :8] = -0x8000  # negative zero
    x = raw.view(torch.bfloat16).to(DEV)
    y, z = torch.empty_like(x), torch.empty_like(x)
    atlas.cube_reorder(x, y, grid, cube)
    atlas.cube_unorder(y, z, grid, cube)
    torch.cuda.synchronize()
    assert torch.equal(z.view(torch.int16), x.view(torch.int16))
    expect = orc().cube_reorder(raw.numpy().view(np.uint8).reshape(n, -1), grid, cube)
    assert y.cpu().view(torch.uint8).numpy().reshape(n, -1).tobytes() == expect.tobytes()


@pytest.mark.parametrize("grid,cube,heads,hd,dtype", CASES)
@pytest.mark.parametrize("theta,split64,scales", ROPES)
def test_reorder_rope_matches_oracle(grid, cube, heads, hd, dtype, theta, split64, scales):
    n = grid[0] * grid[1] * grid[2]
    split = split64 if hd == 64 else split_for(hd)
    x = rand(n, heads, hd, dtype, 0)
    y = torch.empty_like(x)
    atlas.cube_reorder(x, y, grid, cube, atlas.make_rope(theta, split, scales))
    torch.cuda.synchronize()
    check_no_device_error()
    xd = f64(x)
    exact_raster = orc().rope3d_grid(xd, grid, theta, split, scales)
    exact = orc().cube_reorder(exact_raster, grid, cube)
    x_in = orc().cube_reorder(xd, grid, cube)
    assert_rope_close(f64(y), exact, x_in, dtype)


@pytest.mark.parametrize("grid,cube,heads,hd,dtype", CASES[:5])
def test_rope3d_in_place_and_composition(grid, cube, heads, hd, dtype):
    n = grid[0] * grid[1] * grid[2]
    split = split_for(hd)
    rope = atlas.make_rope(10000.0, split, (4.0, 8.0, 8.0))
    x = rand(n, heads, hd, dtype, 3)
    y = torch.empty_like(x)
    atlas.rope3d(x, y, grid, rope)
    xi = x.clone()
    atlas.rope3d(xi, xi, grid, rope)
    fused = torch.empty_like(x)
    atlas.cube_reorder(x, fused, grid, cube, rope)
    two_step = torch.empty_like(x)
    atlas.cube_reorder(y, two_step, grid, cube)
    torch.cuda.synchronize()
    check_no_device_error()
    assert torch.equal(xi.view(torch.uint8), y.view(torch.uint8))
    assert torch.equal(fused.view(torch.uint8), two_step.view(torch.uint8))
    exact = orc().rope3d_grid(f64(x), grid, 10000.0, split, (4.0, 8.0, 8.0))
    assert_rope_close(f64(y), exact, f64(x), dtype)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_zero_scales_equal_pure_reorder(dtype):
    grid, cube, heads, hd = (4, 8, 8), (2, 4, 4), 3, 64
    n = 256
    x = rand(n, heads, hd, dtype, 4)
    a, b = torch.empty_like(x), torch.empty_like(x)
    atlas.cube_reorder(x, a, grid, cube, atlas.make_rope(10000.0, (16, 24, 24), (0, 0, 0)))
    atlas.cube_reorder(x, b, grid, cube)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@pytest.mark.parametrize("name", ["720p", "global_only", "4k", "4k_long"])
def test_full_size_reorder_rope(name):
    """At full size: the permutation bit-exact everywhere (oracle indices,
    gathered on device), RoPE on sampled rows, unorder restoring the input."""
    w = WORKLOADS[name]
    torch.cuda.empty_cache()
    if w.n_detail == 0:
        grid, rows, scales = w.global_grid, w.n_global, w.global_scales
    else:
        grid, rows, scales = w.grid, w.n_detail, w.detail_scales
    x = normal((rows, w.heads, w.head_dim), "q_d", w.torch_dtype, device=DEV)
    y = torch.empty_like(x)
    rope = atlas.make_rope(w.theta, w.split, scales)
    if w.n_detail:
        atlas.cube_reorder(x, y, grid, w.cube)
        pos = torch.from_numpy(orc().cube_positions(grid, w.cube)).to(DEV)
        inv = torch.empty_like(pos)
        inv[pos] = torch.arange(rows, device=DEV)
        assert torch.equal(y.view(torch.int16), x[inv].view(torch.int16))
        z = torch.empty_like(x)
        atlas.cube_unorder(y, z, grid, w.cube)
        assert torch.equal(z.view(torch.int16), x.view(torch.int16))
        del z
        atlas.cube_reorder(x, y, grid, w.cube, rope)
        gen = np.random.default_rng(0)
        sample = np.unique(np.concatenate([[0, rows - 1], gen.integers(0, rows, 2000)]))
        got = f64(y[pos[torch.as_tensor(sample, device=DEV)]])
    else:
        atlas.rope3d(x, y, grid, rope)
        gen = np.random.default_rng(0)
        sample = np.unique(np.concatenate([[0, rows - 1], gen.integers(0, rows, 2000)]))
        got = f64(y[torch.as_tensor(sample, device=DEV)])
    torch.cuda.synchronize()
    check_no_device_error()
    xs = f64(x[torch.as_tensor(sample, device=DEV)])
    exact = orc().rope3d_rows(xs, sample, grid, w.theta, w.split, scales)
    assert_rope_close(got, exact, xs, w.dtype)
    del x, y
    torch.cuda.empty_cache()


def test_plain_c_program_on_the_gpu(tmp_path):
    """The boundary from C on the GPU: tests/c_abi/gpu_chain.c allocates with
    the CUDA runtime, reorders arbitrary bytes through libatlas.so, and
    compares them bit for bit with the oracle's permutation (linked only in
    this test), then checks that the unorder restores the input."""
    import os
    import subprocess
    import oracle
    from video_dit_windowed_b200 import atlas as _atlas
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = os.path.join(root, "tests", "c_abi", "gpu_chain.c")
    exe = str(tmp_path / "gpu_chain")
    libdir = os.path.dirname(_atlas.LIB_PATH)
    odir = os.path.dirname(oracle.LIB_PATH)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cmd = ["gcc", "-std=c11", "-Wall", "-Werror", "-O1", src,
           "-I", os.path.join(root, "include"), "-I", os.path.join(cuda, "include"),
           "-L", libdir, "-l:libatlas.so", f"-Wl,-rpath,{libdir}",
           "-L", odir, "-l:liboracle_atlas.so", f"-Wl,-rpath,{odir}",
           "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}",
           "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
