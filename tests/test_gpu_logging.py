"""Launch logging and NVTX ranges (both off by default).

ATLAS_LOG=1 makes every kernel launch print one line to stderr (kernel, grid,
block, dynamic shared memory and the work it walks); ATLAS_NVTX=1 wraps every
C-ABI call in an NVTX range. The chain runs in a child process so that the
environment is read fresh, and its results must not change.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

SCRIPT = textwrap.dedent("""
    import torch
    from video_dit_windowed_b200 import atlas
    from video_dit_windowed_b200.workloads import normal
    grid, cube, N, G, L = (6, 16, 16), (3, 8, 8), 1536, 96, 192
    rope = atlas.make_rope(10000.0, (44, 42, 42), (1.0, 1.0, 1.0))
    x = {s: normal((N if s.endswith("_d") else G, 2, 128), s, torch.bfloat16, seed=5,
                   device="cuda") for s in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")}
    q, k = torch.empty_like(x["q_d"]), torch.empty_like(x["k_d"])
    atlas.cube_reorder(x["q_d"], q, grid, cube, rope)
    atlas.cube_reorder(x["k_d"], k, grid, cube, rope)
    o_d, o_g = torch.empty_like(q), torch.empty_like(x["q_g"])
    atlas.local_global_attn(q, k, x["v_d"], L, x["q_g"], x["k_g"], x["v_g"], o_d, o_g)
    torch.cuda.synchronize()
    assert atlas.last_device_error() == 0
    print(float(o_d.float().sum()), float(o_g.float().sum()))
""")


def run(env_extra):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root + os.pathsep + os.environ.get("PYTHONPATH", ""))
    for k in ("ATLAS_LOG", "ATLAS_NVTX"):
        env.pop(k, None)
    env.update(env_extra)
    res = subprocess.run([sys.executable, "-c", SCRIPT], cwd=root, env=env, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    return res


def test_launch_log_lines_and_unchanged_results():
    quiet = run({})
    assert "[atlas]" not in quiet.stderr
    loud = run({"ATLAS_LOG": "1", "ATLAS_NVTX": "1"})
    lines = [l for l in loud.stderr.splitlines() if l.startswith("[atlas]")]
    assert sum("permute_rope_kernel" in l for l in lines) == 2, lines
    attn = [l for l in lines if "attn_tc_kernel" in l]
    assert len(attn) == 1 and "grid" in attn[0] and "units" in attn[0], lines
    assert loud.stdout == quiet.stdout
