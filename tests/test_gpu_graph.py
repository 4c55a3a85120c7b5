"""The path's C-ABI calls inside a CUDA graph.

Every entry point is capturable once its first call on the device has run
(that call may cache a RoPE table and set kernel attributes): the calls only
enqueue kernels on the given stream and allocate nothing. A step captured
with torch.cuda.CUDAGraph and replayed must give the bits of the eager step,
for the forward path and the backward.
"""
import pytest
import torch

from helpers import check_no_device_error
from video_dit_windowed_b200 import atlas
from video_dit_windowed_b200.workloads import WORKLOADS, make_inputs, normal

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _step(w, x, bufs, rd, rg, lse):
    q_d, k_d, v_d, q_g, k_g, o_d, o_g, o_r = bufs
    atlas.cube_reorder(x["q_d"], q_d, w.grid, w.cube, rd)
    atlas.cube_reorder(x["k_d"], k_d, w.grid, w.cube, rd)
    atlas.cube_reorder(x["v_d"], v_d, w.grid, w.cube)
    atlas.rope3d(x["q_g"], q_g, w.global_grid, rg)
    atlas.rope3d(x["k_g"], k_g, w.global_grid, rg)
    atlas.local_global_attn(q_d, k_d, v_d, w.window_len, q_g, k_g, x["v_g"], o_d, o_g, lse)
    atlas.cube_unorder(o_d, o_r, w.grid, w.cube)


@pytest.mark.parametrize("name", ["tiny", "720p"])
def test_forward_step_in_cuda_graph(name):
    import dataclasses
    w = WORKLOADS[name]
    if name == "720p":
        w = dataclasses.replace(w, heads=4)
    x = make_inputs(w, device=DEV)
    rd = atlas.make_rope(w.theta, w.split, w.detail_scales)
    rg = atlas.make_rope(w.theta, w.split, w.global_scales)
    e = torch.empty_like
    bufs = [e(x["q_d"]), e(x["k_d"]), e(x["v_d"]), e(x["q_g"]), e(x["k_g"]), e(x["q_d"]),
            e(x["q_g"]), e(x["q_d"])]
    lse = torch.empty(w.heads, w.n_detail + w.n_global, dtype=torch.float32, device=DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _step(w, x, bufs, rd, rg, lse)             # first calls: caches and attributes
    torch.cuda.synchronize()
    eager = [b.clone() for b in bufs] + [lse.clone()]
    for b in bufs:
        b.zero_()
    lse.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _step(w, x, bufs, rd, rg, lse)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    check_no_device_error()
    for a, b in zip(eager, bufs + [lse]):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    # new inputs in the same buffers flow through the same graph
    x["q_d"].copy_(normal(x["q_d"].shape, "q_g", x["q_d"].dtype, seed=9, device=DEV))
    g.replay()
    ref = e(bufs[7])
    with torch.cuda.stream(s):
        _step(w, x, [e(b) for b in bufs[:7]] + [ref], rd, rg, torch.empty_like(lse))
    torch.cuda.synchronize()
    assert torch.equal(ref.view(torch.uint8), bufs[7].view(torch.uint8))


def test_backward_in_cuda_graph():
    N, L, G, heads, hd = 1536, 768, 300, 2, 128
    mk = lambda rows, st: normal((rows, heads, hd), st, torch.bfloat16, seed=3, device=DEV)
    t = {st: mk(N if st.endswith("_d") else G, st) for st in ("q_d", "k_d", "v_d", "q_g",
                                                             "k_g", "v_g")}
    do_d, do_g = mk(N, 0), mk(G, 3)
    o_d, o_g = torch.empty_like(t["q_d"]), torch.empty_like(t["q_g"])
    lse = torch.empty(1, heads, N + G, dtype=torch.float32, device=DEV)
    grads = [torch.empty_like(t[st]) for st in ("q_d", "k_d", "v_d", "q_g", "k_g", "v_g")]
    delta = torch.empty_like(lse)

    def step():
        atlas.local_global_attn_ex(t["q_d"], t["k_d"], t["v_d"], t["q_g"], t["k_g"], t["v_g"],
                                   o_d, o_g, lse, window_len=L)
        atlas.local_global_attn_bwd(t["q_d"], t["k_d"], t["v_d"], o_d, do_d, t["q_g"], t["k_g"],
                                    t["v_g"], o_g, do_g, lse, *grads, delta, window_len=L)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        step()
    torch.cuda.synchronize()
    eager = [x.clone() for x in grads]
    for x in grads:
        x.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    g.replay()
    torch.cuda.synchronize()
    check_no_device_error()
    for a, b in zip(eager, grads):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
