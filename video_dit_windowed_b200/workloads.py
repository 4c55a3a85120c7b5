"""Workload shapes and the seeded synthetic-input generator.

This module holds data only: the five token-grid workloads (sizes, cube
shapes, RoPE splits and per-axis position scales) and a seeded N(0,1) input
generator. It contains none of the attention path's arithmetic, so both the
CUDA path's callers and the fp64 oracle's callers can draw their inputs from
it without sharing any of the method.

Inputs are iid N(0,1). Each tensor has its own stream id (q_d=0, k_d=1, v_d=2,
q_g=3, k_g=4, v_g=5) and every workload uses seed 0. The generator is torch's
(Philox, counter-based, on CUDA devices; mt19937 on the CPU): values drawn on
a GPU differ from values drawn on the CPU, so a parity test always hands the
oracle the exact bits the GPU consumed (copied back), never a regeneration.
Samples are drawn in float32 and rounded to bfloat16 round-to-nearest-even.

Position scales follow the pages' two rules (AtlasVid technical summary,
Methodologie 1 Fase 1: temporal indices times r_t; Methodologie 2, position
alignment: global-proxy coordinates times the resolution ratios W/w, H/h,
T/t): a token's RoPE position is (t*s_t, h*s_h, w*s_w) with no offset.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

STREAMS = {"q_d": 0, "k_d": 1, "v_d": 2, "q_g": 3, "k_g": 4, "v_g": 5}


@dataclass(frozen=True)
class Workload:
    name: str
    grid: tuple            # detail grid (T, H, W); (0, 0, 0) when there is none
    cube: tuple            # cube (ct, ch, cw)
    global_grid: tuple     # proxy grid (t, h, w); (0, 0, 0) when there is none
    heads: int
    head_dim: int
    dtype: str             # "bf16" or "fp32"
    split: tuple           # RoPE head_dim split (d_t, d_h, d_w)
    detail_scales: tuple   # (s_t, s_h, s_w) for detail tokens
    global_scales: tuple   # (s_t, s_h, s_w) for global tokens
    theta: float = 10000.0
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def n_detail(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def window_len(self) -> int:
        ct, ch, cw = self.cube
        return ct * ch * cw

    @property
    def n_windows(self) -> int:
        if not self.n_detail:
            return 0
        n = 1
        for E, c in zip(self.grid, self.cube):
            n *= -(-E // c)
        return n

    @property
    def partial(self) -> bool:
        """True when the cube does not divide the grid (variable windows)."""
        return bool(self.n_detail) and any(E % c for E, c in zip(self.grid, self.cube))

    def extents(self, axis: int, cube=None, grid=None):
        """Cube extents along one axis (the last one partial if need be)."""
        E = (grid or self.grid)[axis]
        c = (cube or self.cube)[axis]
        return [min(c, E - b * c) for b in range(-(-E // c))]

    @property
    def n_global(self) -> int:
        t, h, w = self.global_grid
        return t * h * w

    @property
    def softmax_scale(self) -> float:
        return self.head_dim ** -0.5

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def aligned_boxes(self, axis: int):
        """Global tokens aligned with each detail cube along one axis: global
        index x of e tokens sits at detail position x*E/e, in detail cube
        floor(x*E/(c*e)); cube b holds global indices [ceil(b*c*e/E),
        ceil((b+1)*c*e/E)) clipped to e."""
        E, c, e = self.grid[axis], self.cube[axis], self.global_grid[axis]
        start = lambda b: min(-(-(b * c * e) // E), e)
        return [start(b + 1) - start(b) for b in range(-(-E // c))]

    def allowed_pairs(self, mask: str = "all") -> int:
        """Allowed (query, key) pairs of one problem and one head. mask:
        "all" (detail: own cube + every global key), "aligned" (own cube +
        the global tokens aligned with it), "raster" (windows of window_len
        consecutive raster rows + every global key), "dense" (every token
        sees every token)."""
        N, G = self.n_detail, self.n_global
        if mask == "dense":
            return (N + G) ** 2
        if mask == "raster":
            return N * self.window_len + N * G + G * G
        win = 1
        for a in range(3):
            win *= sum(e * e for e in self.extents(a)) if N else 0
        if mask == "all":
            return win + N * G + G * G
        cross = 1
        for a in range(3):
            cross *= sum(e * g for e, g in zip(self.extents(a), self.aligned_boxes(a))) if N else 0
        return win + cross + G * G

    def unmasked_flops(self, mask: str = "all") -> int:
        """2*D FLOPs for q.k plus 2*D for p*v, per allowed (query, key) pair."""
        return 4 * self.head_dim * self.heads * self.allowed_pairs(mask)

    def reorder_rope_bytes(self) -> int:
        """One read and one write of detail Q, K, V plus global Q, K."""
        rows = 3 * self.n_detail + 2 * self.n_global
        return 2 * rows * self.heads * self.head_dim * self.elem_bytes


WORKLOADS = {
    "tiny": Workload(
        "tiny", (4, 8, 8), (2, 4, 4), (2, 4, 4), 2, 64, "fp32", (16, 24, 24),
        (1.0, 1.0, 1.0), (4.0, 2.0, 2.0),
        note="256 detail tokens, 8 windows of 32; 32 global tokens"),
    "720p": Workload(
        "720p", (21, 48, 80), (3, 16, 16), (21, 12, 20), 40, 128, "bf16",
        (44, 42, 42), (1.0, 1.0, 1.0), (1.0, 4.0, 4.0),
        note="80,640 detail tokens, 105 windows of 768; 5,040 global tokens"),
    "global_only": Workload(
        "global_only", (0, 0, 0), (1, 1, 1), (21, 30, 52), 40, 128, "bf16",
        (44, 42, 42), (1.0, 1.0, 1.0), (4.0, 1.0, 1.0),
        note="full self-attention over 32,760 proxy tokens, r_t=4"),
    "4k": Workload(
        "4k", (21, 144, 240), (3, 16, 16), (21, 18, 30), 40, 128, "bf16",
        (44, 42, 42), (1.0, 1.0, 1.0), (1.0, 8.0, 8.0),
        note="725,760 detail tokens, 945 windows of 768; 11,340 global tokens"),
    "4k_long": Workload(
        "4k_long", (42, 144, 240), (6, 16, 16), (21, 18, 30), 40, 128, "bf16",
        (44, 42, 42), (2.0, 1.0, 1.0), (4.0, 8.0, 8.0),
        note="1,451,520 detail tokens, 945 windows of 1,536; 11,340 global"),
    # Lengths the pages report generating (8K 29 frames, 2K 321 frames). Latent
    # grid: frames (F-1)/4+1, pixels / 16 per side (8x VAE, 2x2 patches); the
    # cube does not divide every axis, so windows include partial cubes.
    "8k29": Workload(
        "8k29", (8, 270, 480), (3, 16, 16), (8, 27, 48), 40, 128, "bf16",
        (44, 42, 42), (1.0, 1.0, 1.0), (1.0, 10.0, 10.0),
        note="7680x4320, 29 frames: 1,036,800 detail tokens (partial cubes along t and h); "
             "10,368 global tokens at ratio 10"),
    "2k321": Workload(
        "2k321", (81, 90, 160), (3, 16, 16), (27, 18, 32), 40, 128, "bf16",
        (44, 42, 42), (1.0, 1.0, 1.0), (3.0, 5.0, 5.0),
        note="2560x1440, 321 frames: 1,166,400 detail tokens (partial cubes along h); "
             "15,552 global tokens at ratios 3, 5, 5"),
}

# The order the workloads are listed in (small CPU-checkable case first).
ORDER = ["tiny", "720p", "global_only", "4k", "4k_long"]


def generator(stream: str | int, seed: int = 0, device="cpu") -> torch.Generator:
    sid = STREAMS[stream] if isinstance(stream, str) else int(stream)
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + sid)
    return g


def normal(shape, stream, dtype=torch.bfloat16, seed: int = 0, device="cpu",
           chunk_elems: int = 1 << 28, out: torch.Tensor | None = None):
    """iid N(0,1) samples of ``shape`` drawn in float32 chunks of
    ``chunk_elems`` and rounded to ``dtype``; deterministic for a given
    (stream, seed, device, chunk_elems)."""
    g = generator(stream, seed, device)
    if out is None:
        out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        tmp = torch.randn(e - s, generator=g, dtype=torch.float32, device=device)
        flat[s:e].copy_(tmp)
        del tmp
    return out


def make_inputs(w: Workload, device="cpu", pin: bool = False, batch: int = 1):
    """Raster-ordered detail Q/K/V [batch*N, heads, D] and global Q/K/V
    [batch*G, heads, D] (problems stacked along the rows)."""
    dt = w.torch_dtype
    shp_d = (batch * w.n_detail, w.heads, w.head_dim)
    shp_g = (batch * w.n_global, w.heads, w.head_dim)
    t = {}
    for name, shp in (("q_d", shp_d), ("k_d", shp_d), ("v_d", shp_d),
                      ("q_g", shp_g), ("k_g", shp_g), ("v_g", shp_g)):
        t[name] = normal(shp, name, dt, w.seed, device)
        if pin and device == "cpu":
            t[name] = t[name].pin_memory()
    return t
