"""Pins that tie the fp64 oracle to facts fixed outside the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with a fact that the pages or the mathematics fix:
an independent construction (numpy reshape/transpose for the cube order,
torch's dense scaled-dot-product attention with an explicit boolean mask for
the attention), a closed form (literal RoPE angles, O = V for 1-token
windows, mean of V when all logits tie), an invariant (bijection, exact
inverse, pair norms, relative-position property, rows summing to 1), or a
special case that reduces to textbook full attention. The test modules run
them against the real oracle (all must pass) and against copies of the
oracle with a planted mistake (each mutant must fail at least one).

Passages: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie 1
Fase 1 (temporal RoPE scale r_t), Fase 2 (cube reorder, window attention), 2
(asymmetric hierarchical attention; position alignment).
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(v) for v in line.split()])
    return rows


# ---------------------------------------------------------------------------
# Cube reorder
# ---------------------------------------------------------------------------

CUBE_CASES = [
    ((4, 8, 8), (2, 4, 4)),
    ((3, 6, 10), (3, 2, 5)),
    ((2, 4, 6), (1, 2, 3)),
    ((6, 4, 4), (2, 4, 2)),
    ((5, 3, 7), (1, 1, 1)),
    ((2, 3, 4), (2, 3, 4)),
]


def rearrange_order(grid, cube):
    """order[j] = raster index of the token at cube position j, built with a
    reshape/transpose: (T/ct, ct, H/ch, ch, W/cw, cw) -> cube axes first."""
    T, H, W = grid
    ct, ch, cw = cube
    idx = np.arange(T * H * W, dtype=np.int64).reshape(
        T // ct, ct, H // ch, ch, W // cw, cw)
    return idx.transpose(0, 2, 4, 1, 3, 5).reshape(-1)


def pin_cube_matches_rearrange(o):
    for grid, cube in CUBE_CASES:
        pos = o.cube_positions(grid, cube)
        order = rearrange_order(grid, cube)
        assert np.array_equal(pos[order], np.arange(pos.size)), (grid, cube)


def pin_cube_bijection(o):
    for grid, cube in CUBE_CASES:
        pos = o.cube_positions(grid, cube)
        assert np.array_equal(np.sort(pos), np.arange(pos.size)), (grid, cube)


def pin_cube_worked_example(o):
    for row in _golden_rows("cube_positions_example.txt"):
        T, H, W, ct, ch, cw, t, h, w, r, j = (int(v) for v in row)
        assert (t * H + h) * W + w == r
        assert o.cube_position((T, H, W), (ct, ch, cw), r) == j, row


def pin_cube_locality(o):
    """Every block of L consecutive positions is one geometric cube."""
    for grid, cube in CUBE_CASES:
        T, H, W = grid
        ct, ch, cw = cube
        L = ct * ch * cw
        pos = o.cube_positions(grid, cube)
        inv = np.empty_like(pos)
        inv[pos] = np.arange(pos.size)
        t, h, w = inv // (H * W), (inv // W) % H, inv % W
        for b in range(pos.size // L):
            sl = slice(b * L, (b + 1) * L)
            for coord, c in ((t, ct), (h, ch), (w, cw)):
                lo = coord[sl].min()
                assert lo % c == 0 and coord[sl].max() - lo == c - 1, (grid, cube, b)


def pin_cube_roundtrip_bytes(o):
    rng = np.random.default_rng(1)
    for grid, cube in CUBE_CASES:
        n = grid[0] * grid[1] * grid[2]
        x = rng.integers(0, 256, size=(n, 3, 10), dtype=np.uint8)
        # include NaN payload patterns when viewed as float32 / bfloat16
        x[::3, 0, :4] = np.frombuffer(np.array([0x7FC00001], np.uint32).tobytes(), np.uint8)
        y = o.cube_reorder(x, grid, cube)
        z = o.cube_unorder(y, grid, cube)
        assert z.tobytes() == x.tobytes(), (grid, cube)
        order = rearrange_order(grid, cube)
        assert y.tobytes() == x[order].tobytes(), (grid, cube)


def pin_cube_special_cases(o):
    for grid in ((3, 5, 7), (2, 2, 2)):
        n = grid[0] * grid[1] * grid[2]
        assert np.array_equal(o.cube_positions(grid, (1, 1, 1)), np.arange(n))
        assert np.array_equal(o.cube_positions(grid, grid), np.arange(n))


# Grids the cube does not divide: the last cube along such an axis is partial.
PARTIAL_CASES = [
    ((5, 7, 9), (2, 3, 4)),
    ((3, 5, 6), (2, 2, 4)),
    ((4, 8, 10), (2, 4, 4)),
    ((1, 3, 2), (3, 4, 5)),
    ((4, 8, 8), (2, 4, 4)),
]


def lexsort_order(grid, cube):
    """order[j] = raster index at cube position j, by sorting every token on
    (cube t, cube h, cube w, t in cube, h in cube, w in cube)."""
    T, H, W = grid
    ct, ch, cw = cube
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    t, h, w = t.ravel(), h.ravel(), w.ravel()
    return np.lexsort((w % cw, h % ch, t % ct, w // cw, h // ch, t // ct))


def pin_cube_partial_matches_lexsort(o):
    for grid, cube in PARTIAL_CASES + CUBE_CASES:
        pos = o.cube_positions(grid, cube)
        order = lexsort_order(grid, cube)
        assert np.array_equal(pos[order], np.arange(pos.size)), (grid, cube)


def pin_cube_windows_are_cubes(o):
    """Window offsets bound exactly the tokens of one (possibly partial) cube."""
    for grid, cube in PARTIAL_CASES + CUBE_CASES:
        T, H, W = grid
        ct, ch, cw = cube
        off = o.cube_windows(grid, cube)
        order = lexsort_order(grid, cube)
        t, h, w = order // (H * W), (order // W) % H, order % W
        key = ((t // ct) * -(-H // ch) + h // ch) * -(-W // cw) + w // cw
        counts = np.bincount(key, minlength=off.size - 1)
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)])), (grid, cube)
        for c in range(off.size - 1):
            assert np.all(key[off[c]:off[c + 1]] == c)


CUBE_PINS = [pin_cube_matches_rearrange, pin_cube_bijection, pin_cube_partial_matches_lexsort,
             pin_cube_windows_are_cubes,
             pin_cube_worked_example, pin_cube_locality,
             pin_cube_roundtrip_bytes, pin_cube_special_cases]


# ---------------------------------------------------------------------------
# 3D RoPE
# ---------------------------------------------------------------------------

def pin_rope_literal_angles(o):
    """theta=100, 4 channels per axis: frequencies are exactly 1 and 0.1."""
    for row in _golden_rows("rope_literal_angles.txt"):
        theta, dt, dh, dw, T, H, W, t, h, w, st, sh, sw = row[:13]
        angles = row[13:]
        grid = (int(T), int(H), int(W))
        r = (int(t) * grid[1] + int(h)) * grid[2] + int(w)
        D = int(dt + dh + dw)
        rng = np.random.default_rng(7)
        x = rng.standard_normal((1, 2, D))
        y = o.rope3d_rows(x, [r], grid, theta, (int(dt), int(dh), int(dw)),
                          (st, sh, sw))
        for head in range(2):
            for k, phi in enumerate(angles):
                x0, x1 = x[0, head, 2 * k], x[0, head, 2 * k + 1]
                c, s = math.cos(phi), math.sin(phi)
                assert abs(y[0, head, 2 * k] - (x0 * c - x1 * s)) < 1e-13, (row, k)
                assert abs(y[0, head, 2 * k + 1] - (x0 * s + x1 * c)) < 1e-13, (row, k)


def pin_rope_zero_scale_identity(o):
    grid = (3, 4, 5)
    n = 60
    x = np.random.default_rng(2).standard_normal((n, 3, 16))
    y = o.rope3d_grid(x, grid, 10000.0, (4, 6, 6), (0.0, 0.0, 0.0))
    assert np.array_equal(x, y)
    # origin token is never rotated, whatever the scales
    y = o.rope3d_rows(x[:1], [0], grid, 10000.0, (4, 6, 6), (4.0, 8.0, 8.0))
    assert np.array_equal(x[:1], y)


def pin_rope_pair_norms(o):
    grid = (4, 6, 8)
    x = np.random.default_rng(3).standard_normal((192, 2, 128))
    y = o.rope3d_grid(x, grid, 10000.0, (44, 42, 42), (4.0, 8.0, 8.0))
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    assert np.max(np.abs(nx - ny)) < 1e-12


def pin_rope_relative_position(o):
    """<R(p)q, R(p')k> depends only on p - p' (axis by axis)."""
    grid = (6, 7, 9)
    H, W = grid[1], grid[2]
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))
    split, scales = (16, 24, 24), (4.0, 2.0, 3.0)

    def dot_at(pq, pk):
        rq = (pq[0] * H + pq[1]) * W + pq[2]
        rk = (pk[0] * H + pk[1]) * W + pk[2]
        a = o.rope3d_rows(q, [rq], grid, 10000.0, split, scales)
        b = o.rope3d_rows(k, [rk], grid, 10000.0, split, scales)
        return float(np.sum(a * b))

    base = dot_at((1, 2, 3), (0, 0, 1))
    for shift in ((1, 0, 0), (0, 3, 0), (0, 0, 4), (4, 4, 5)):
        pq = (1 + shift[0], 2 + shift[1], 3 + shift[2])
        pk = (0 + shift[0], 0 + shift[1], 1 + shift[2])
        assert abs(dot_at(pq, pk) - base) < 1e-11, shift
    # and a different offset gives a different value (the angle is not lost)
    assert abs(dot_at((2, 2, 3), (0, 0, 1)) - base) > 1e-6


def pin_rope_temporal_scale(o):
    """Scaling the temporal index by r_t equals placing the token at t*r_t."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 2, 64))
    split = (16, 24, 24)
    for r_t in (2.0, 4.0):
        for (t, h, w) in ((1, 2, 3), (3, 0, 5)):
            small = (4, 4, 8)
            tall = (4 * 4, 4, 8)
            a = o.rope3d_rows(x, [(t * 4 + h) * 8 + w], small, 10000.0, split,
                              (r_t, 1.0, 1.0))
            tt = int(t * r_t)
            b = o.rope3d_rows(x, [(tt * 4 + h) * 8 + w], tall, 10000.0, split,
                              (1.0, 1.0, 1.0))
            assert np.max(np.abs(a - b)) < 1e-12


def pin_rope_complex_form(o):
    """At unit scales the result equals the complex-multiplication form of
    rotary embedding, per axis: (x0 + i x1) * exp(i * p * theta^(-2k/d))."""
    grid = (3, 4, 5)
    n = 60
    x = torch.randn(n, 2, 64, dtype=torch.float64,
                    generator=torch.Generator().manual_seed(6))
    y = o.rope3d_grid(x.numpy(), grid, 10000.0, (16, 24, 24), (1.0, 1.0, 1.0))
    pos = torch.stack(torch.meshgrid(torch.arange(3), torch.arange(4),
                                     torch.arange(5), indexing="ij"), -1).reshape(n, 3)
    parts = []
    off = 0
    for axis, d in enumerate((16, 24, 24)):
        freqs = 10000.0 ** (-torch.arange(0, d, 2, dtype=torch.float64) / d)
        ang = pos[:, axis:axis + 1].double() * freqs[None, :]          # [n, d/2]
        xc = torch.view_as_complex(x[..., off:off + d].reshape(n, 2, d // 2, 2).contiguous())
        rot = xc * torch.polar(torch.ones_like(ang), ang)[:, None, :]
        parts.append(torch.view_as_real(rot).reshape(n, 2, d))
        off += d
    ref = torch.cat(parts, -1).numpy()
    assert np.max(np.abs(ref - y)) < 1e-12


def pin_rope_heads_identical(o):
    grid = (2, 3, 4)
    x1 = np.random.default_rng(8).standard_normal((24, 1, 32))
    x = np.repeat(x1, 4, axis=1)
    y = o.rope3d_grid(x, grid, 10000.0, (8, 12, 12), (4.0, 2.0, 2.0))
    for hd in range(4):
        assert np.array_equal(y[:, hd], y[:, 0])


def pin_rope_negated_scales_transpose(o):
    """Rotation with negated scales is the inverse and the transpose of the
    rotation: R(-s) R(s) x = x and <R(s) x, y> = <x, R(-s) y> (what the
    backward of the reorder with RoPE uses)."""
    rng = np.random.default_rng(3)
    grid, split, sc = (3, 4, 5), (4, 6, 6), (2.0, 1.0, 3.0)
    neg = tuple(-v for v in sc)
    x = rng.standard_normal((60, 2, 16))
    y = rng.standard_normal((60, 2, 16))
    rx = o.rope3d_grid(x, grid, 100.0, split, sc)
    assert np.max(np.abs(o.rope3d_grid(rx, grid, 100.0, split, neg) - x)) < 1e-13
    lhs = np.sum(rx * y)
    rhs = np.sum(x * o.rope3d_grid(y, grid, 100.0, split, neg))
    assert abs(lhs - rhs) < 1e-11 * max(1.0, abs(lhs))


ROPE_PINS = [pin_rope_literal_angles, pin_rope_negated_scales_transpose, pin_rope_zero_scale_identity,
             pin_rope_pair_norms, pin_rope_relative_position,
             pin_rope_temporal_scale, pin_rope_complex_form,
             pin_rope_heads_identical]


# ---------------------------------------------------------------------------
# Asymmetric global-local attention
# ---------------------------------------------------------------------------

def geometric_mask(grid, cube, G):
    """Boolean allowed-matrix over [detail (cube order); global], built from
    cube ids that a reshape assigns to each token: a detail query may see
    keys with its own cube id and every global key; a global query may see
    only global keys."""
    T, H, W = grid
    ct, ch, cw = cube
    N = T * H * W
    if N:
        ids = np.arange(N // (ct * ch * cw)).reshape(T // ct, H // ch, W // cw)
        cube_of_raster = np.broadcast_to(
            ids[:, None, :, None, :, None],
            (T // ct, ct, H // ch, ch, W // cw, cw)).reshape(-1)
        cube_of_pos = cube_of_raster[rearrange_order(grid, cube)]
    else:
        cube_of_pos = np.zeros(0, dtype=np.int64)
    allowed = np.zeros((N + G, N + G), dtype=bool)
    allowed[:N, :N] = cube_of_pos[:, None] == cube_of_pos[None, :]
    allowed[:N, N:] = True
    allowed[N:, N:] = True
    return allowed


ATTN_CASES = [
    # grid, cube, G, heads, D
    ((4, 8, 8), (2, 4, 4), 32, 2, 64),
    ((2, 4, 6), (1, 2, 3), 5, 2, 16),
    ((2, 4, 4), (2, 2, 2), 1, 1, 8),
    ((3, 4, 4), (3, 4, 4), 0, 2, 16),
    ((2, 2, 4), (1, 1, 1), 0, 1, 8),
    ((0, 0, 0), (1, 1, 1), 40, 2, 16),
    ((2, 6, 4), (2, 3, 2), 7, 3, 32),
]


def _rand_case(grid, G, heads, D, seed):
    g = torch.Generator().manual_seed(seed)
    N = grid[0] * grid[1] * grid[2]
    mk = lambda n: torch.randn(n, heads, D, dtype=torch.float64, generator=g).numpy()
    return N, mk(N), mk(N), mk(N), mk(G), mk(G), mk(G)


def pin_attention_dense_sdpa(o):
    """Equal to dense masked softmax attention over all N+G tokens."""
    for ci, (grid, cube, G, heads, D) in enumerate(ATTN_CASES):
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 100 + ci)
        L = cube[0] * cube[1] * cube[2]
        scale = 1.0 / math.sqrt(D)
        od, og, lse = o.attention_full(qd, kd, vd, L, qg, kg, vg, scale)
        mask = torch.from_numpy(geometric_mask(grid, cube, G))
        q = torch.from_numpy(np.concatenate([qd, qg])).permute(1, 0, 2)
        k = torch.from_numpy(np.concatenate([kd, kg])).permute(1, 0, 2)
        v = torch.from_numpy(np.concatenate([vd, vg])).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=mask, scale=scale).permute(1, 0, 2).numpy()
        got = np.concatenate([od, og])
        assert np.max(np.abs(ref - got)) < 1e-12, (grid, cube, G)
        logits = (q @ k.transpose(1, 2)).numpy() * scale
        logits = np.where(mask.numpy()[None], logits, -np.inf)
        mx = logits.max(-1, keepdims=True)
        ref_lse = (mx + np.log(np.exp(logits - mx).sum(-1, keepdims=True)))[..., 0]
        assert np.max(np.abs(ref_lse - lse)) < 1e-12, (grid, cube, G)


def pin_attention_full_when_one_cube(o):
    """One cube covering the volume and no global tokens: full attention."""
    grid, heads, D = (2, 4, 4), 2, 16
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, 0, heads, D, 11)
    od, _, _ = o.attention_full(qd, kd, vd, N, qg, kg, vg, 0.3)
    q, k, v = (torch.from_numpy(a).permute(1, 0, 2) for a in (qd, kd, vd))
    ref = torch.softmax(q @ k.transpose(1, 2) * 0.3, -1) @ v
    assert np.max(np.abs(ref.permute(1, 0, 2).numpy() - od)) < 1e-12


def pin_attention_single_token_windows(o):
    """1x1x1 cubes and no global tokens: each row sees only itself, O = V."""
    grid, heads, D = (2, 3, 4), 2, 8
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, 0, heads, D, 12)
    od, _, lse = o.attention_full(qd, kd, vd, 1, qg, kg, vg, 0.25)
    assert np.array_equal(od, vd)
    ref_lse = 0.25 * np.einsum("nhd,nhd->hn", qd, kd)
    assert np.max(np.abs(ref_lse - lse)) < 1e-12


def pin_attention_zero_keys_mean(o):
    """K = 0: every allowed logit ties, O = mean of the allowed V rows."""
    grid, cube, G, heads, D = (2, 4, 4), (1, 2, 2), 6, 2, 8
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 13)
    kd[:] = 0.0
    kg[:] = 0.0
    L = 4
    od, og, lse = o.attention_full(qd, kd, vd, L, qg, kg, vg, 0.5)
    for i in range(N):
        w = i // L
        allowed_v = np.concatenate([vd[w * L:(w + 1) * L], vg])
        assert np.max(np.abs(od[i] - allowed_v.mean(0))) < 1e-12
    assert np.max(np.abs(og - vg.mean(0, keepdims=True))) < 1e-12
    assert np.max(np.abs(lse[:, :N] - math.log(L + G))) < 1e-12
    assert np.max(np.abs(lse[:, N:] - math.log(G))) < 1e-12


def pin_attention_rows_sum_to_one(o):
    for grid, cube, G, heads, D in ATTN_CASES:
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 14)
        vd[:] = 1.0
        vg[:] = 1.0
        L = cube[0] * cube[1] * cube[2]
        od, og, _ = o.attention_full(qd, kd, vd, L, qg, kg, vg, 1.0)
        assert np.max(np.abs(np.concatenate([od, og]) - 1.0)) < 1e-12


def pin_attention_global_ignores_detail(o):
    """Global rows see no detail key: changing detail K/V changes nothing."""
    grid, cube, G, heads, D = (2, 4, 4), (2, 2, 2), 9, 2, 16
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 15)
    _, og1, l1 = o.attention_full(qd, kd, vd, 8, qg, kg, vg, 0.25)
    _, og2, l2 = o.attention_full(qd, kd * 3.0 + 1.0, -vd, 8, qg, kg, vg, 0.25)
    assert np.array_equal(og1, og2) and np.array_equal(l1[:, N:], l2[:, N:])


def pin_attention_probe_mass(o):
    """V columns = indicators of (own window, other windows, global): the
    output columns are the attention mass on each group; the mass outside
    the own window and the global set is exactly 0."""
    grid, cube, G, heads, D = (2, 4, 8), (1, 2, 4), 5, 1, 8
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 16)
    L = 8
    nwin = N // L
    for w in range(nwin):
        vd[:] = 0.0
        vg[:] = 0.0
        vd[w * L:(w + 1) * L, :, 0] = 1.0
        vd[:w * L, :, 1] = 1.0
        vd[(w + 1) * L:, :, 1] = 1.0
        vg[:, :, 2] = 1.0
        od, og, _ = o.attention_full(qd, kd, vd, L, qg, kg, vg, 0.35)
        rows = slice(w * L, (w + 1) * L)
        assert np.all(od[rows, :, 1] == 0.0)
        assert np.all(od[rows, :, 0] > 0.0) and np.all(od[rows, :, 2] > 0.0)
        assert np.max(np.abs(od[rows, :, 0] + od[rows, :, 2] - 1.0)) < 1e-12
        assert np.all(og[:, :, 0] == 0.0) and np.all(og[:, :, 1] == 0.0)


def pin_attention_rejects_missing_rows(o):
    """A detail query whose window rows are not supplied is an error."""
    D = 8
    q = np.ones((1, D))
    k = np.zeros((4, D))
    try:
        o.attention_head(16, 8, 0, 1.0, k, k, 0, None, None, [9], q)
    except ValueError:
        pass
    else:
        raise AssertionError("missing window rows not detected")
    out, _ = o.attention_head(16, 8, 0, 1.0, np.zeros((8, D)), np.ones((8, D)),
                              8, None, None, [9], q)
    assert np.array_equal(out, np.ones((1, D)))


def pin_attention_partial_cubes_dense_sdpa(o):
    """Variable windows (partial cubes): equal to dense masked attention
    whose mask comes from token coordinates (same cube <=> same floor
    division), with detail tokens in the lexsort cube order."""
    for ci, (grid, cube) in enumerate(PARTIAL_CASES[:3]):
        T, H, W = grid
        ct, ch, cw = cube
        G, heads, D = 6, 2, 16
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 300 + ci)
        order = lexsort_order(grid, cube)
        t, h, w = order // (H * W), (order // W) % H, order % W
        key = np.stack([t // ct, h // ch, w // cw], -1)
        same = np.all(key[:, None, :] == key[None, :, :], -1)
        mask = np.zeros((N + G, N + G), dtype=bool)
        mask[:N, :N] = same
        mask[:N, N:] = True
        mask[N:, N:] = True
        off = o.cube_windows(grid, cube)
        od, og, lse = o.attention_full(qd, kd, vd, 1, qg, kg, vg, 0.25, win_off=off)
        q = torch.from_numpy(np.concatenate([qd, qg])).permute(1, 0, 2)
        k = torch.from_numpy(np.concatenate([kd, kg])).permute(1, 0, 2)
        v = torch.from_numpy(np.concatenate([vd, vg])).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=torch.from_numpy(mask), scale=0.25).permute(1, 0, 2).numpy()
        assert np.max(np.abs(ref - np.concatenate([od, og]))) < 1e-12, (grid, cube)


def pin_attention_offsets_equal_fixed_windows(o):
    """Offsets k*L give exactly the fixed-length-window result."""
    grid, cube, G, heads, D = (4, 8, 8), (2, 4, 4), 9, 2, 16
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 17)
    a = o.attention_full(qd, kd, vd, 32, qg, kg, vg, 0.3)
    b = o.attention_full(qd, kd, vd, 1, qg, kg, vg, 0.3, win_off=np.arange(0, N + 1, 32))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# "Aligned proxy tokens only": detail grid, cube, global grid.
ALIGNED_CASES = [
    ((4, 8, 8), (2, 4, 4), (2, 4, 4)),     # ratios 2, 2, 2; they divide the cube
    ((3, 8, 12), (3, 4, 4), (3, 2, 3)),    # ratios 1, 4, 4
    ((5, 7, 9), (2, 3, 4), (2, 3, 4)),     # ratios 2.5, 7/3, 9/4; partial cubes
    ((4, 6, 10), (2, 4, 4), (4, 3, 5)),    # ratios 1, 2, 2; partial cubes along h and w
]


def aligned_mask(grid, cube, global_grid):
    """Allowed-matrix of the aligned variant from token coordinates: detail
    cube ids by floor division, detail tokens in lexsort cube order; a global
    token's cube is the one holding its scaled position, floor(g*T/(t*c)) on
    each axis."""
    T, H, W = grid
    ct, ch, cw = cube
    t, h, w = global_grid
    N, G = T * H * W, t * h * w
    order = lexsort_order(grid, cube)
    dkey = np.stack([order // (H * W) // ct, (order // W) % H // ch, order % W // cw], -1)
    g = np.arange(G)
    gkey = np.stack([(g // (h * w)) * T // (t * ct), ((g // w) % h) * H // (h * ch),
                     (g % w) * W // (w * cw)], -1)
    mask = np.zeros((N + G, N + G), dtype=bool)
    mask[:N, :N] = np.all(dkey[:, None, :] == dkey[None, :, :], -1)
    mask[:N, N:] = np.all(dkey[:, None, :] == gkey[None, :, :], -1)
    mask[N:, N:] = True
    return mask


def pin_attention_aligned_dense_sdpa(o):
    """Aligned variant equal to dense masked attention (mask above)."""
    for ci, (grid, cube, gg) in enumerate(ALIGNED_CASES):
        G, heads, D = gg[0] * gg[1] * gg[2], 2, 16
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 400 + ci)
        od, og, lse = o.attention_full_aligned(qd, kd, vd, grid, cube, qg, kg, vg, gg, 0.3)
        mask = torch.from_numpy(aligned_mask(grid, cube, gg))
        q = torch.from_numpy(np.concatenate([qd, qg])).permute(1, 0, 2)
        k = torch.from_numpy(np.concatenate([kd, kg])).permute(1, 0, 2)
        v = torch.from_numpy(np.concatenate([vd, vg])).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k, v, attn_mask=mask, scale=0.3).permute(1, 0, 2).numpy()
        assert np.max(np.abs(ref - np.concatenate([od, og]))) < 1e-12, (grid, cube, gg)
        logits = np.where(mask.numpy()[None], (q @ k.transpose(1, 2)).numpy() * 0.3, -np.inf)
        mx = logits.max(-1, keepdims=True)
        ref_lse = (mx + np.log(np.exp(logits - mx).sum(-1, keepdims=True)))[..., 0]
        assert np.max(np.abs(ref_lse - lse)) < 1e-12, (grid, cube, gg)


def pin_attention_aligned_counts(o):
    """K = 0: LSE = log(number of allowed keys). Along an axis of E detail
    and e global tokens, the global indices whose scaled position g*E/e lies
    in [a, a+x) number ceil((a+x)*e/E) - ceil(a*e/E)."""
    for ci, (grid, cube, gg) in enumerate(ALIGNED_CASES):
        G, heads, D = gg[0] * gg[1] * gg[2], 1, 8
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 410 + ci)
        kd[:] = 0.0
        kg[:] = 0.0
        _, _, lse = o.attention_full_aligned(qd, kd, vd, grid, cube, qg, kg, vg, gg, 0.7)
        order = lexsort_order(grid, cube)
        n_allowed = np.empty(N)
        for j, r in enumerate(order):
            coords = (r // (grid[1] * grid[2]), (r // grid[2]) % grid[1], r % grid[2])
            n_det, n_glob = 1, 1
            for x, E, c, e in zip(coords, grid, cube, gg):
                a = (x // c) * c
                ext = min(c, E - a)
                n_det *= ext
                n_glob *= -(-(a + ext) * e // E) - -(-a * e // E)
            n_allowed[j] = n_det + n_glob
        assert np.max(np.abs(lse[0, :N] - np.log(n_allowed))) < 1e-12, (grid, cube, gg)
        assert np.max(np.abs(lse[0, N:] - math.log(G))) < 1e-12


def pin_attention_aligned_one_cube_sees_all(o):
    """A single cube covering the volume is aligned with every global token:
    the aligned variant equals the all-global-keys one."""
    grid, gg, heads, D = (2, 4, 6), (1, 2, 3), 2, 16
    G = 6
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 420)
    a = o.attention_full_aligned(qd, kd, vd, grid, grid, qg, kg, vg, gg, 0.25)
    b = o.attention_full(qd, kd, vd, N, qg, kg, vg, 0.25)
    for x, y in zip(a, b):
        assert np.max(np.abs(x - y)) < 1e-12


# ---------------------------------------------------------------------------
# Backward
# ---------------------------------------------------------------------------

def _autograd_grads(mask, qd, kd, vd, qg, kg, vg, dod, dog, scale):
    """torch autograd (float64) of dense masked attention, loss = <dO, O>."""
    ts = [torch.from_numpy(np.concatenate([a, b])).permute(1, 0, 2).clone().requires_grad_(True)
          for a, b in ((qd, qg), (kd, kg), (vd, vg))]
    out = torch.nn.functional.scaled_dot_product_attention(
        *ts, attn_mask=torch.from_numpy(mask), scale=scale)
    dout = torch.from_numpy(np.concatenate([dod, dog])).permute(1, 0, 2)
    (out * dout).sum().backward()
    N = qd.shape[0]
    grads = [t.grad.permute(1, 0, 2).numpy() for t in ts]
    return [g[:N] for g in grads] + [g[N:] for g in grads]


def pin_bwd_autograd_dense(o):
    """Gradients equal torch autograd of dense masked attention (explicit
    boolean masks built from coordinates), for fixed windows, partial cubes
    and the aligned variant."""
    cases = []
    for ci, (grid, cube, G, heads, D) in enumerate(ATTN_CASES[:4]):
        cases.append(("fixed", grid, cube, G, None, heads, D, geometric_mask(grid, cube, G)))
    for grid, cube in PARTIAL_CASES[:2]:
        T, H, W = grid
        order = lexsort_order(grid, cube)
        key = np.stack([order // (H * W) // cube[0], (order // W) % H // cube[1],
                        order % W // cube[2]], -1)
        N, G = T * H * W, 5
        m = np.zeros((N + G, N + G), dtype=bool)
        m[:N, :N] = np.all(key[:, None] == key[None], -1)
        m[:N, N:] = True
        m[N:, N:] = True
        cases.append(("partial", grid, cube, G, None, 2, 8, m))
    for grid, cube, gg in ALIGNED_CASES[:3]:
        cases.append(("aligned", grid, cube, gg[0] * gg[1] * gg[2], gg, 2, 8,
                      aligned_mask(grid, cube, gg)))
    for ci, (kind, grid, cube, G, gg, heads, D, mask) in enumerate(cases):
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 500 + ci)
        dod = _rand_case(grid, G, heads, D, 600 + ci)[1]
        dog = _rand_case(grid, G, heads, D, 700 + ci)[4]
        if kind == "fixed":
            got = o.attention_bwd_full(qd, kd, vd, cube[0] * cube[1] * cube[2], qg, kg, vg, dod,
                                       dog, 0.4)
        elif kind == "partial":
            got = o.attention_bwd_full(qd, kd, vd, 1, qg, kg, vg, dod, dog, 0.4,
                                       win_off=o.cube_windows(grid, cube))
        else:
            got = o.attention_bwd_full_aligned(qd, kd, vd, grid, cube, qg, kg, vg, gg, dod, dog,
                                               0.4)
        ref = _autograd_grads(mask, qd, kd, vd, qg, kg, vg, dod, dog, 0.4)
        for name, a, b in zip(("dq_d", "dk_d", "dv_d", "dq_g", "dk_g", "dv_g"), got, ref):
            assert np.max(np.abs(a - b), initial=0.0) < 1e-11, (kind, grid, name)


def pin_bwd_finite_differences(o):
    """Central differences of <dO, O> through the FORWARD oracle agree with
    the backward oracle (fixed windows and aligned variant)."""
    rng = np.random.default_rng(7)
    for kind in ("fixed", "aligned"):
        grid, cube, gg = (2, 4, 4), (1, 2, 2), (2, 2, 2)
        G, heads, D = 8, 1, 4
        N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 800)
        dod = rng.standard_normal(qd.shape)
        dog = rng.standard_normal(qg.shape)
        scale = 0.45

        def loss(ts):
            if kind == "fixed":
                od, og, _ = o.attention_full(ts[0], ts[1], ts[2], 4, ts[3], ts[4], ts[5], scale)
            else:
                od, og, _ = o.attention_full_aligned(ts[0], ts[1], ts[2], grid, cube, ts[3],
                                                     ts[4], ts[5], gg, scale)
            return float(np.sum(od * dod) + np.sum(og * dog))
        base = [qd, kd, vd, qg, kg, vg]
        if kind == "fixed":
            grads = o.attention_bwd_full(qd, kd, vd, 4, qg, kg, vg, dod, dog, scale)
        else:
            grads = o.attention_bwd_full_aligned(qd, kd, vd, grid, cube, qg, kg, vg, gg, dod,
                                                 dog, scale)
        order = [0, 1, 2, 3, 4, 5]   # grads come as (dq_d, dk_d, dv_d, dq_g, dk_g, dv_g)
        h = 1e-6
        for t_idx, g_idx in zip(order, order):
            for _ in range(6):
                idx = tuple(int(rng.integers(0, n)) for n in base[t_idx].shape)
                plus = [b.copy() for b in base]
                minus = [b.copy() for b in base]
                plus[t_idx][idx] += h
                minus[t_idx][idx] -= h
                fd = (loss(plus) - loss(minus)) / (2 * h)
                an = grads[g_idx][idx]
                assert abs(fd - an) < 1e-7 * max(1.0, abs(an)), (kind, t_idx, idx, fd, an)


def pin_bwd_single_token_windows(o):
    """1x1x1 cubes, G = 0: O = V, so dV = dO exactly and dQ = dK = 0."""
    grid, heads, D = (2, 3, 4), 2, 8
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, 0, heads, D, 810)
    dod = _rand_case(grid, 0, heads, D, 811)[1]
    dqd, dkd, dvd, _, _, _ = o.attention_bwd_full(qd, kd, vd, 1, qg, kg, vg, dod, qg, 0.5)
    assert np.array_equal(dvd, dod)
    assert np.max(np.abs(dqd)) < 1e-14 and np.max(np.abs(dkd)) < 1e-14


# ---------------------------------------------------------------------------
# Projections around the path
# ---------------------------------------------------------------------------

def pin_proj_matches_loops(o):
    """QKV projection + RoPE + reorder equals plain loops: each output
    element a dot product of one x row with one w row, pairs rotated by the
    literal angle p*theta^(-2k/d) of the token's axis position, the row
    placed at its lexsort cube position."""
    rng = np.random.default_rng(9)
    grid, cube, heads, hd, C = (2, 3, 2), (2, 2, 1), 2, 4, 5
    split, scales, theta = (2, 0, 2), (1.5, 1.0, 2.0), 100.0
    T, H, W = grid
    n = T * H * W
    x = rng.standard_normal((2 * n, C))            # two problems
    w = rng.standard_normal((3 * heads * hd, C))
    q, k, v = o.qkv_proj_reorder(x, w, grid, cube, heads, hd, theta, split, scales)
    order = lexsort_order(grid, cube)
    for b in range(2):
        for j in range(n):
            r = int(order[j])
            t_, h_, w_ = r // (H * W), (r // W) % H, r % W
            for which, got in enumerate((q, k, v)):
                for hh in range(heads):
                    vals = [sum(x[b * n + r, c] * w[which * heads * hd + hh * hd + d, c]
                                for c in range(C)) for d in range(hd)]
                    if which < 2:
                        off = 0
                        for pos, dd, sc in ((t_, split[0], scales[0]), (h_, split[1], scales[1]),
                                            (w_, split[2], scales[2])):
                            for kk in range(dd // 2):
                                ang = pos * sc * theta ** (-2.0 * kk / dd)
                                a0, a1 = vals[off + 2 * kk], vals[off + 2 * kk + 1]
                                vals[off + 2 * kk] = a0 * math.cos(ang) - a1 * math.sin(ang)
                                vals[off + 2 * kk + 1] = a0 * math.sin(ang) + a1 * math.cos(ang)
                            off += dd
                    assert np.max(np.abs(got[b * n + j, hh] - np.array(vals))) < 1e-12


def pin_out_proj_matches_loops(o):
    """Output projection of cube-ordered rows equals the raster row's plain
    dot products (the row a cube position holds goes back to its token)."""
    rng = np.random.default_rng(10)
    grid, cube, hdim, C = (3, 2, 3), (2, 2, 2), 6, 4
    n = 18
    oc = rng.standard_normal((n, hdim))
    w = rng.standard_normal((C, hdim))
    y = o.out_proj_unorder(oc, w, grid, cube)
    order = lexsort_order(grid, cube)
    for j in range(n):
        r = int(order[j])
        for c in range(C):
            assert abs(y[r, c] - sum(oc[j, e] * w[c, e] for e in range(hdim))) < 1e-12


PROJ_PINS = [pin_proj_matches_loops, pin_out_proj_matches_loops]

def pin_bwd_sampled_equals_full(o):
    """Selected rows of the backward equal the same rows of the full one."""
    grid, cube, G, heads, D = (2, 4, 8), (1, 2, 4), 11, 1, 8
    N, qd, kd, vd, qg, kg, vg = _rand_case(grid, G, heads, D, 820)
    dod = _rand_case(grid, G, heads, D, 821)[1]
    dog = _rand_case(grid, G, heads, D, 822)[4]
    full = o.attention_bwd_full(qd, kd, vd, 8, qg, kg, vg, dod, dog, 0.3)
    cat = lambda a, b: np.concatenate([a[:, 0], b[:, 0]])
    rows = np.array([0, 5, 17, N - 1, N, N + G - 1])
    dq, dk, dv = o.attention_bwd_sampled(cat(qd, qg), cat(kd, kg), cat(vd, vg), cat(dod, dog),
                                         N, 8, 0.3, rows, rows[::-1])
    for got, a, b, sel in ((dq, full[0], full[3], rows), (dk, full[1], full[4], rows[::-1]),
                           (dv, full[2], full[5], rows[::-1])):
        ref = cat(a, b)[sel]
        assert np.max(np.abs(got - ref)) < 1e-13


BWD_PINS = [pin_bwd_autograd_dense, pin_bwd_finite_differences, pin_bwd_single_token_windows,
            pin_bwd_sampled_equals_full]

ATTN_PINS = [pin_attention_dense_sdpa, pin_attention_partial_cubes_dense_sdpa,
             pin_attention_aligned_dense_sdpa, pin_attention_aligned_counts,
             pin_attention_aligned_one_cube_sees_all,
             pin_attention_offsets_equal_fixed_windows, pin_attention_full_when_one_cube,
             pin_attention_single_token_windows, pin_attention_zero_keys_mean,
             pin_attention_rows_sum_to_one, pin_attention_global_ignores_detail,
             pin_attention_probe_mass, pin_attention_rejects_missing_rows]

ALL_PINS = CUBE_PINS + ROPE_PINS + ATTN_PINS + BWD_PINS + PROJ_PINS
