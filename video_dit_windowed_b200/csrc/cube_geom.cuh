// cube_geom.cuh -- token-grid index arithmetic of the cube order, shared by
// the gather kernel (permute_rope.cu) and the projection GEMM's epilogue
// (gemm_proj.cu).
//
// Passage: "Technische Samenvatting: AtlasVid", Methodologie 1, Fase 2 (the
// tokens of one spatiotemporal cube made contiguous). Raster index
// r = (t*H + h)*W + w; cubes in raster order over the cube grid, tokens of a
// cube in raster order over its extent; the last cube along an axis the cube
// does not divide is partial.
#pragma once

#include <stdint.h>

namespace atlas {
namespace geom {

// Unsigned division by a run-time constant for dividends below 2^31:
// q = (n * m) >> s with m = ceil(2^s / d), s = 31 + ceil(log2 d). For
// n < 2^31 the error term n*(m - 2^s/d)/2^s stays below 1/d, so the floor is
// exact.
struct FastDiv {
    uint64_t m = 1ull << 31;
    uint32_t s = 31;
    uint32_t d = 1;
    FastDiv() = default;
    explicit FastDiv(uint32_t div) : d(div) {
        if (div == 0) div = d = 1;  // never used for division by zero
        uint32_t l = 0;
        while ((1ull << l) < div) ++l;
        s = 31 + l;
        m = ((1ull << s) + div - 1) / div;
    }
    __host__ __device__ __forceinline__ uint32_t div(uint32_t n) const {
        return static_cast<uint32_t>((static_cast<uint64_t>(n) * m) >> s);
    }
};

struct Geom {
    uint32_t T, H, W, ct, ch, cw, cubes_h, cubes_w, L;
    FastDiv by_W, by_H, by_ct, by_ch, by_cw, by_cubes_w, by_cubes_h, by_L;
    // aligned order of a global grid (T x H x W here) against a detail grid
    // DT x DH x DW cut into ct x ch x cw cubes; 0 when unused
    uint32_t DT, DH, DW;
};

// Raster coordinates of a raster row.
__device__ __forceinline__ void raster_coords(const Geom &g, uint32_t r, uint32_t &t,
                                              uint32_t &h, uint32_t &w) {
    uint32_t tw = g.by_W.div(r);
    w = r - tw * g.W;
    t = g.by_H.div(tw);
    h = tw - t * g.H;
}

// Cube-order position of the token at (t, h, w).
__device__ __forceinline__ uint32_t cube_position(const Geom &g, uint32_t t, uint32_t h,
                                                  uint32_t w) {
    uint32_t bt = g.by_ct.div(t), bh = g.by_ch.div(h), bw = g.by_cw.div(w);
    uint32_t cube = (bt * g.cubes_h + bh) * g.cubes_w + bw;
    uint32_t local = ((t - bt * g.ct) * g.ch + (h - bh * g.ch)) * g.cw + (w - bw * g.cw);
    return cube * g.L + local;
}

// Raster coordinates of the token at cube-order position j.
__device__ __forceinline__ void cube_coords(const Geom &g, uint32_t j, uint32_t &t,
                                            uint32_t &h, uint32_t &w) {
    uint32_t cube = g.by_L.div(j);
    uint32_t local = j - cube * g.L;
    uint32_t c1 = g.by_cubes_w.div(cube);
    uint32_t bw = cube - c1 * g.cubes_w;
    uint32_t bt = g.by_cubes_h.div(c1);
    uint32_t bh = c1 - bt * g.cubes_h;
    uint32_t l1 = g.by_cw.div(local);
    uint32_t lw = local - l1 * g.cw;
    uint32_t lt = g.by_ch.div(l1);
    uint32_t lh = l1 - lt * g.ch;
    t = bt * g.ct + lt;
    h = bh * g.ch + lh;
    w = bw * g.cw + lw;
}

// Grids the cube does not divide: the last cube along such an axis is
// partial (keeps the tokens that exist) and stays contiguous. Tokens before
// cube (bt, bh, bw): the whole slabs of bt*ct frames, then bh cube rows of
// its slab, then bw cubes of its row; inside a cube, raster order over the
// cube's own extent. Plain 32-bit division: only this path needs it.
__device__ __forceinline__ uint32_t extent(uint32_t E, uint32_t c, uint32_t b) {
    return min(c, E - b * c);
}

__device__ __forceinline__ uint32_t cube_position_general(const Geom &g, uint32_t t,
                                                          uint32_t h, uint32_t w) {
    const uint32_t bt = t / g.ct, bh = h / g.ch, bw = w / g.cw;
    const uint32_t et = extent(g.T, g.ct, bt), eh = extent(g.H, g.ch, bh),
                   ew = extent(g.W, g.cw, bw);
    const uint32_t before = bt * g.ct * g.H * g.W + et * (bh * g.ch) * g.W + et * eh * (bw * g.cw);
    return before + ((t - bt * g.ct) * eh + (h - bh * g.ch)) * ew + (w - bw * g.cw);
}

__device__ __forceinline__ void cube_coords_general(const Geom &g, uint32_t j, uint32_t &t,
                                                    uint32_t &h, uint32_t &w) {
    const uint32_t slab = g.ct * g.H * g.W;
    const uint32_t bt = j / slab;
    uint32_t rem = j - bt * slab;
    const uint32_t et = extent(g.T, g.ct, bt);
    const uint32_t row = et * g.ch * g.W;
    const uint32_t bh = rem / row;
    rem -= bh * row;
    const uint32_t eh = extent(g.H, g.ch, bh);
    const uint32_t cube = et * eh * g.cw;
    const uint32_t bw = rem / cube;
    rem -= bw * cube;
    const uint32_t ew = extent(g.W, g.cw, bw);
    const uint32_t plane = eh * ew;
    const uint32_t lt = rem / plane;
    rem -= lt * plane;
    const uint32_t lh = rem / ew;
    t = bt * g.ct + lt;
    h = bh * g.ch + lh;
    w = bw * g.cw + (rem - lh * ew);
}

// ---------------------------------------------------------------------------
// Aligned order of the global-proxy tokens ("Technische Samenvatting:
// AtlasVid", Methodologie 2, position alignment): global index x of an axis
// of e tokens sits at detail position x*E/e of the detail axis of E tokens,
// and belongs to the detail cube (of c tokens) holding that point:
// box(x) = floor(x*E / (c*e)). Box b spans global indices
// [ceil(b*c*e/E), ceil((b+1)*c*e/E)) clamped to e (it may be empty), the boxes
// of an axis partition it, and a global token's box triple is the detail
// cube it is aligned with. The aligned order lists the tokens box by box in
// the cube grid's raster order, raster order inside a box: the cube order of
// the partial-cube case with these boundaries.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint32_t box_of(uint32_t x, uint32_t e, uint32_t E,
                                                   uint32_t c) {
    return static_cast<uint32_t>(static_cast<uint64_t>(x) * E / (static_cast<uint64_t>(c) * e));
}
__host__ __device__ __forceinline__ uint32_t box_start(uint32_t b, uint32_t e, uint32_t E,
                                                      uint32_t c) {
    const uint64_t v = (static_cast<uint64_t>(b) * c * e + E - 1) / E;
    return static_cast<uint32_t>(v < e ? v : e);
}

__device__ __forceinline__ uint32_t aligned_position(const Geom &g, uint32_t t, uint32_t h,
                                                     uint32_t w) {
    const uint32_t bt = box_of(t, g.T, g.DT, g.ct), bh = box_of(h, g.H, g.DH, g.ch),
                   bw = box_of(w, g.W, g.DW, g.cw);
    const uint32_t st = box_start(bt, g.T, g.DT, g.ct), sh = box_start(bh, g.H, g.DH, g.ch),
                   sw = box_start(bw, g.W, g.DW, g.cw);
    const uint32_t et = box_start(bt + 1, g.T, g.DT, g.ct) - st;
    const uint32_t eh = box_start(bh + 1, g.H, g.DH, g.ch) - sh;
    const uint32_t ew = box_start(bw + 1, g.W, g.DW, g.cw) - sw;
    const uint32_t before = st * g.H * g.W + et * sh * g.W + et * eh * sw;
    return before + ((t - st) * eh + (h - sh)) * ew + (w - sw);
}

// Inverse: the raster coordinates of the token at aligned position j. The
// t-slab of box bt holds positions [st*H*W, (st+et)*H*W), so j / (H*W) is a
// global t inside it; likewise along h and w within the slab.
__device__ __forceinline__ void aligned_coords(const Geom &g, uint32_t j, uint32_t &t,
                                               uint32_t &h, uint32_t &w) {
    const uint32_t bt = box_of(j / (g.H * g.W), g.T, g.DT, g.ct);
    const uint32_t st = box_start(bt, g.T, g.DT, g.ct);
    const uint32_t et = box_start(bt + 1, g.T, g.DT, g.ct) - st;
    uint32_t rem = j - st * g.H * g.W;
    const uint32_t bh = box_of(rem / (et * g.W), g.H, g.DH, g.ch);
    const uint32_t sh = box_start(bh, g.H, g.DH, g.ch);
    const uint32_t eh = box_start(bh + 1, g.H, g.DH, g.ch) - sh;
    rem -= et * sh * g.W;
    const uint32_t bw = box_of(rem / (et * eh), g.W, g.DW, g.cw);
    const uint32_t sw = box_start(bw, g.W, g.DW, g.cw);
    const uint32_t ew = box_start(bw + 1, g.W, g.DW, g.cw) - sw;
    rem -= et * eh * sw;
    const uint32_t plane = eh * ew;
    const uint32_t lt = rem / plane;
    rem -= lt * plane;
    const uint32_t lh = rem / ew;
    t = st + lt;
    h = sh + lh;
    w = sw + (rem - lh * ew);
}

// Host: the geometry of a T x H x W grid cut into ct x ch x cw cubes.
inline Geom make_geom(uint32_t T, uint32_t H, uint32_t W, uint32_t ct, uint32_t ch,
                      uint32_t cw) {
    Geom g;
    g.T = T;
    g.H = H;
    g.W = W;
    g.ct = ct;
    g.ch = ch;
    g.cw = cw;
    // (cube counts of the divisible path; at least 1 so the dividers stay
    // defined when a partial cube covers a whole axis)
    g.cubes_h = H / ch > 0 ? H / ch : 1;
    g.cubes_w = W / cw > 0 ? W / cw : 1;
    g.L = ct * ch * cw;
    g.by_W = FastDiv(W);
    g.by_H = FastDiv(H);
    g.by_ct = FastDiv(ct);
    g.by_ch = FastDiv(ch);
    g.by_cw = FastDiv(cw);
    g.by_cubes_w = FastDiv(g.cubes_w);
    g.by_cubes_h = FastDiv(g.cubes_h);
    g.by_L = FastDiv(g.L);
    g.DT = g.DH = g.DW = 0;
    return g;
}

}  // namespace geom
}  // namespace atlas
