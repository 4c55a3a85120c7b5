// permute_rope.cu -- cube reorder / unorder and 3D RoPE: one row-gather pass.
//
// Passages: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie
// 1, Fase 2 (tokens of one spatiotemporal cube made contiguous), Fase 1
// (temporal RoPE index times r_t) and Methodologie 2, position alignment
// (global RoPE coordinates times the resolution ratios).
//
// The pass is HBM-bound: every destination row (heads*head_dim elements,
// 10 KB for 40 heads x 128 bf16) is one contiguous read of its source row and
// one contiguous write. Each group of threads (32, 64 or 128 by row size)
// owns one row at a time; a
// thread owns a fixed 16-byte slot of the head (so its RoPE pairs, and hence
// its cos/sin table entries, are the same for every head of the row) and
// moves that slot for heads hg, hg + G/vph, ... with all loads of a row in
// flight before the first store. Row index arithmetic (cube <-> raster) is
// done once per row per thread with multiply-shift division (the index math
// itself is in cube_geom.cuh). A batch of problems of one grid is one launch:
// output row rr belongs to problem rr / (T*H*W) and is permuted inside it.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "atlas_internal.cuh"
#include "cube_geom.cuh"

namespace atlas {
namespace {

using geom::FastDiv;
using geom::Geom;
using geom::raster_coords;
using geom::cube_position;
using geom::cube_coords;
using geom::cube_position_general;
using geom::cube_coords_general;

struct Params {
    const uint8_t *src;
    uint8_t *dst;
    uint32_t rows;          // tokens of one problem
    uint32_t total_rows;    // tokens of all problems (batch * rows)
    FastDiv by_rows;
    uint32_t row_vecs;      // 16-byte vectors per row
    uint32_t vph;           // 16-byte vectors per head (power of two <= 128)
    uint32_t heads;
    Geom g;
    const float2 *tab;      // RoPE cos/sin table, NULL without RoPE
    uint32_t tab_base[3];   // first entry of each axis section
    uint32_t half[3];       // d_axis / 2 for t, h, w
};

constexpr int kThreads = 256;     // row groups of G threads per block (G = 128 or 32)
constexpr int kMaxInFlight = 8;   // 16-byte loads in flight per thread per row

__device__ __forceinline__ uint4 ld_stream(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Coherent streaming load, for the in-place RoPE pass (src may equal dst).
__device__ __forceinline__ uint4 ld_stream_coherent(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint8_t *p, const uint4 &v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Rotate the pairs of one 16-byte vector. bf16: 4 pairs, fp32: 2 pairs.
template <int EB>
__device__ __forceinline__ uint4 rotate(uint4 v, const float2 *cs);

template <>
__device__ __forceinline__ uint4 rotate<2>(uint4 v, const float2 *cs) {
    uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        float x0 = __uint_as_float(u[p] << 16);
        float x1 = __uint_as_float(u[p] & 0xffff0000u);
        float c = cs[p].x, s = cs[p].y;
        float y0 = fmaf(x0, c, -(x1 * s));
        float y1 = fmaf(x0, s, x1 * c);
        __nv_bfloat162 b = __floats2bfloat162_rn(y0, y1);  // .x = y0 (low half)
        u[p] = *reinterpret_cast<uint32_t *>(&b);
    }
    return make_uint4(u[0], u[1], u[2], u[3]);
}

template <>
__device__ __forceinline__ uint4 rotate<4>(uint4 v, const float2 *cs) {
    float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                  __uint_as_float(v.w)};
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        float x0 = f[2 * p], x1 = f[2 * p + 1];
        float c = cs[p].x, s = cs[p].y;
        f[2 * p] = fmaf(x0, c, -(x1 * s));
        f[2 * p + 1] = fmaf(x0, s, x1 * c);
    }
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}

// MODE 0: dst in cube order, src raster (reorder). MODE 1: dst raster, src
// cube order (unorder). MODE 2: dst and src raster (RoPE only). MODE 3 / 4:
// as 0 / 1 for grids the cube does not divide (partial cubes). MODE 5 / 6:
// as 0 / 1 with the aligned order of global-proxy tokens (cube_geom.cuh). With ROPE the
// row is rotated for the grid position (t, h, w) of its token, in every mode
// (unorder + rotation with negated scales is the transpose of reorder +
// rotation, i.e. its gradient).
template <int EB, bool ROPE, int MODE, int G>
__global__ void __launch_bounds__(kThreads) permute_rope_kernel(const Params p) {
    constexpr int kGroup = G;
    constexpr uint32_t kGroups = kThreads / G;    // rows in flight per block
    constexpr int kPairs = 16 / EB / 2;  // RoPE pairs in one 16-byte vector
    const uint32_t tid = threadIdx.x & (kGroup - 1);
    const uint32_t group = threadIdx.x / kGroup;
    const uint64_t row_bytes = static_cast<uint64_t>(p.row_vecs) * 16u;

    // This thread's fixed slot within a head, and its pairs' table layout.
    const uint32_t slot = ROPE ? tid % p.vph : 0;
    const uint32_t hg = ROPE ? tid / p.vph : 0;
    const uint32_t n_hg = ROPE ? kGroup / p.vph : 0;
    uint32_t pair_axis[kPairs], pair_off[kPairs], pair_stride[kPairs];
    if (ROPE) {
#pragma unroll
        for (int q = 0; q < kPairs; ++q) {
            uint32_t P = slot * kPairs + q;  // pair index within the head
            uint32_t a = P < p.half[0] ? 0u : (P < p.half[0] + p.half[1] ? 1u : 2u);
            uint32_t k = a == 0 ? P : (a == 1 ? P - p.half[0] : P - p.half[0] - p.half[1]);
            pair_axis[q] = a;
            pair_off[q] = (a == 0 ? p.tab_base[0] : (a == 1 ? p.tab_base[1] : p.tab_base[2])) + k;
            pair_stride[q] = a == 0 ? p.half[0] : (a == 1 ? p.half[1] : p.half[2]);
        }
    }

    for (uint32_t rr = blockIdx.x * kGroups + group; rr < p.total_rows;
         rr += gridDim.x * kGroups) {
        // Problem b of the batch, and the row within it.
        const uint32_t b = p.by_rows.div(rr);
        const uint32_t row = rr - b * p.rows;
        uint32_t t = 0, h = 0, w = 0, src_row;
        if (MODE == 0) {
            cube_coords(p.g, row, t, h, w);
            src_row = (t * p.g.H + h) * p.g.W + w;
        } else if (MODE == 1) {
            raster_coords(p.g, row, t, h, w);
            src_row = cube_position(p.g, t, h, w);
        } else if (MODE == 3) {
            cube_coords_general(p.g, row, t, h, w);
            src_row = (t * p.g.H + h) * p.g.W + w;
        } else if (MODE == 4) {
            raster_coords(p.g, row, t, h, w);
            src_row = cube_position_general(p.g, t, h, w);
        } else if (MODE == 5) {
            geom::aligned_coords(p.g, row, t, h, w);
            src_row = (t * p.g.H + h) * p.g.W + w;
        } else if (MODE == 6) {
            raster_coords(p.g, row, t, h, w);
            src_row = geom::aligned_position(p.g, t, h, w);
        } else {
            raster_coords(p.g, row, t, h, w);
            src_row = row;
        }
        const uint8_t *s =
            p.src + (static_cast<uint64_t>(b) * p.rows + src_row) * row_bytes;
        uint8_t *d = p.dst + static_cast<uint64_t>(rr) * row_bytes;

        if (!ROPE) {
            for (uint32_t v0 = tid; v0 < p.row_vecs; v0 += kGroup * kMaxInFlight) {
                uint4 buf[kMaxInFlight];
#pragma unroll
                for (int i = 0; i < kMaxInFlight; ++i) {
                    uint32_t v = v0 + i * kGroup;
                    if (v < p.row_vecs) buf[i] = ld_stream(s + v * 16u);
                }
#pragma unroll
                for (int i = 0; i < kMaxInFlight; ++i) {
                    uint32_t v = v0 + i * kGroup;
                    if (v < p.row_vecs) st_stream(d + v * 16u, buf[i]);
                }
            }
        } else {
            float2 cs[kPairs];
#pragma unroll
            for (int q = 0; q < kPairs; ++q) {
                const uint32_t c = pair_axis[q] == 0 ? t : (pair_axis[q] == 1 ? h : w);
                cs[q] = __ldg(p.tab + pair_off[q] + c * pair_stride[q]);
            }
            for (uint32_t h0 = hg; h0 < p.heads; h0 += n_hg * kMaxInFlight) {
                uint4 buf[kMaxInFlight];
#pragma unroll
                for (int i = 0; i < kMaxInFlight; ++i) {
                    uint32_t hd = h0 + i * n_hg;
                    if (hd < p.heads) {
                        const uint8_t *a = s + (hd * p.vph + slot) * 16u;
                        buf[i] = MODE == 2 ? ld_stream_coherent(a) : ld_stream(a);
                    }
                }
#pragma unroll
                for (int i = 0; i < kMaxInFlight; ++i) {
                    uint32_t hd = h0 + i * n_hg;
                    if (hd < p.heads)
                        st_stream(d + (hd * p.vph + slot) * 16u, rotate<EB>(buf[i], cs));
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// RoPE table: fp64 angles rounded to fp32 cos/sin, cached per device.
// Layout: axis t entries [t][k] (k < d_t/2), then axis h [h][k], then w.
// ---------------------------------------------------------------------------
using TableKey = std::tuple<int, int64_t, int64_t, int64_t, int32_t, int32_t, int32_t,
                            uint64_t, uint64_t, uint64_t, uint64_t>;
std::mutex g_tab_mutex;
std::map<TableKey, float2 *> g_tables;

uint64_t bits_of(double v) {
    uint64_t b;
    std::memcpy(&b, &v, sizeof b);
    return b;
}

atlas_status rope_table(int device, int64_t T, int64_t H, int64_t W, const atlas_rope &r,
                        float2 **out) {
    TableKey key{device, T, H, W, r.d_t, r.d_h, r.d_w, bits_of(r.theta), bits_of(r.scale_t),
                 bits_of(r.scale_h), bits_of(r.scale_w)};
    std::lock_guard<std::mutex> lock(g_tab_mutex);
    auto it = g_tables.find(key);
    if (it != g_tables.end()) {
        *out = it->second;
        return ATLAS_OK;
    }
    const int64_t ext[3] = {T, H, W};
    const int32_t width[3] = {r.d_t, r.d_h, r.d_w};
    const double scale[3] = {r.scale_t, r.scale_h, r.scale_w};
    std::vector<float2> host;
    for (int a = 0; a < 3; ++a) {
        for (int64_t c = 0; c < ext[a]; ++c) {
            for (int32_t k = 0; k < width[a] / 2; ++k) {
                double omega = std::pow(r.theta, -2.0 * k / static_cast<double>(width[a]));
                double phi = (static_cast<double>(c) * scale[a]) * omega;
                host.push_back(make_float2(static_cast<float>(std::cos(phi)),
                                           static_cast<float>(std::sin(phi))));
            }
        }
    }
    if (host.empty()) host.push_back(make_float2(1.f, 0.f));
    float2 *dev = nullptr;
    if (cudaMalloc(&dev, host.size() * sizeof(float2)) != cudaSuccess) return ATLAS_ERR_CUDA;
    if (cudaMemcpy(dev, host.data(), host.size() * sizeof(float2), cudaMemcpyHostToDevice) !=
        cudaSuccess) {
        cudaFree(dev);
        return ATLAS_ERR_CUDA;
    }
    g_tables.emplace(key, dev);
    *out = dev;
    return ATLAS_OK;
}

template <int EB, bool ROPE, int MODE, int G>
atlas_status launch_g(const Params &p, const DeviceInfo &dev, cudaStream_t stream) {
    constexpr uint32_t kGroups = kThreads / G;
    uint32_t blocks_needed = (p.total_rows + kGroups - 1) / kGroups;
    uint32_t grid = std::min<uint32_t>(blocks_needed, static_cast<uint32_t>(dev.sm_count) * 8u);
    if (grid == 0) return ATLAS_OK;
    if (log_enabled())
        log_launch("permute_rope_kernel", static_cast<int>(grid), kThreads, 0,
                   "mode %d rope %d elem_bytes %d row_group %d rows %u row_bytes %u", MODE,
                   ROPE ? 1 : 0, EB, G, p.total_rows, p.row_vecs * 16u);
    permute_rope_kernel<EB, ROPE, MODE, G><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

// Group width by row size, so that a thread keeps several 16-byte loads in
// flight: 128-thread groups for rows above 8 KB (5 loads per thread at 40
// heads x 128 bf16), 64 threads up to 8 KB, 32 up to 4 KB (8 rows per block).
// RoPE needs a head's vectors to fit the group.
template <int EB, bool ROPE, int MODE>
atlas_status launch(const Params &p, const DeviceInfo &dev, cudaStream_t stream) {
    if (p.row_vecs <= 256 && p.vph <= 32) return launch_g<EB, ROPE, MODE, 32>(p, dev, stream);
    if (p.row_vecs <= 512 && p.vph <= 64) return launch_g<EB, ROPE, MODE, 64>(p, dev, stream);
    return launch_g<EB, ROPE, MODE, 128>(p, dev, stream);
}

// mode: 0 reorder, 1 unorder, 2 raster RoPE; `general` selects the
// partial-cube index arithmetic for reorder and unorder.
template <int EB>
atlas_status dispatch(const Params &p, bool rope, int mode, bool general, const DeviceInfo &dev,
                      cudaStream_t stream) {
    if (mode == 5 || mode == 6) {   // aligned order of global tokens
        if (rope)
            return mode == 5 ? launch<EB, true, 5>(p, dev, stream)
                             : launch<EB, true, 6>(p, dev, stream);
        return mode == 5 ? launch<EB, false, 5>(p, dev, stream)
                         : launch<EB, false, 6>(p, dev, stream);
    }
    if (rope) {
        if (mode == 2) return launch<EB, true, 2>(p, dev, stream);
        if (mode == 1)
            return general ? launch<EB, true, 4>(p, dev, stream)
                           : launch<EB, true, 1>(p, dev, stream);
        return general ? launch<EB, true, 3>(p, dev, stream) : launch<EB, true, 0>(p, dev, stream);
    }
    if (mode == 0)
        return general ? launch<EB, false, 3>(p, dev, stream) : launch<EB, false, 0>(p, dev, stream);
    return general ? launch<EB, false, 4>(p, dev, stream) : launch<EB, false, 1>(p, dev, stream);
}

// ---------------------------------------------------------------------------
// Variant that allocates nothing (atlas_cube_reorder_noalloc): the cos/sin
// table lives in a fixed file-scope device array instead of a cached
// cudaMalloc'd buffer. Every call on a device shares the array, so calls that
// overlap on the GPU (e.g. on two streams) race on its contents.
// ---------------------------------------------------------------------------
constexpr size_t kStaticRopeEntries = 32768;  // 256 KB of (cos, sin) per device
static __device__ __align__(256) float2 g_static_rope_table[kStaticRopeEntries];

std::mutex g_static_mutex;                      // guards the arrays below
float2 g_static_host_table[kStaticRopeEntries];  // host staging, reused per call
float2 *g_static_table_dev[64] = {nullptr};      // device address, per device

// What the array of each device was last filled with (grid extents and
// RoPE): a call with the same ones skips the host fill and the copy.
struct StaticTableKey {
    bool valid = false;
    int64_t T = 0, H = 0, W = 0;
    atlas_rope rope{};
    bool same(int64_t t, int64_t h, int64_t w, const atlas_rope &r) const {
        return valid && T == t && H == h && W == w && rope.theta == r.theta &&
               rope.d_t == r.d_t && rope.d_h == r.d_h && rope.d_w == r.d_w &&
               rope.scale_t == r.scale_t && rope.scale_h == r.scale_h &&
               rope.scale_w == r.scale_w;
    }
};
StaticTableKey g_static_key[64];

// Device address of the static table on `device` (the current device). The
// array's name is only a host-side stand-in; its address is resolved once per
// device with that device current. Caller holds g_static_mutex.
atlas_status static_table_address(int device, float2 **out) {
    if (device < 0 || device >= 64) return ATLAS_ERR_DEVICE;
    if (g_static_table_dev[device] == nullptr) {
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_static_rope_table) != cudaSuccess)
            return ATLAS_ERR_CUDA;
        g_static_table_dev[device] = static_cast<float2 *>(addr);
    }
    *out = g_static_table_dev[device];
    return ATLAS_OK;
}

size_t rope_table_entries(int64_t T, int64_t H, int64_t W, const atlas_rope &r) {
    return static_cast<size_t>(T) * (r.d_t / 2) + static_cast<size_t>(H) * (r.d_h / 2) +
           static_cast<size_t>(W) * (r.d_w / 2);
}

// Same layout and arithmetic as the cached table (fp64 angles, rounded once).
void fill_rope_table(float2 *out, int64_t T, int64_t H, int64_t W, const atlas_rope &r) {
    const int64_t ext[3] = {T, H, W};
    const int32_t width[3] = {r.d_t, r.d_h, r.d_w};
    const double scale[3] = {r.scale_t, r.scale_h, r.scale_w};
    size_t n = 0;
    for (int a = 0; a < 3; ++a)
        for (int64_t c = 0; c < ext[a]; ++c)
            for (int32_t k = 0; k < width[a] / 2; ++k) {
                double omega = std::pow(r.theta, -2.0 * k / static_cast<double>(width[a]));
                double phi = (static_cast<double>(c) * scale[a]) * omega;
                out[n++] = make_float2(static_cast<float>(std::cos(phi)),
                                       static_cast<float>(std::sin(phi)));
            }
}

void fill_geometry(Params &p, const PermuteArgs &a) {
    p.src = static_cast<const uint8_t *>(a.src);
    p.dst = static_cast<uint8_t *>(a.dst);
    p.rows = static_cast<uint32_t>(a.T * a.H * a.W);
    p.total_rows = static_cast<uint32_t>(a.batch * a.T * a.H * a.W);
    p.by_rows = FastDiv(p.rows);
    p.heads = static_cast<uint32_t>(a.heads);
    p.row_vecs = static_cast<uint32_t>(static_cast<int64_t>(a.heads) * a.head_dim *
                                       a.elem_bytes / 16);
    p.vph = static_cast<uint32_t>(a.head_dim * a.elem_bytes / 16);
    p.g = geom::make_geom(static_cast<uint32_t>(a.T), static_cast<uint32_t>(a.H),
                          static_cast<uint32_t>(a.W), static_cast<uint32_t>(a.ct),
                          static_cast<uint32_t>(a.ch), static_cast<uint32_t>(a.cw));
    p.g.DT = static_cast<uint32_t>(a.DT);
    p.g.DH = static_cast<uint32_t>(a.DH);
    p.g.DW = static_cast<uint32_t>(a.DW);
}

}  // namespace

atlas_status launch_permute_rope(const PermuteArgs &a, cudaStream_t stream) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    Params p{};
    fill_geometry(p, a);
    const bool rope = a.rope != nullptr;
    if (rope) {
        float2 *tab = nullptr;
        atlas_status st = rope_table(dev.device, a.T, a.H, a.W, *a.rope, &tab);
        if (st != ATLAS_OK) return st;
        p.tab = tab;
        p.half[0] = static_cast<uint32_t>(a.rope->d_t / 2);
        p.half[1] = static_cast<uint32_t>(a.rope->d_h / 2);
        p.half[2] = static_cast<uint32_t>(a.rope->d_w / 2);
        p.tab_base[0] = 0;
        p.tab_base[1] = static_cast<uint32_t>(a.T) * p.half[0];
        p.tab_base[2] = p.tab_base[1] + static_cast<uint32_t>(a.H) * p.half[1];
    }
    const bool general = (a.T % a.ct) || (a.H % a.ch) || (a.W % a.cw);
    if (a.elem_bytes == 2) return dispatch<2>(p, rope, a.mode, general, dev, stream);
    return dispatch<4>(p, rope, a.mode, general, dev, stream);
}

atlas_status rope_table_for(int64_t T, int64_t H, int64_t W, const atlas_rope &rope,
                            const float2 **out) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    float2 *tab = nullptr;
    atlas_status st = rope_table(dev.device, T, H, W, rope, &tab);
    *out = tab;
    return st;
}

int64_t cached_rope_tables() {
    std::lock_guard<std::mutex> lock(g_tab_mutex);
    return static_cast<int64_t>(g_tables.size());
}

atlas_status release_rope_tables() {
    std::lock_guard<std::mutex> lock(g_tab_mutex);
    atlas_status st = ATLAS_OK;
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto &kv : g_tables) {
        cudaSetDevice(std::get<0>(kv.first));
        if (cudaDeviceSynchronize() != cudaSuccess) st = ATLAS_ERR_CUDA;
        if (cudaFree(kv.second) != cudaSuccess) st = ATLAS_ERR_CUDA;
    }
    g_tables.clear();
    cudaSetDevice(cur);
    return st;
}

atlas_status launch_permute_rope_noalloc(const PermuteArgs &a, cudaStream_t stream) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    Params p{};
    fill_geometry(p, a);
    const bool general = (a.T % a.ct) || (a.H % a.ch) || (a.W % a.cw);
    if (a.rope == nullptr) {
        if (a.elem_bytes == 2) return dispatch<2>(p, false, 0, general, dev, stream);
        return dispatch<4>(p, false, 0, general, dev, stream);
    }
    const atlas_rope &r = *a.rope;
    const size_t n = rope_table_entries(a.T, a.H, a.W, r);
    if (n > kStaticRopeEntries) return ATLAS_ERR_CAPACITY;
    std::lock_guard<std::mutex> lock(g_static_mutex);
    float2 *tab = nullptr;
    atlas_status st = static_table_address(dev.device, &tab);
    if (st != ATLAS_OK) return st;
    StaticTableKey &key = g_static_key[dev.device];
    if (!key.same(a.T, a.H, a.W, r)) {
        key.valid = false;
        fill_rope_table(g_static_host_table, a.T, a.H, a.W, r);
        // From pageable host memory: returns once the staging copy is taken,
        // so the host buffer may be refilled by the next call; ordered on
        // `stream` before the kernel.
        if (n > 0 && cudaMemcpyAsync(tab, g_static_host_table, n * sizeof(float2),
                                     cudaMemcpyHostToDevice, stream) != cudaSuccess)
            return ATLAS_ERR_CUDA;
        key.valid = true;
        key.T = a.T;
        key.H = a.H;
        key.W = a.W;
        key.rope = r;
    }
    p.tab = tab;
    p.half[0] = static_cast<uint32_t>(r.d_t / 2);
    p.half[1] = static_cast<uint32_t>(r.d_h / 2);
    p.half[2] = static_cast<uint32_t>(r.d_w / 2);
    p.tab_base[0] = 0;
    p.tab_base[1] = static_cast<uint32_t>(a.T) * p.half[0];
    p.tab_base[2] = p.tab_base[1] + static_cast<uint32_t>(a.H) * p.half[1];
    if (a.elem_bytes == 2) return dispatch<2>(p, true, 0, general, dev, stream);
    return dispatch<4>(p, true, 0, general, dev, stream);
}

}  // namespace atlas
