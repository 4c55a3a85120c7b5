// atlas_api.cu -- the C-ABI of libatlas.so: argument validation and dispatch.
//
// Every entry point checks its arguments on the host and returns a status
// without launching anything when they are bad. See include/atlas.h for the
// contract of each call and the passages it implements.
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "atlas_internal.cuh"
#include "cube_geom.cuh"

namespace atlas {

namespace {
bool env_flag(const char *name) {
    const char *v = std::getenv(name);
    return v != nullptr && v[0] != '\0' && std::strcmp(v, "0") != 0;
}
}  // namespace

bool log_enabled() {
    static const bool on = env_flag("ATLAS_LOG");
    return on;
}

TraceScope::TraceScope(const char *name) {
    static const bool nvtx = env_flag("ATLAS_NVTX");
    on = nvtx;
    if (on) nvtxRangePushA(name);
}

TraceScope::~TraceScope() {
    if (on) nvtxRangePop();
}

void log_launch(const char *kernel, int grid, int block, size_t smem, const char *fmt, ...) {
    if (!log_enabled()) return;
    char detail[256];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(detail, sizeof detail, fmt, ap);
    va_end(ap);
    int dev = -1;
    cudaGetDevice(&dev);
    std::fprintf(stderr, "[atlas] dev %d %s grid %d block %d smem %zu %s\n", dev, kernel, grid,
                 block, smem, detail);
}

__device__ uint32_t g_device_error = 0;

uint32_t *device_error_word() {
    static std::mutex mu;
    static uint32_t *addr[64] = {nullptr};
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<uint32_t *>(p);
    }
    return addr[dev];
}

namespace {
std::atomic<int> g_stall_request{0};
}  // namespace

bool take_stall_request() { return g_stall_request.exchange(0) != 0; }

bool current_device(DeviceInfo *out) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo &c = cache[dev];
    if (c.device != dev) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return false;
        c.device = dev;
        c.sm_count = prop.multiProcessorCount;
        c.major = prop.major;
        c.minor = prop.minor;
        c.smem_optin = prop.sharedMemPerBlockOptin;
    }
    *out = c;
    return c.major == 10 && c.minor == 0;
}

bool set_smem_limit(const void *func, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void *>> done;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({dev, func})) return true;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    done.insert({dev, func});
    return true;
}

namespace {

int elem_bytes(atlas_dtype dt) {
    switch (dt) {
        case ATLAS_BF16: return 2;
        case ATLAS_FP32: return 4;
    }
    return 0;
}

// Row-index arithmetic in the kernels is 32-bit: the token count and every
// intermediate index stay below 2^31.
constexpr int64_t kMaxRows = (1ll << 31) - 1;

atlas_status check_grid(atlas_grid3 g, int32_t heads, int32_t head_dim, atlas_dtype dt) {
    if (g.T < 1 || g.H < 1 || g.W < 1 || heads < 1 || head_dim < 1) return ATLAS_ERR_SHAPE;
    if (g.T > kMaxRows || g.H > kMaxRows || g.W > kMaxRows) return ATLAS_ERR_SHAPE;
    if (g.T * g.H > kMaxRows || g.T * g.H * g.W > kMaxRows) return ATLAS_ERR_SHAPE;
    const int eb = elem_bytes(dt);
    if (eb == 0) return ATLAS_ERR_UNSUPPORTED;
    if ((static_cast<int64_t>(head_dim) * eb) % 16 != 0) return ATLAS_ERR_ALIGN;
    return ATLAS_OK;
}

// A cube that does not divide the grid leaves partial cubes at the far edges.
atlas_status check_cube(atlas_grid3 g, atlas_cube3 c) {
    (void)g;
    if (c.ct < 1 || c.ch < 1 || c.cw < 1) return ATLAS_ERR_SHAPE;
    return ATLAS_OK;
}

atlas_status check_rope(const atlas_rope &r, int32_t head_dim, atlas_dtype dt) {
    if (r.d_t < 0 || r.d_h < 0 || r.d_w < 0) return ATLAS_ERR_UNSUPPORTED;
    if ((r.d_t | r.d_h | r.d_w) & 1) return ATLAS_ERR_UNSUPPORTED;
    if (r.d_t + r.d_h + r.d_w != head_dim) return ATLAS_ERR_UNSUPPORTED;
    if (!(r.theta > 0.0) || !std::isfinite(r.theta)) return ATLAS_ERR_UNSUPPORTED;
    if (!std::isfinite(r.scale_t) || !std::isfinite(r.scale_h) || !std::isfinite(r.scale_w))
        return ATLAS_ERR_UNSUPPORTED;
    // The kernel gives each thread one 16-byte slot of a head: the slots of a
    // head must tile a 128-thread group.
    const int vph = head_dim * elem_bytes(dt) / 16;
    if (vph < 1 || vph > 128 || (vph & (vph - 1))) return ATLAS_ERR_UNSUPPORTED;
    return ATLAS_OK;
}

}  // namespace
}  // namespace atlas

using namespace atlas;

namespace atlas {
namespace {

// Shared validation of the permutation entry points; `bytes` receives the
// size of one tensor (all problems).
atlas_status check_permute(const void *src, const void *dst, int64_t batch, atlas_grid3 grid,
                           int32_t heads, int32_t head_dim, atlas_dtype dtype, size_t *bytes) {
    if (!src || !dst) return ATLAS_ERR_NULL;
    atlas_status st = check_grid(grid, heads, head_dim, dtype);
    if (st != ATLAS_OK) return st;
    if (batch < 1 || batch > kMaxRows || grid.T * grid.H * grid.W > kMaxRows / batch)
        return ATLAS_ERR_SHAPE;
    if (!aligned16(src) || !aligned16(dst)) return ATLAS_ERR_ALIGN;
    *bytes = static_cast<size_t>(batch * grid.T * grid.H * grid.W) * heads * head_dim *
             elem_bytes(dtype);
    return ATLAS_OK;
}

atlas_status reorder(const void *src, void *dst, int64_t batch, atlas_grid3 grid,
                     atlas_cube3 cube, int32_t heads, int32_t head_dim, atlas_dtype dtype,
                     const atlas_rope *rope, atlas_stream_t stream, bool noalloc) {
    size_t bytes = 0;
    atlas_status st = check_permute(src, dst, batch, grid, heads, head_dim, dtype, &bytes);
    if (st != ATLAS_OK) return st;
    if ((st = check_cube(grid, cube)) != ATLAS_OK) return st;
    if (rope && (st = check_rope(*rope, head_dim, dtype)) != ATLAS_OK) return st;
    if (ranges_overlap(src, bytes, dst, bytes)) return ATLAS_ERR_ALIAS;
    PermuteArgs a{src, dst, grid.T, grid.H, grid.W, cube.ct, cube.ch, cube.cw,
                  heads, head_dim, elem_bytes(dtype), 0, rope, batch};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return noalloc ? launch_permute_rope_noalloc(a, s) : launch_permute_rope(a, s);
}

atlas_status unorder(const void *src, void *dst, int64_t batch, atlas_grid3 grid,
                     atlas_cube3 cube, int32_t heads, int32_t head_dim, atlas_dtype dtype,
                     const atlas_rope *rope, atlas_stream_t stream) {
    size_t bytes = 0;
    atlas_status st = check_permute(src, dst, batch, grid, heads, head_dim, dtype, &bytes);
    if (st != ATLAS_OK) return st;
    if ((st = check_cube(grid, cube)) != ATLAS_OK) return st;
    if (rope && (st = check_rope(*rope, head_dim, dtype)) != ATLAS_OK) return st;
    if (ranges_overlap(src, bytes, dst, bytes)) return ATLAS_ERR_ALIAS;
    PermuteArgs a{src, dst, grid.T, grid.H, grid.W, cube.ct, cube.ch, cube.cw,
                  heads, head_dim, elem_bytes(dtype), 1, rope, batch};
    return launch_permute_rope(a, reinterpret_cast<cudaStream_t>(stream));
}

atlas_status rope3d(const void *src, void *dst, int64_t batch, atlas_grid3 grid, int32_t heads,
                    int32_t head_dim, atlas_dtype dtype, const atlas_rope *rope,
                    atlas_stream_t stream) {
    if (!rope) return ATLAS_ERR_NULL;
    size_t bytes = 0;
    atlas_status st = check_permute(src, dst, batch, grid, heads, head_dim, dtype, &bytes);
    if (st != ATLAS_OK) return st;
    if ((st = check_rope(*rope, head_dim, dtype)) != ATLAS_OK) return st;
    if (src != dst && ranges_overlap(src, bytes, dst, bytes)) return ATLAS_ERR_ALIAS;
    PermuteArgs a{src, dst, grid.T, grid.H, grid.W, 1, 1, 1,
                  heads, head_dim, elem_bytes(dtype), 2, rope, batch};
    return launch_permute_rope(a, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace atlas

ATLAS_API atlas_status atlas_cube_reorder(const void *src, void *dst, atlas_grid3 grid,
                                          atlas_cube3 cube, int32_t heads, int32_t head_dim,
                                          atlas_dtype dtype, const atlas_rope *rope,
                                          atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::reorder(src, dst, 1, grid, cube, heads, head_dim, dtype, rope, stream, false);
}

ATLAS_API atlas_status atlas_cube_reorder_noalloc(const void *src, void *dst, atlas_grid3 grid,
                                                  atlas_cube3 cube, int32_t heads,
                                                  int32_t head_dim, atlas_dtype dtype,
                                                  const atlas_rope *rope,
                                                  atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::reorder(src, dst, 1, grid, cube, heads, head_dim, dtype, rope, stream, true);
}

ATLAS_API atlas_status atlas_cube_unorder(const void *src, void *dst, atlas_grid3 grid,
                                          atlas_cube3 cube, int32_t heads, int32_t head_dim,
                                          atlas_dtype dtype, atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::unorder(src, dst, 1, grid, cube, heads, head_dim, dtype, nullptr, stream);
}

ATLAS_API atlas_status atlas_rope3d(const void *src, void *dst, atlas_grid3 grid, int32_t heads,
                                    int32_t head_dim, atlas_dtype dtype, const atlas_rope *rope,
                                    atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::rope3d(src, dst, 1, grid, heads, head_dim, dtype, rope, stream);
}

ATLAS_API atlas_status atlas_cube_reorder_batched(const void *src, void *dst, int64_t batch,
                                                  atlas_grid3 grid, atlas_cube3 cube,
                                                  int32_t heads, int32_t head_dim,
                                                  atlas_dtype dtype, const atlas_rope *rope,
                                                  atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::reorder(src, dst, batch, grid, cube, heads, head_dim, dtype, rope, stream,
                          false);
}

ATLAS_API atlas_status atlas_cube_unorder_batched(const void *src, void *dst, int64_t batch,
                                                  atlas_grid3 grid, atlas_cube3 cube,
                                                  int32_t heads, int32_t head_dim,
                                                  atlas_dtype dtype, atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::unorder(src, dst, batch, grid, cube, heads, head_dim, dtype, nullptr, stream);
}

namespace atlas {
namespace {

// Reorder to (mode 5) or from (mode 6) the aligned order of global tokens.
atlas_status aligned_perm(const void *src, void *dst, int64_t batch, atlas_grid3 grid,
                          atlas_cube3 cube, atlas_grid3 gg, int32_t heads, int32_t head_dim,
                          atlas_dtype dtype, const atlas_rope *rope, atlas_stream_t stream,
                          int mode) {
    size_t bytes = 0;
    atlas_status st = check_permute(src, dst, batch, gg, heads, head_dim, dtype, &bytes);
    if (st != ATLAS_OK) return st;
    if (grid.T < 1 || grid.H < 1 || grid.W < 1 || grid.T > kMaxRows || grid.H > kMaxRows ||
        grid.W > kMaxRows)
        return ATLAS_ERR_SHAPE;
    if ((st = check_cube(grid, cube)) != ATLAS_OK) return st;
    if (rope && (st = check_rope(*rope, head_dim, dtype)) != ATLAS_OK) return st;
    if (ranges_overlap(src, bytes, dst, bytes)) return ATLAS_ERR_ALIAS;
    PermuteArgs a{src, dst, gg.T, gg.H, gg.W, cube.ct, cube.ch, cube.cw,
                  heads, head_dim, elem_bytes(dtype), mode, rope, batch,
                  grid.T, grid.H, grid.W};
    return launch_permute_rope(a, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace atlas

ATLAS_API atlas_status atlas_aligned_global_reorder(const void *src, void *dst, int64_t batch,
                                                    atlas_grid3 grid, atlas_cube3 cube,
                                                    atlas_grid3 global_grid, int32_t heads,
                                                    int32_t head_dim, atlas_dtype dtype,
                                                    const atlas_rope *rope,
                                                    atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::aligned_perm(src, dst, batch, grid, cube, global_grid, heads, head_dim, dtype,
                               rope, stream, 5);
}

ATLAS_API atlas_status atlas_aligned_global_unorder(const void *src, void *dst, int64_t batch,
                                                    atlas_grid3 grid, atlas_cube3 cube,
                                                    atlas_grid3 global_grid, int32_t heads,
                                                    int32_t head_dim, atlas_dtype dtype,
                                                    const atlas_rope *rope,
                                                    atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::aligned_perm(src, dst, batch, grid, cube, global_grid, heads, head_dim, dtype,
                               rope, stream, 6);
}

ATLAS_API atlas_status atlas_aligned_global_offsets(atlas_grid3 grid, atlas_cube3 cube,
                                                    atlas_grid3 global_grid, int32_t *offsets,
                                                    int64_t capacity, int64_t *n_windows) {
    ATLAS_TRACE();
    if (!n_windows) return ATLAS_ERR_NULL;
    if (grid.T < 1 || grid.H < 1 || grid.W < 1 || cube.ct < 1 || cube.ch < 1 || cube.cw < 1 ||
        global_grid.T < 1 || global_grid.H < 1 || global_grid.W < 1)
        return ATLAS_ERR_SHAPE;
    if (grid.T > kMaxRows || grid.H > kMaxRows || grid.W > kMaxRows ||
        global_grid.T * global_grid.H * global_grid.W > kMaxRows)
        return ATLAS_ERR_SHAPE;
    auto n_along = [](int64_t e, int64_t c) { return (e + c - 1) / c; };
    const int64_t nt = n_along(grid.T, cube.ct), nh = n_along(grid.H, cube.ch),
                  nw = n_along(grid.W, cube.cw);
    *n_windows = nt * nh * nw;
    if (!offsets) return ATLAS_OK;   // size query
    if (capacity < *n_windows + 1) return ATLAS_ERR_CAPACITY;
    using atlas::geom::box_start;
    const uint32_t T = static_cast<uint32_t>(global_grid.T), H = static_cast<uint32_t>(global_grid.H),
                   W = static_cast<uint32_t>(global_grid.W);
    const uint32_t DT = static_cast<uint32_t>(grid.T), DH = static_cast<uint32_t>(grid.H),
                   DW = static_cast<uint32_t>(grid.W);
    int64_t n = 0;
    for (uint32_t bt = 0; bt < nt; ++bt)
        for (uint32_t bh = 0; bh < nh; ++bh)
            for (uint32_t bw = 0; bw < nw; ++bw) {
                const uint32_t st = box_start(bt, T, DT, cube.ct), sh = box_start(bh, H, DH, cube.ch),
                               sw = box_start(bw, W, DW, cube.cw);
                const uint32_t et = box_start(bt + 1, T, DT, cube.ct) - st;
                const uint32_t eh = box_start(bh + 1, H, DH, cube.ch) - sh;
                offsets[n++] = static_cast<int32_t>(st * H * W + et * sh * W + et * eh * sw);
            }
    offsets[n] = static_cast<int32_t>(static_cast<int64_t>(T) * H * W);
    return ATLAS_OK;
}

ATLAS_API atlas_status atlas_cube_unorder_rope(const void *src, void *dst, int64_t batch,
                                               atlas_grid3 grid, atlas_cube3 cube,
                                               int32_t heads, int32_t head_dim,
                                               atlas_dtype dtype, const atlas_rope *rope,
                                               atlas_stream_t stream) {
    ATLAS_TRACE();
    if (!rope) return ATLAS_ERR_NULL;
    return atlas::unorder(src, dst, batch, grid, cube, heads, head_dim, dtype, rope, stream);
}

ATLAS_API atlas_status atlas_rope3d_batched(const void *src, void *dst, int64_t batch,
                                            atlas_grid3 grid, int32_t heads, int32_t head_dim,
                                            atlas_dtype dtype, const atlas_rope *rope,
                                            atlas_stream_t stream) {
    ATLAS_TRACE();
    return atlas::rope3d(src, dst, batch, grid, heads, head_dim, dtype, rope, stream);
}

namespace atlas {
namespace {

// Shared validation of the attention entry points: sizes, windows, dtype
// and the alignment of the six inputs. Fills `a` (outputs left empty);
// *bd / *bg receive the bytes of one detail / global tensor (all problems).
atlas_status attn_layout(const void *q_d, const void *k_d, const void *v_d, int64_t n_detail,
                         const void *q_g, const void *k_g, const void *v_g, int64_t n_global,
                         const atlas_attn_layout &ly, int32_t heads, int32_t head_dim,
                         float softmax_scale, atlas_dtype dtype, AttnArgs *a, size_t *bd,
                         size_t *bg) {
    if (n_detail < 0 || n_global < 0 || heads < 1 || ly.batch < 1) return ATLAS_ERR_SHAPE;
    if (ly.batch > kMaxRows || n_detail > kMaxRows / ly.batch ||
        n_global > kMaxRows / ly.batch || static_cast<int64_t>(heads) > 65535)
        return ATLAS_ERR_SHAPE;
    int64_t window_len = ly.window_len, n_win = 0;
    const int32_t *win_off = n_detail > 0 ? ly.window_offsets : nullptr;
    const int32_t *gwin_off = n_detail > 0 ? ly.global_window_offsets : nullptr;
    if (n_detail > 0) {
        if (win_off == nullptr) {
            if (window_len < 1 || n_detail % window_len != 0) return ATLAS_ERR_SHAPE;
            n_win = n_detail / window_len;
            if (gwin_off && ly.n_windows != n_win) return ATLAS_ERR_SHAPE;
        } else {
            n_win = ly.n_windows;
            if (n_win < 1 || n_win > n_detail) return ATLAS_ERR_SHAPE;
            if (reinterpret_cast<uintptr_t>(win_off) & 3u) return ATLAS_ERR_ALIGN;
            window_len = 1;
        }
        if (gwin_off && (reinterpret_cast<uintptr_t>(gwin_off) & 3u)) return ATLAS_ERR_ALIGN;
    } else {
        window_len = 1;
    }
    if (n_detail > 0 && (!q_d || !k_d || !v_d)) return ATLAS_ERR_NULL;
    if (n_global > 0 && (!q_g || !k_g || !v_g)) return ATLAS_ERR_NULL;
    if (elem_bytes(dtype) == 0) return ATLAS_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return ATLAS_ERR_UNSUPPORTED;
    const void *ptrs[] = {q_d, k_d, v_d, q_g, k_g, v_g};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return ATLAS_ERR_ALIGN;
    const size_t eb = static_cast<size_t>(elem_bytes(dtype)) * heads * head_dim;
    *bd = eb * static_cast<size_t>(n_detail * ly.batch);
    *bg = eb * static_cast<size_t>(n_global * ly.batch);
    float scale = softmax_scale > 0.f ? softmax_scale
                                      : 1.f / std::sqrt(static_cast<float>(head_dim));
    *a = AttnArgs{q_d, k_d, v_d, n_detail, window_len, q_g, k_g, v_g, n_global,
                  heads, head_dim, scale, nullptr, nullptr, nullptr, win_off,
                  win_off ? n_win : 0, ly.batch, gwin_off, n_win};
    return ATLAS_OK;
}

// A buffer of `bytes` at `p` (NULL or empty: nothing) overlaps none of `n`
// others.
struct Span {
    const void *p;
    size_t bytes;
};
bool overlaps_any(const Span &x, const Span *others, int n) {
    if (!x.p || !x.bytes) return false;
    for (int i = 0; i < n; ++i)
        if (others[i].p && others[i].bytes && &others[i] != &x &&
            ranges_overlap(x.p, x.bytes, others[i].p, others[i].bytes))
            return true;
    return false;
}

atlas_status local_global_attn(const void *q_d, const void *k_d, const void *v_d,
                               int64_t n_detail, const void *q_g, const void *k_g,
                               const void *v_g, int64_t n_global, const atlas_attn_layout &ly,
                               int32_t heads, int32_t head_dim, float softmax_scale,
                               atlas_dtype dtype, void *o_d, void *o_g, float *lse,
                               atlas_stream_t stream) {
    AttnArgs a;
    size_t bd = 0, bg = 0;
    atlas_status st = attn_layout(q_d, k_d, v_d, n_detail, q_g, k_g, v_g, n_global, ly, heads,
                                  head_dim, softmax_scale, dtype, &a, &bd, &bg);
    if (st != ATLAS_OK) return st;
    if ((n_detail > 0 && !o_d) || (n_global > 0 && !o_g)) return ATLAS_ERR_NULL;
    if ((o_d && !aligned16(o_d)) || (o_g && !aligned16(o_g))) return ATLAS_ERR_ALIGN;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return ATLAS_ERR_ALIGN;
    // Outputs must not overlap inputs or each other.
    const Span all[] = {{q_d, bd}, {k_d, bd}, {v_d, bd}, {q_g, bg}, {k_g, bg}, {v_g, bg},
                        {o_d, bd}, {o_g, bg}};
    if (overlaps_any(all[6], all, 8) || overlaps_any(all[7], all, 8)) return ATLAS_ERR_ALIAS;
    if (n_detail + n_global == 0) return ATLAS_OK;
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    a.o_d = o_d;
    a.o_g = o_g;
    a.lse = lse;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return dtype == ATLAS_BF16 ? launch_attn_tc_bf16(a, s) : launch_attn_simt_f32(a, s);
}

atlas_status local_global_attn_bwd(const void *const in_d[5], int64_t n_detail,
                                   const void *const in_g[5], int64_t n_global,
                                   const atlas_attn_layout &ly, int32_t heads, int32_t head_dim,
                                   float softmax_scale, atlas_dtype dtype, const float *lse,
                                   float *delta, void *const grad_d[3], void *const grad_g[3],
                                   atlas_stream_t stream) {
    // in_*: q, k, v, o, do; grad_*: dq, dk, dv.
    AttnArgs a;
    size_t bd = 0, bg = 0;
    atlas_status st = attn_layout(in_d[0], in_d[1], in_d[2], n_detail, in_g[0], in_g[1],
                                  in_g[2], n_global, ly, heads, head_dim, softmax_scale, dtype,
                                  &a, &bd, &bg);
    if (st != ATLAS_OK) return st;
    if (!lse || !delta) return ATLAS_ERR_NULL;
    for (int i = 3; i < 5; ++i) {
        if ((n_detail > 0 && !in_d[i]) || (n_global > 0 && !in_g[i])) return ATLAS_ERR_NULL;
        if ((in_d[i] && !aligned16(in_d[i])) || (in_g[i] && !aligned16(in_g[i])))
            return ATLAS_ERR_ALIGN;
    }
    for (int i = 0; i < 3; ++i) {
        if ((n_detail > 0 && !grad_d[i]) || (n_global > 0 && !grad_g[i])) return ATLAS_ERR_NULL;
        if ((grad_d[i] && !aligned16(grad_d[i])) || (grad_g[i] && !aligned16(grad_g[i])))
            return ATLAS_ERR_ALIGN;
    }
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(delta) & 3u))
        return ATLAS_ERR_ALIGN;
    const size_t bl = sizeof(float) * static_cast<size_t>(ly.batch) * heads *
                      static_cast<size_t>(n_detail + n_global);
    Span all[17];
    int n = 0;
    for (int i = 0; i < 5; ++i) all[n++] = {in_d[i], bd};
    for (int i = 0; i < 5; ++i) all[n++] = {in_g[i], bg};
    all[n++] = {lse, bl};
    all[n++] = {delta, bl};   // index 11
    for (int i = 0; i < 3; ++i) all[n++] = {grad_d[i], bd};
    for (int i = 0; i < 2; ++i) all[n++] = {grad_g[i], bg};
    Span dv_g{grad_g[2], bg};
    // Written buffers (delta, the gradients) overlap nothing else.
    for (int i = 11; i < n; ++i)
        if (overlaps_any(all[i], all, n) || overlaps_any(all[i], &dv_g, 1))
            return ATLAS_ERR_ALIAS;
    if (overlaps_any(dv_g, all, n)) return ATLAS_ERR_ALIAS;
    if (n_detail + n_global == 0) return ATLAS_OK;
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    a.o_d = const_cast<void *>(in_d[3]);
    a.o_g = const_cast<void *>(in_g[3]);
    a.lse = const_cast<float *>(lse);
    AttnBwdArgs b{a, in_d[4], in_g[4], delta, grad_d[0], grad_d[1], grad_d[2],
                  grad_g[0], grad_g[1], grad_g[2], elem_bytes(dtype)};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = launch_attn_bwd_delta(b, s)) != ATLAS_OK) return st;
    return dtype == ATLAS_BF16 ? launch_attn_bwd_tc_bf16(b, s) : launch_attn_bwd_simt_f32(b, s);
}

}  // namespace
}  // namespace atlas

ATLAS_API atlas_status atlas_local_global_attn(const void *q_d, const void *k_d, const void *v_d,
                                               int64_t n_detail, int64_t window_len,
                                               const void *q_g, const void *k_g, const void *v_g,
                                               int64_t n_global, int32_t heads, int32_t head_dim,
                                               float softmax_scale, atlas_dtype dtype, void *o_d,
                                               void *o_g, float *lse, atlas_stream_t stream) {
    ATLAS_TRACE();
    atlas_attn_layout ly{1, window_len, nullptr, 0, nullptr};
    return atlas::local_global_attn(q_d, k_d, v_d, n_detail, q_g, k_g, v_g, n_global, ly, heads,
                                    head_dim, softmax_scale, dtype, o_d, o_g, lse, stream);
}

ATLAS_API atlas_status atlas_local_global_attn_windows(
    const void *q_d, const void *k_d, const void *v_d, int64_t n_detail,
    const int32_t *window_offsets, int64_t n_windows, const void *q_g, const void *k_g,
    const void *v_g, int64_t n_global, int32_t heads, int32_t head_dim, float softmax_scale,
    atlas_dtype dtype, void *o_d, void *o_g, float *lse, atlas_stream_t stream) {
    ATLAS_TRACE();
    if (n_detail > 0 && window_offsets == nullptr) return ATLAS_ERR_NULL;
    atlas_attn_layout ly{1, 1, window_offsets, n_windows, nullptr};
    return atlas::local_global_attn(q_d, k_d, v_d, n_detail, q_g, k_g, v_g, n_global, ly, heads,
                                    head_dim, softmax_scale, dtype, o_d, o_g, lse, stream);
}

ATLAS_API atlas_status atlas_local_global_attn_ex(
    const void *q_d, const void *k_d, const void *v_d, int64_t n_detail, const void *q_g,
    const void *k_g, const void *v_g, int64_t n_global, const atlas_attn_layout *layout,
    int32_t heads, int32_t head_dim, float softmax_scale, atlas_dtype dtype, void *o_d,
    void *o_g, float *lse, atlas_stream_t stream) {
    ATLAS_TRACE();
    if (!layout) return ATLAS_ERR_NULL;
    return atlas::local_global_attn(q_d, k_d, v_d, n_detail, q_g, k_g, v_g, n_global, *layout,
                                    heads, head_dim, softmax_scale, dtype, o_d, o_g, lse, stream);
}

ATLAS_API atlas_status atlas_local_global_attn_bwd(
    const void *q_d, const void *k_d, const void *v_d, const void *o_d, const void *do_d,
    int64_t n_detail, const void *q_g, const void *k_g, const void *v_g, const void *o_g,
    const void *do_g, int64_t n_global, const atlas_attn_layout *layout, int32_t heads,
    int32_t head_dim, float softmax_scale, atlas_dtype dtype, const float *lse, float *delta,
    void *dq_d, void *dk_d, void *dv_d, void *dq_g, void *dk_g, void *dv_g,
    atlas_stream_t stream) {
    ATLAS_TRACE();
    if (!layout) return ATLAS_ERR_NULL;
    const void *in_d[5] = {q_d, k_d, v_d, o_d, do_d};
    const void *in_g[5] = {q_g, k_g, v_g, o_g, do_g};
    void *gd[3] = {dq_d, dk_d, dv_d};
    void *gg[3] = {dq_g, dk_g, dv_g};
    return atlas::local_global_attn_bwd(in_d, n_detail, in_g, n_global, *layout, heads,
                                        head_dim, softmax_scale, dtype, lse, delta, gd, gg,
                                        stream);
}

namespace atlas {
namespace {

// Shared checks of the two projection entry points.
atlas_status check_proj(const void *x, const void *w, int64_t batch, atlas_grid3 grid,
                        atlas_cube3 cube, int32_t c_in, atlas_dtype dtype) {
    if (!x || !w) return ATLAS_ERR_NULL;
    if (grid.T < 1 || grid.H < 1 || grid.W < 1 || batch < 1 || c_in < 1) return ATLAS_ERR_SHAPE;
    if (grid.T > kMaxRows || grid.H > kMaxRows || grid.W > kMaxRows ||
        grid.T * grid.H > kMaxRows || grid.T * grid.H * grid.W > kMaxRows / batch)
        return ATLAS_ERR_SHAPE;
    atlas_status st = check_cube(grid, cube);
    if (st != ATLAS_OK) return st;
    if (dtype != ATLAS_BF16 || c_in % 64 != 0) return ATLAS_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w)) return ATLAS_ERR_ALIGN;
    return ATLAS_OK;
}

}  // namespace
}  // namespace atlas

ATLAS_API atlas_status atlas_qkv_proj_reorder(const void *x, const void *w, int64_t batch,
                                              atlas_grid3 grid, atlas_cube3 cube, int32_t c_in,
                                              int32_t heads, int32_t head_dim, atlas_dtype dtype,
                                              const atlas_rope *rope, void *q, void *k, void *v,
                                              atlas_stream_t stream) {
    ATLAS_TRACE();
    atlas_status st = atlas::check_proj(x, w, batch, grid, cube, c_in, dtype);
    if (st != ATLAS_OK) return st;
    if (!q || !k || !v) return ATLAS_ERR_NULL;
    if (heads < 1 || head_dim < 1) return ATLAS_ERR_SHAPE;
    if (head_dim % 32 != 0 || (static_cast<int64_t>(heads) * head_dim) % 256 != 0 ||
        static_cast<int64_t>(heads) * head_dim * 3 > (1ll << 30))
        return ATLAS_ERR_UNSUPPORTED;
    if (rope && (st = atlas::check_rope(*rope, head_dim, dtype)) != ATLAS_OK) return st;
    if (!atlas::aligned16(q) || !atlas::aligned16(k) || !atlas::aligned16(v)) return ATLAS_ERR_ALIGN;
    const size_t rows = static_cast<size_t>(batch * grid.T * grid.H * grid.W);
    const size_t bx = rows * c_in * 2, bw = static_cast<size_t>(3) * heads * head_dim * c_in * 2;
    const size_t bo = rows * heads * head_dim * 2;
    const atlas::Span all[] = {{x, bx}, {w, bw}, {q, bo}, {k, bo}, {v, bo}};
    for (int i = 2; i < 5; ++i)
        if (atlas::overlaps_any(all[i], all, 5)) return ATLAS_ERR_ALIAS;
    atlas::ProjArgs a{x, w, batch, grid.T, grid.H, grid.W, cube.ct, cube.ch, cube.cw, c_in, 0,
                      heads, head_dim, rope, {q, k, v}};
    return atlas::launch_qkv_proj(a, reinterpret_cast<cudaStream_t>(stream));
}

ATLAS_API atlas_status atlas_out_proj_unorder(const void *o, const void *w, int64_t batch,
                                              atlas_grid3 grid, atlas_cube3 cube, int32_t c_in,
                                              int32_t c_out, atlas_dtype dtype, void *y,
                                              atlas_stream_t stream) {
    ATLAS_TRACE();
    atlas_status st = atlas::check_proj(o, w, batch, grid, cube, c_in, dtype);
    if (st != ATLAS_OK) return st;
    if (!y) return ATLAS_ERR_NULL;
    if (c_out < 1) return ATLAS_ERR_SHAPE;
    if (c_out % 256 != 0) return ATLAS_ERR_UNSUPPORTED;
    if (!atlas::aligned16(y)) return ATLAS_ERR_ALIGN;
    const size_t rows = static_cast<size_t>(batch * grid.T * grid.H * grid.W);
    const atlas::Span all[] = {{o, rows * c_in * 2}, {w, static_cast<size_t>(c_out) * c_in * 2},
                               {y, rows * c_out * 2}};
    if (atlas::overlaps_any(all[2], all, 3)) return ATLAS_ERR_ALIAS;
    atlas::ProjArgs a{o, w, batch, grid.T, grid.H, grid.W, cube.ct, cube.ch, cube.cw, c_in,
                      c_out, 0, 0, nullptr, {y, nullptr, nullptr}};
    return atlas::launch_out_proj(a, reinterpret_cast<cudaStream_t>(stream));
}

ATLAS_API atlas_status atlas_aligned_global_cube(atlas_grid3 grid, atlas_cube3 cube,
                                                 atlas_grid3 global_grid,
                                                 atlas_cube3 *global_cube) {
    ATLAS_TRACE();
    if (!global_cube) return ATLAS_ERR_NULL;
    if (grid.T < 1 || grid.H < 1 || grid.W < 1 || global_grid.T < 1 || global_grid.H < 1 ||
        global_grid.W < 1 || cube.ct < 1 || cube.ch < 1 || cube.cw < 1)
        return ATLAS_ERR_SHAPE;
    const int64_t E[3] = {grid.T, grid.H, grid.W};
    const int64_t e[3] = {global_grid.T, global_grid.H, global_grid.W};
    const int64_t c[3] = {cube.ct, cube.ch, cube.cw};
    int32_t out[3];
    for (int i = 0; i < 3; ++i) {
        if (E[i] % e[i] != 0) return ATLAS_ERR_UNSUPPORTED;
        const int64_t r = E[i] / e[i];
        if (c[i] % r != 0) return ATLAS_ERR_UNSUPPORTED;
        out[i] = static_cast<int32_t>(c[i] / r);
    }
    *global_cube = atlas_cube3{out[0], out[1], out[2]};
    return ATLAS_OK;
}

ATLAS_API atlas_status atlas_cube_window_offsets(atlas_grid3 grid, atlas_cube3 cube,
                                                 int32_t *offsets, int64_t capacity,
                                                 int64_t *n_windows) {
    ATLAS_TRACE();
    if (!n_windows) return ATLAS_ERR_NULL;
    if (grid.T < 1 || grid.H < 1 || grid.W < 1 || cube.ct < 1 || cube.ch < 1 || cube.cw < 1)
        return ATLAS_ERR_SHAPE;
    if (grid.T * grid.H * grid.W > kMaxRows) return ATLAS_ERR_SHAPE;
    auto n_along = [](int64_t e, int64_t c) { return (e + c - 1) / c; };
    auto ext = [](int64_t e, int64_t c, int64_t b) { return (b + 1) * c <= e ? c : e - b * c; };
    const int64_t nt = n_along(grid.T, cube.ct), nh = n_along(grid.H, cube.ch),
                  nw = n_along(grid.W, cube.cw);
    *n_windows = nt * nh * nw;
    if (!offsets) return ATLAS_OK;  // size query
    if (capacity < *n_windows + 1) return ATLAS_ERR_CAPACITY;
    int64_t n = 0, pos = 0;
    for (int64_t bt = 0; bt < nt; ++bt)
        for (int64_t bh = 0; bh < nh; ++bh)
            for (int64_t bw = 0; bw < nw; ++bw) {
                offsets[n++] = static_cast<int32_t>(pos);
                pos += ext(grid.T, cube.ct, bt) * ext(grid.H, cube.ch, bh) *
                       ext(grid.W, cube.cw, bw);
            }
    offsets[n] = static_cast<int32_t>(pos);
    return ATLAS_OK;
}

ATLAS_API const char *atlas_status_string(atlas_status status) {
    switch (status) {
        case ATLAS_OK: return "ATLAS_OK";
        case ATLAS_ERR_NULL: return "ATLAS_ERR_NULL: a required pointer is NULL";
        case ATLAS_ERR_SHAPE: return "ATLAS_ERR_SHAPE: inconsistent sizes";
        case ATLAS_ERR_ALIGN: return "ATLAS_ERR_ALIGN: pointer or row not 16-byte aligned";
        case ATLAS_ERR_UNSUPPORTED: return "ATLAS_ERR_UNSUPPORTED: dtype, head_dim or RoPE split";
        case ATLAS_ERR_ALIAS: return "ATLAS_ERR_ALIAS: input and output overlap";
        case ATLAS_ERR_CUDA: return "ATLAS_ERR_CUDA: a CUDA call or launch failed";
        case ATLAS_ERR_TIMEOUT: return "ATLAS_ERR_TIMEOUT: a kernel's bounded wait expired";
        case ATLAS_ERR_DEVICE: return "ATLAS_ERR_DEVICE: no compute capability 10.0 device";
        case ATLAS_ERR_CAPACITY: return "ATLAS_ERR_CAPACITY: fixed internal buffer too small";
    }
    return "ATLAS_ERR_UNKNOWN";
}

ATLAS_API atlas_status atlas_last_device_error(atlas_stream_t stream, uint32_t *code) {
    ATLAS_TRACE();
    if (!code) return ATLAS_ERR_NULL;
    *code = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return ATLAS_ERR_CUDA;
    uint32_t v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return ATLAS_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess)
        return ATLAS_ERR_CUDA;
    *code = v;
    return v ? ATLAS_ERR_TIMEOUT : ATLAS_OK;
}

ATLAS_API atlas_status atlas_release_caches(void) {
    ATLAS_TRACE(); return release_rope_tables(); }

ATLAS_API int64_t atlas_cached_rope_tables(void) { return cached_rope_tables(); }

ATLAS_API atlas_status atlas_debug_stall_next_attention(void) {
    ATLAS_TRACE();
    g_stall_request.store(1);
    return ATLAS_OK;
}

ATLAS_API int32_t atlas_version(void) { return 100; }
