// attn_bwd.cu -- backward of the asymmetric local-global attention: the
// delta pass (delta_i = <dO_i, O_i>, any dtype) and SIMT fp32 gradient
// kernels.
//
// Passages: "Technische Samenvatting: AtlasVid", Methodologie 2 (the
// asymmetric mask; training adapts the attention projections, which needs
// dQ, dK and dV). With P the row softmax of s = scale*<q,k> over the allowed
// keys and dO the gradient of the output:
//   dS_ij = P_ij (<dO_i, v_j> - delta_i),
//   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
//   dv_j = sum_i P_ij dO_i.
// The fp32 kernels serve the small fp32 workloads: one warp per (row, head),
// exact fp32 products, P recomputed from the forward's LSE. dQ walks a query
// row's allowed keys; dK and dV walk the queries allowed to see a key row:
// a detail key is seen by the queries of its own window; a global key by
// every detail query of its problem (or, in the aligned variant, by the
// queries of the one window whose global range holds it) and by every global
// query of its problem.
#include <cuda_bf16.h>

#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kWarps = 8;

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ int64_t clamp64(int64_t x, int64_t lo, int64_t hi) {
    return x < lo ? lo : (x > hi ? hi : x);
}

// Geometry shared by the kernels below (all counts per problem).
struct Geo {
    int64_t N, L, G, batch, n_win;
    int32_t heads;
    const int32_t *win_off, *gwin_off;
};

__device__ __forceinline__ int64_t window_of(const Geo &g, int64_t x) {
    if (g.win_off == nullptr) return x / g.L;
    int64_t a = 0, c = g.n_win - 1;
    while (a < c) {
        const int64_t mid = (a + c + 1) / 2;
        if (g.win_off[mid] <= x) a = mid; else c = mid - 1;
    }
    return a;
}
// Rows of window w (which holds x), clamped as the forward clamps them.
__device__ __forceinline__ void window_rows(const Geo &g, int64_t w, int64_t x, int64_t &lo,
                                            int64_t &hi) {
    if (g.win_off == nullptr) {
        lo = w * g.L;
        hi = lo + g.L;
    } else {
        lo = clamp64(g.win_off[w], 0, x);
        hi = clamp64(g.win_off[w + 1], x + 1, g.N);
    }
}
__device__ __forceinline__ void global_rows(const Geo &g, int64_t w, int64_t &lo, int64_t &hi) {
    if (g.gwin_off == nullptr) {
        lo = 0;
        hi = g.G;
    } else {
        lo = clamp64(g.gwin_off[w], 0, g.G);
        hi = clamp64(g.gwin_off[w + 1], lo, g.G);
    }
}

// ---------------------------------------------------------------------------
// delta_i = <dO_i, O_i>, fp32, for every row and head.
// ---------------------------------------------------------------------------
template <typename T, int HD>
__global__ void __launch_bounds__(kWarps * 32) delta_kernel(const T *o_d, const T *do_d,
                                                            const T *o_g, const T *do_g,
                                                            float *delta, Geo g) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + threadIdx.x / 32;
    const int head = blockIdx.y;
    const int64_t nd_all = g.batch * g.N;
    if (row >= nd_all + g.batch * g.G) return;
    const bool detail = row < nd_all;
    const int64_t b = detail ? row / g.N : (row - nd_all) / g.G;
    const int64_t local = detail ? row - b * g.N : row - nd_all - b * g.G;
    const int64_t off = ((detail ? row : row - nd_all) * g.heads + head) * HD;
    const T *o = (detail ? o_d : o_g) + off;
    const T *d = (detail ? do_d : do_g) + off;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) acc = fmaf(to_f(o[lane + 32 * e]), to_f(d[lane + 32 * e]), acc);
    acc = warp_sum(acc);
    if (lane == 0) delta[(b * g.heads + head) * (g.N + g.G) + (detail ? local : g.N + local)] = acc;
}

// ---------------------------------------------------------------------------
// fp32 dQ: one warp per (query row, head).
// ---------------------------------------------------------------------------
struct BwdPtr {
    const float *q_d, *k_d, *v_d, *do_d, *q_g, *k_g, *v_g, *do_g;
    const float *lse, *delta;
    float *dq_d, *dk_d, *dv_d, *dq_g, *dk_g, *dv_g;
    float scale;
};

template <int HD>
__device__ __forceinline__ void dq_keys(const float *k, const float *v, int64_t k0, int64_t k1,
                                        int64_t stride, const float (&q)[HD / 32],
                                        const float (&go)[HD / 32], float scale, float lse,
                                        float delta, float (&dq)[HD / 32]) {
    const int lane = threadIdx.x & 31;
    for (int64_t key = k0; key < k1; ++key) {
        const float *kr = k + key * stride, *vr = v + key * stride;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) {
            s = fmaf(q[e], kr[lane + 32 * e], s);
            dp = fmaf(go[e], vr[lane + 32 * e], dp);
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const float p = expf(s * scale - lse);
        const float ds = p * (dp - delta);
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) dq[e] = fmaf(ds, kr[lane + 32 * e], dq[e]);
    }
}

template <int HD>
__global__ void __launch_bounds__(kWarps * 32) dq_simt_kernel(const BwdPtr p, const Geo g) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + threadIdx.x / 32;
    const int head = blockIdx.y;
    const int64_t nd_all = g.batch * g.N;
    if (row >= nd_all + g.batch * g.G) return;
    const bool detail = row < nd_all;
    const int64_t b = detail ? row / g.N : (row - nd_all) / g.G;
    const int64_t local = detail ? row - b * g.N : row - nd_all - b * g.G;
    const int64_t stride = static_cast<int64_t>(g.heads) * HD;
    const int64_t off = (detail ? row : row - nd_all) * stride + head * HD;
    const float *qr = (detail ? p.q_d : p.q_g) + off, *gr = (detail ? p.do_d : p.do_g) + off;
    float q[HD / 32], go[HD / 32], dq[HD / 32];
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) {
        q[e] = qr[lane + 32 * e];
        go[e] = gr[lane + 32 * e];
        dq[e] = 0.f;
    }
    const int64_t col = (b * g.heads + head) * (g.N + g.G) + (detail ? local : g.N + local);
    const float lse = p.lse[col], delta = p.delta[col];
    int64_t g_lo = 0, g_hi = g.G;
    if (detail) {
        const int64_t w = window_of(g, local);
        int64_t lo, hi;
        window_rows(g, w, local, lo, hi);
        global_rows(g, w, g_lo, g_hi);
        dq_keys<HD>(p.k_d + b * g.N * stride + head * HD, p.v_d + b * g.N * stride + head * HD,
                    lo, hi, stride, q, go, p.scale, lse, delta, dq);
    }
    dq_keys<HD>(p.k_g + b * g.G * stride + head * HD, p.v_g + b * g.G * stride + head * HD,
                g_lo, g_hi, stride, q, go, p.scale, lse, delta, dq);
    float *out = (detail ? p.dq_d : p.dq_g) + off;
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) out[lane + 32 * e] = dq[e] * p.scale;
}

// ---------------------------------------------------------------------------
// fp32 dK, dV: one warp per (key row, head).
// ---------------------------------------------------------------------------
template <int HD>
__device__ __forceinline__ void kv_queries(const BwdPtr &p, const Geo &g, const float *q,
                                           const float *go, int64_t q0, int64_t q1,
                                           int64_t stride, int64_t col0,
                                           const float (&k)[HD / 32], const float (&v)[HD / 32],
                                           float (&dk)[HD / 32], float (&dv)[HD / 32]) {
    const int lane = threadIdx.x & 31;
    for (int64_t i = q0; i < q1; ++i) {
        const float *qr = q + i * stride, *gr = go + i * stride;
        float s = 0.f, dp = 0.f;
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) {
            s = fmaf(qr[lane + 32 * e], k[e], s);
            dp = fmaf(gr[lane + 32 * e], v[e], dp);
        }
        s = warp_sum(s);
        dp = warp_sum(dp);
        const float pr = expf(s * p.scale - p.lse[col0 + i]);
        const float ds = pr * (dp - p.delta[col0 + i]);
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) {
            dk[e] = fmaf(ds, qr[lane + 32 * e], dk[e]);
            dv[e] = fmaf(pr, gr[lane + 32 * e], dv[e]);
        }
    }
}

template <int HD>
__global__ void __launch_bounds__(kWarps * 32) dkdv_simt_kernel(const BwdPtr p, const Geo g) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + threadIdx.x / 32;
    const int head = blockIdx.y;
    const int64_t nd_all = g.batch * g.N;
    if (row >= nd_all + g.batch * g.G) return;
    const bool detail = row < nd_all;
    const int64_t b = detail ? row / g.N : (row - nd_all) / g.G;
    const int64_t local = detail ? row - b * g.N : row - nd_all - b * g.G;
    const int64_t stride = static_cast<int64_t>(g.heads) * HD;
    const int64_t off = (detail ? row : row - nd_all) * stride + head * HD;
    const float *kr = (detail ? p.k_d : p.k_g) + off, *vr = (detail ? p.v_d : p.v_g) + off;
    float k[HD / 32], v[HD / 32], dk[HD / 32], dv[HD / 32];
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) {
        k[e] = kr[lane + 32 * e];
        v[e] = vr[lane + 32 * e];
        dk[e] = 0.f;
        dv[e] = 0.f;
    }
    const int64_t col0 = (b * g.heads + head) * (g.N + g.G);   // LSE / delta row base
    const float *qd = p.q_d + b * g.N * stride + head * HD;
    const float *gd = p.do_d + b * g.N * stride + head * HD;
    if (detail) {
        int64_t lo, hi;
        window_rows(g, window_of(g, local), local, lo, hi);
        kv_queries<HD>(p, g, qd, gd, lo, hi, stride, col0, k, v, dk, dv);
    } else {
        // detail queries that see this global key
        int64_t lo = 0, hi = g.N;
        if (g.gwin_off != nullptr) {
            int64_t a = 0, c = g.n_win - 1;       // last window whose range starts <= local
            while (a < c) {
                const int64_t mid = (a + c + 1) / 2;
                if (g.gwin_off[mid] <= local) a = mid; else c = mid - 1;
            }
            int64_t glo, ghi;
            global_rows(g, a, glo, ghi);
            lo = hi = 0;
            if (glo <= local && local < ghi) {
                const int64_t first = g.win_off ? clamp64(g.win_off[a], 0, g.N) : a * g.L;
                const int64_t last = g.win_off ? clamp64(g.win_off[a + 1], first, g.N)
                                               : (a + 1) * g.L;
                lo = first;
                hi = last;
            }
        }
        if (g.N > 0) kv_queries<HD>(p, g, qd, gd, lo, hi, stride, col0, k, v, dk, dv);
        kv_queries<HD>(p, g, p.q_g + b * g.G * stride + head * HD,
                       p.do_g + b * g.G * stride + head * HD, 0, g.G, stride, col0 + g.N, k, v,
                       dk, dv);
    }
    float *ok = (detail ? p.dk_d : p.dk_g) + off, *ov = (detail ? p.dv_d : p.dv_g) + off;
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) {
        ok[lane + 32 * e] = dk[e] * p.scale;
        ov[lane + 32 * e] = dv[e];
    }
}

Geo geo_of(const AttnArgs &a) {
    Geo g;
    g.N = a.n_detail;
    g.L = a.n_detail > 0 ? a.window_len : 1;
    g.G = a.n_global;
    g.batch = a.batch;
    g.n_win = a.win_off ? a.n_win : a.n_gwin;
    g.heads = a.heads;
    g.win_off = a.win_off;
    g.gwin_off = a.gwin_off;
    return g;
}

dim3 row_grid(const AttnArgs &a) {
    const int64_t rows = a.batch * (a.n_detail + a.n_global);
    return dim3(static_cast<unsigned>((rows + kWarps - 1) / kWarps),
                static_cast<unsigned>(a.heads));
}

template <typename T, int HD>
atlas_status delta_hd(const AttnBwdArgs &b, cudaStream_t stream) {
    const AttnArgs &a = b.fwd;
    if (log_enabled())
        log_launch("delta_kernel", static_cast<int>(row_grid(a).x * row_grid(a).y), kWarps * 32, 0,
                   "head_dim %d rows %lld heads %d", HD,
                   static_cast<long long>(a.batch * (a.n_detail + a.n_global)), a.heads);
    delta_kernel<T, HD><<<row_grid(a), kWarps * 32, 0, stream>>>(
        static_cast<const T *>(a.o_d), static_cast<const T *>(b.do_d),
        static_cast<const T *>(a.o_g), static_cast<const T *>(b.do_g), b.delta, geo_of(a));
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

template <int HD>
atlas_status bwd_simt_hd(const AttnBwdArgs &b, cudaStream_t stream) {
    const AttnArgs &a = b.fwd;
    BwdPtr p;
    p.q_d = static_cast<const float *>(a.q_d);
    p.k_d = static_cast<const float *>(a.k_d);
    p.v_d = static_cast<const float *>(a.v_d);
    p.do_d = static_cast<const float *>(b.do_d);
    p.q_g = static_cast<const float *>(a.q_g);
    p.k_g = static_cast<const float *>(a.k_g);
    p.v_g = static_cast<const float *>(a.v_g);
    p.do_g = static_cast<const float *>(b.do_g);
    p.lse = a.lse;
    p.delta = b.delta;
    p.dq_d = static_cast<float *>(b.dq_d);
    p.dk_d = static_cast<float *>(b.dk_d);
    p.dv_d = static_cast<float *>(b.dv_d);
    p.dq_g = static_cast<float *>(b.dq_g);
    p.dk_g = static_cast<float *>(b.dk_g);
    p.dv_g = static_cast<float *>(b.dv_g);
    p.scale = a.scale;
    const Geo g = geo_of(a);
    if (log_enabled())
        log_launch("dq_simt_kernel + dkdv_simt_kernel", static_cast<int>(row_grid(a).x * row_grid(a).y),
                   kWarps * 32, 0, "head_dim %d (fp32)", HD);
    dq_simt_kernel<HD><<<row_grid(a), kWarps * 32, 0, stream>>>(p, g);
    dkdv_simt_kernel<HD><<<row_grid(a), kWarps * 32, 0, stream>>>(p, g);
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

}  // namespace

atlas_status launch_attn_bwd_delta(const AttnBwdArgs &b, cudaStream_t stream) {
    if (b.fwd.batch * (b.fwd.n_detail + b.fwd.n_global) == 0) return ATLAS_OK;
    const int hd = b.fwd.head_dim;
    if (b.elem_bytes == 2) {
        if (hd == 128) return delta_hd<__nv_bfloat16, 128>(b, stream);
        if (hd == 64) return delta_hd<__nv_bfloat16, 64>(b, stream);
    } else {
        if (hd == 128) return delta_hd<float, 128>(b, stream);
        if (hd == 64) return delta_hd<float, 64>(b, stream);
    }
    return ATLAS_ERR_UNSUPPORTED;
}

atlas_status launch_attn_bwd_simt_f32(const AttnBwdArgs &b, cudaStream_t stream) {
    if (b.fwd.head_dim == 128) return bwd_simt_hd<128>(b, stream);
    if (b.fwd.head_dim == 64) return bwd_simt_hd<64>(b, stream);
    return ATLAS_ERR_UNSUPPORTED;
}

}  // namespace atlas
