// attn_simt.cu -- asymmetric local-global attention, fp32 I/O, SIMT fp32.
//
// Passages: as attn_tc.cu ("Technische Samenvatting: AtlasVid", Methodologie
// 1 Fase 2 and Methodologie 2). This kernel serves fp32 tensors, whose
// workloads here are small and launch-bound: one warp per (query row, head),
// exact fp32 products, an online softmax with expf, keys streamed in order
// (own window first, then the global keys).
#include "atlas_internal.cuh"

namespace atlas {
namespace {

constexpr int kWarps = 8;

struct Params {
    const float *q_d, *k_d, *v_d, *q_g, *k_g, *v_g;
    float *o_d, *o_g, *lse;
    int64_t N, L, G;         // detail rows, window length, global rows of ONE problem
    int64_t batch;           // problems stacked along the rows
    int32_t heads;
    float scale;
    const int32_t *win_off;  // window offsets over one problem (NULL: windows of L rows)
    int64_t n_win;
    const int32_t *gwin_off; // global key offsets per window (NULL: every global key)
};

template <int HD>
__device__ __forceinline__ void accumulate_keys(const float *k, const float *v, int64_t k0,
                                                int64_t k1, int64_t row_stride,
                                                const float (&q)[HD / 32], float scale,
                                                float &m, float &l, float (&o)[HD / 32]) {
    const int lane = threadIdx.x & 31;
    for (int64_t key = k0; key < k1; ++key) {
        const float *kr = k + key * row_stride;
        const float *vr = v + key * row_stride;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) dot = fmaf(q[e], kr[lane + 32 * e], dot);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float s = dot * scale;
        const float m_new = fmaxf(m, s);
        const float corr = expf(m - m_new);
        const float p = expf(s - m_new);
        l = l * corr + p;
#pragma unroll
        for (int e = 0; e < HD / 32; ++e) o[e] = fmaf(p, vr[lane + 32 * e], o[e] * corr);
        m = m_new;
    }
}

// x limited to [lo, hi] (lo <= hi).
__device__ __forceinline__ int64_t clamp64(int64_t x, int64_t lo, int64_t hi) {
    return x < lo ? lo : (x > hi ? hi : x);
}

template <int HD>
__global__ void __launch_bounds__(kWarps * 32) attn_simt_kernel(const Params p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarps + threadIdx.x / 32;
    const int head = blockIdx.y;
    const int64_t nd_all = p.batch * p.N;
    if (row >= nd_all + p.batch * p.G) return;
    const bool detail = row < nd_all;
    // Problem b, and the row's index within its problem's detail or global rows.
    const int64_t b = detail ? row / p.N : (row - nd_all) / p.G;
    const int64_t local = detail ? row - b * p.N : row - nd_all - b * p.G;
    const int64_t stride = static_cast<int64_t>(p.heads) * HD;
    const float *qr = (detail ? p.q_d + row * stride : p.q_g + (row - nd_all) * stride) + head * HD;
    float q[HD / 32], o[HD / 32];
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) {
        q[e] = qr[lane + 32 * e];
        o[e] = 0.f;
    }
    float m = -__builtin_huge_valf(), l = 0.f;
    int64_t g_lo = 0, g_hi = p.G;
    if (detail) {
        int64_t lo, hi, w;
        if (p.win_off == nullptr) {
            w = local / p.L;
            lo = w * p.L;
            hi = lo + p.L;
        } else {  // last window whose start is <= local; range clamped to hold it
            int64_t a = 0, c = p.n_win - 1;
            while (a < c) {
                const int64_t mid = (a + c + 1) / 2;
                if (p.win_off[mid] <= local) a = mid; else c = mid - 1;
            }
            w = a;
            lo = clamp64(p.win_off[a], 0, local);
            hi = clamp64(p.win_off[a + 1], local + 1, p.N);
        }
        if (p.gwin_off != nullptr) {
            g_lo = clamp64(p.gwin_off[w], 0, p.G);
            g_hi = clamp64(p.gwin_off[w + 1], g_lo, p.G);
        }
        accumulate_keys<HD>(p.k_d + (b * p.N) * stride + head * HD,
                            p.v_d + (b * p.N) * stride + head * HD, lo, hi, stride, q, p.scale,
                            m, l, o);
    }
    if (g_hi > g_lo)
        accumulate_keys<HD>(p.k_g + (b * p.G) * stride + head * HD,
                            p.v_g + (b * p.G) * stride + head * HD, g_lo, g_hi, stride, q,
                            p.scale, m, l, o);
    float *out = (detail ? p.o_d + row * stride : p.o_g + (row - nd_all) * stride) + head * HD;
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < HD / 32; ++e) out[lane + 32 * e] = o[e] * inv;
    if (p.lse != nullptr && lane == 0)
        p.lse[(b * p.heads + head) * (p.N + p.G) + (detail ? local : p.N + local)] = m + logf(l);
}

template <int HD>
atlas_status launch_hd(const Params &p, cudaStream_t stream) {
    const int64_t rows = p.batch * (p.N + p.G);
    if (rows == 0) return ATLAS_OK;
    dim3 grid(static_cast<unsigned>((rows + kWarps - 1) / kWarps), static_cast<unsigned>(p.heads));
    if (log_enabled())
        log_launch("attn_simt_kernel", static_cast<int>(grid.x * grid.y), kWarps * 32, 0,
                   "head_dim %d rows %lld heads %d (fp32)", HD, static_cast<long long>(rows),
                   p.heads);
    attn_simt_kernel<HD><<<grid, kWarps * 32, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

}  // namespace

atlas_status launch_attn_simt_f32(const AttnArgs &a, cudaStream_t stream) {
    Params p{};
    p.q_d = static_cast<const float *>(a.q_d);
    p.k_d = static_cast<const float *>(a.k_d);
    p.v_d = static_cast<const float *>(a.v_d);
    p.q_g = static_cast<const float *>(a.q_g);
    p.k_g = static_cast<const float *>(a.k_g);
    p.v_g = static_cast<const float *>(a.v_g);
    p.o_d = static_cast<float *>(a.o_d);
    p.o_g = static_cast<float *>(a.o_g);
    p.lse = a.lse;
    p.N = a.n_detail;
    p.L = a.n_detail > 0 ? a.window_len : 1;
    p.G = a.n_global;
    p.heads = a.heads;
    p.scale = a.scale;
    p.win_off = a.win_off;
    p.n_win = a.n_win;
    p.batch = a.batch;
    p.gwin_off = a.gwin_off;
    if (a.head_dim == 64) return launch_hd<64>(p, stream);
    if (a.head_dim == 128) return launch_hd<128>(p, stream);
    return ATLAS_ERR_UNSUPPORTED;
}

}  // namespace atlas
