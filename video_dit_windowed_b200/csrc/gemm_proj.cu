// gemm_proj.cu -- the projections on either side of the path as tcgen05
// GEMMs whose epilogue does the path's permutation (and RoPE).
//
// Passages: "Technische Samenvatting: AtlasVid", Methodologie 1, Fase 2 (cube
// reorder), Fase 1 and Methodologie 2 (RoPE, position alignment); the
// projections themselves are the attention layer's linear maps, which the
// summary's training strategy adapts.
//
//   QKV:  [Q | K | V] = X W^T for X in raster order; Q and K rotated by 3D RoPE
//         at each token's grid position, all three written in cube order.
//   OUT:  Y = O W^T for O in cube order, each row written back to its raster
//         position.
// A GEMM acts on rows independently, so permuting its output rows is the
// same as permuting its input rows: both fusions are a row-scattering
// epilogue. The rotation uses the fp32 accumulator, so a rotated row is
// rounded to bf16 once.
//
// C[M, N] = A[M, K] B[N, K]^T, bf16 in, fp32 accumulate: 128 x 256 tiles, K in
// steps of 64 (one 128-byte swizzle atom), 4-stage TMA ring (48 KB a stage),
// persistent CTAs. Warps 0-3: epilogue (thread = accumulator row = tensor
// memory lane); warp 4: TMA producer; warp 5: MMA issuer (one thread). Two
// 256-column accumulators in tensor memory, so one tile's epilogue overlaps
// the next tile's main loop. Tiles are walked in groups of 8 column tiles so
// the CTAs in flight share their A and B tiles in L2. Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "atlas_internal.cuh"
#include "cube_geom.cuh"
#include "sm100_ptx.cuh"

namespace atlas {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kProducerWarp = 4, kMmaWarp = 5, kThreads = 192;
constexpr int kEpilogue = 128;
constexpr uint32_t kTmemCols = 512;   // two 256-column fp32 accumulators
constexpr int kGroupN = 8;            // column tiles per scheduling group

enum Mode { kModeQKV = 0, kModeOut = 1 };

struct Smem {
    static constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
    static constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32 KB
    alignas(1024) uint8_t a[kStages][kABytes];
    alignas(1024) uint8_t b[kStages][kBBytes];
    uint64_t full[kStages], empty[kStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    volatile int abort;
    uint32_t *err_word;
};

struct Params {
    CUtensorMap tm_a, tm_b;
    int32_t M, N, K;
    int32_t m_tiles, n_tiles, k_steps, n_tile_total;
    int32_t mode;
    __nv_bfloat16 *out[3];      // QKV: q, k, v [M, heads, hd]; OUT: y [M, N]
    int32_t heads, hd;          // QKV
    uint32_t rows;              // tokens of one problem
    geom::FastDiv by_rows;
    geom::Geom g;
    int32_t general;            // the cube does not divide the grid
    const float2 *tab;          // RoPE cos/sin (QKV; NULL: no rotation)
    uint32_t tab_base[3], half[3];
    uint32_t *err_word;
};

// Tile t of the walk: groups of kGroupN column tiles, rows inside a group,
// columns fastest.
__device__ __forceinline__ void tile_of(const Params &p, int32_t t, int32_t &m0, int32_t &n0) {
    const int32_t per_group = p.m_tiles * kGroupN;
    const int32_t grp = t / per_group;
    const int32_t rem = t - grp * per_group;
    const int32_t gn = min(kGroupN, p.n_tiles - grp * kGroupN);
    const int32_t mi = rem / gn, ni = rem - mi * gn;
    m0 = mi * kBM;
    n0 = (grp * kGroupN + ni) * kBN;
}

// Destination row of GEMM row m, and the token's raster coordinates.
__device__ __forceinline__ uint32_t dst_row(const Params &p, uint32_t m, uint32_t &t,
                                            uint32_t &h, uint32_t &w) {
    const uint32_t b = p.by_rows.div(m), r = m - b * p.rows;
    uint32_t pos;
    if (p.mode == kModeQKV) {            // raster -> cube order
        geom::raster_coords(p.g, r, t, h, w);
        pos = p.general ? geom::cube_position_general(p.g, t, h, w)
                        : geom::cube_position(p.g, t, h, w);
    } else {                             // cube order -> raster
        if (p.general) geom::cube_coords_general(p.g, r, t, h, w);
        else geom::cube_coords(p.g, r, t, h, w);
        pos = (t * p.g.H + h) * p.g.W + w;
    }
    return b * p.rows + pos;
}

__device__ __forceinline__ bool wait_phase(Smem &sm, uint64_t &bar, uint32_t parity,
                                           uint32_t err, bool honor_abort = true) {
    const uint32_t a = ptx::smem_addr(&bar);
    if (ptx::mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (ptx::mbar_try_wait(a, parity)) return true;
        if ((spin & 63u) == 0) {
            if (honor_abort && sm.abort) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                atomicOr(sm.err_word, err);
                sm.abort = 1;
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Producer: A (128 x 64) and B (256 x 64) tiles per K step into the ring.
// ---------------------------------------------------------------------------
__device__ void producer(const Params &p, Smem &sm) {
    uint32_t it = 0;
    uint32_t armed[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) armed[s] = 0;
    bool ok = true;
    for (int32_t t = blockIdx.x; t < p.n_tile_total && ok; t += gridDim.x) {
        int32_t m0, n0;
        tile_of(p, t, m0, n0);
        for (int32_t k = 0; k < p.k_steps && ok; ++k, ++it) {
            const uint32_t s = it % kStages, round = it / kStages;
            if (round > 0 && !(ok = wait_phase(sm, sm.empty[s], (round - 1) & 1,
                                               kErrTimeoutProducer)))
                break;
            const uint32_t bar = ptx::smem_addr(&sm.full[s]);
            ptx::mbar_arrive_expect_tx(bar, Smem::kABytes + Smem::kBBytes);
            ptx::tma_load_2d(ptx::smem_addr(sm.a[s]), &p.tm_a, bar, k * kBK, m0);
            ptx::tma_load_2d(ptx::smem_addr(sm.b[s]), &p.tm_b, bar, k * kBK, n0);
#pragma unroll
            for (int q = 0; q < kStages; ++q)
                if (q == static_cast<int>(s)) armed[q] = round + 1;
        }
    }
    if (!ok) {
        for (int q = 0; q < kStages; ++q)
            if (armed[q])
                wait_phase(sm, sm.full[q], (armed[q] - 1) & 1, kErrTimeoutTeardown, false);
    }
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread): per tile, K/16 MMAs of 128 x 256 x 16 into the
// tile's accumulator (alternating between the two).
// ---------------------------------------------------------------------------
__device__ void mma_issuer(const Params &p, Smem &sm, uint32_t tmem) {
    constexpr uint32_t kIdesc = ptx::idesc_bf16_f32(kBM, kBN, 0);
    constexpr uint32_t kHi = ptx::desc_sw128_hi(1024);
    constexpr uint32_t kA16 = Smem::kABytes >> 4, kB16 = Smem::kBBytes >> 4;
    const uint32_t a_lo0 = ptx::desc_sw128_lo(ptx::smem_addr(sm.a[0]), 16);
    const uint32_t b_lo0 = ptx::desc_sw128_lo(ptx::smem_addr(sm.b[0]), 16);
    uint32_t it = 0, tile_iter = 0;
    bool ok = true;
    for (int32_t t = blockIdx.x; t < p.n_tile_total && ok; t += gridDim.x, ++tile_iter) {
        const uint32_t ab = tile_iter & 1;
        if (tile_iter >= 2 &&
            !(ok = wait_phase(sm, sm.acc_empty[ab], ((tile_iter >> 1) - 1) & 1, kErrTimeoutMma)))
            break;
        ptx::tc_fence_after();
        const uint32_t d = tmem + ab * kBN;
        for (int32_t k = 0; k < p.k_steps && ok; ++k, ++it) {
            const uint32_t s = it % kStages;
            if (!(ok = wait_phase(sm, sm.full[s], (it / kStages) & 1, kErrTimeoutMma))) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
                ptx::mma_ss(d, ptx::desc_join(a_lo0 + s * kA16 + kk * 2, kHi),
                            ptx::desc_join(b_lo0 + s * kB16 + kk * 2, kHi), kIdesc,
                            (k > 0 || kk > 0) ? 1u : 0u);
            ptx::mma_commit(ptx::smem_addr(&sm.empty[s]));
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&sm.acc_full[ab]));
    }
    ptx::mma_commit(ptx::smem_addr(&sm.drain));
    wait_phase(sm, sm.drain, 0, kErrTimeoutTeardown, false);
}

// ---------------------------------------------------------------------------
// Epilogue: thread = row; 8 chunks of 32 accumulator columns -> (RoPE) ->
// bf16 -> the row's destination.
// ---------------------------------------------------------------------------
__device__ void epilogue(const Params &p, Smem &sm, uint32_t tmem) {
    const uint32_t warp = threadIdx.x / 32, r = threadIdx.x & 127;
    const uint32_t lane_sel = (warp * 32u) << 16;
    uint32_t tile_iter = 0;
    for (int32_t t = blockIdx.x; t < p.n_tile_total; t += gridDim.x, ++tile_iter) {
        int32_t m0, n0;
        tile_of(p, t, m0, n0);
        const uint32_t ab = tile_iter & 1;
        if (!__all_sync(0xffffffffu, wait_phase(sm, sm.acc_full[ab], (tile_iter >> 1) & 1,
                                                kErrTimeoutSoftmax)))
            return;
        ptx::tc_fence_after();
        const int32_t m = m0 + static_cast<int32_t>(r);
        const bool valid = m < p.M;
        uint32_t tt = 0, th = 0, tw = 0, drow = 0;
        if (valid) drow = dst_row(p, static_cast<uint32_t>(m), tt, th, tw);
#pragma unroll 1
        for (int c = 0; c < kBN / 32; ++c) {
            uint32_t v[32];
            ptx::tmem_ld32(tmem + ab * kBN + c * 32 + lane_sel, v);
            if (!valid) continue;
            const int32_t n = n0 + c * 32;
            uint4 *dst;
            if (p.mode == kModeQKV) {
                const int32_t width = p.heads * p.hd;
                const int32_t which = n / width, within = n - which * width;
                const int32_t head = within / p.hd, d0 = within - head * p.hd;
                if (which < 2 && p.tab != nullptr) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const uint32_t P = static_cast<uint32_t>(d0 / 2 + i);   // pair in head
                        const uint32_t ax = P < p.half[0] ? 0u : (P < p.half[0] + p.half[1] ? 1u : 2u);
                        const uint32_t kk = ax == 0 ? P : (ax == 1 ? P - p.half[0]
                                                                   : P - p.half[0] - p.half[1]);
                        const uint32_t pos = ax == 0 ? tt : (ax == 1 ? th : tw);
                        const float2 cs = __ldg(p.tab + p.tab_base[ax] + pos * p.half[ax] + kk);
                        const float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
                        v[2 * i] = __float_as_uint(fmaf(x0, cs.x, -(x1 * cs.y)));
                        v[2 * i + 1] = __float_as_uint(fmaf(x0, cs.y, x1 * cs.x));
                    }
                }
                dst = reinterpret_cast<uint4 *>(
                    p.out[which] + (static_cast<int64_t>(drow) * p.heads + head) * p.hd + d0);
            } else {
                dst = reinterpret_cast<uint4 *>(p.out[0] + static_cast<int64_t>(drow) * p.N + n);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 o;
                o.x = ptx::pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                o.y = ptx::pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                o.z = ptx::pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                o.w = ptx::pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                dst[q] = o;
            }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&sm.acc_empty[ab]));
    }
}

__global__ void __launch_bounds__(kThreads, 1) gemm_proj_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sm = *reinterpret_cast<Smem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&sm.full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(ptx::smem_addr(&sm.acc_full[b]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.acc_empty[b]), kEpilogue);
        }
        ptx::mbar_init(ptx::smem_addr(&sm.drain), 1);
        sm.abort = 0;
        sm.err_word = p.err_word;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&sm.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        ptx::prefetch_tmap(&p.tm_a);
        ptx::prefetch_tmap(&p.tm_b);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const bool tmem_ok = tmem == 0;   // a 512-column allocation starts at column 0
    if (!tmem_ok && threadIdx.x == 0) atomicOr(p.err_word, kErrTmemAlloc);
    if (tmem_ok) {
        if (warp < 4) epilogue(p, sm, tmem);
        else if (lane == 0) {
            if (warp == kProducerWarp) producer(p, sm);
            else mma_issuer(p, sm, tmem);
        }
    }
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

// [rows, cols] bf16 row-major as a 2-D tensor map, box 64 x box_rows,
// 128-byte swizzle.
bool make_matrix_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols,
                     int box_rows) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

atlas_status launch(Params &p, const void *a, const void *b, const DeviceInfo &dev,
                    cudaStream_t stream) {
    if (!make_matrix_map(&p.tm_a, a, p.M, p.K, kBM) || !make_matrix_map(&p.tm_b, b, p.N, p.K, kBN))
        return ATLAS_ERR_CUDA;
    p.err_word = device_error_word();
    if (!p.err_word) return ATLAS_ERR_CUDA;
    p.m_tiles = (p.M + kBM - 1) / kBM;
    p.n_tiles = p.N / kBN;
    p.k_steps = p.K / kBK;
    const int64_t total = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
    if (total == 0) return ATLAS_OK;
    if (total > INT32_MAX) return ATLAS_ERR_SHAPE;
    p.n_tile_total = static_cast<int32_t>(total);
    const size_t smem = sizeof(Smem) + 1024;
    if (!set_smem_limit(reinterpret_cast<const void *>(gemm_proj_kernel),
                        static_cast<int>(smem)))
        return ATLAS_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(total, dev.sm_count));
    if (log_enabled())
        log_launch("gemm_proj_kernel", grid, kThreads, smem,
                   "M %d N %d K %d tiles %d (128x256, groups of %d column tiles)%s", p.M, p.N,
                   p.K, p.n_tile_total, kGroupN, p.tab ? " rope" : "");
    gemm_proj_kernel<<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

void set_rows(Params &p, const ProjArgs &a) {
    p.rows = static_cast<uint32_t>(a.T * a.H * a.W);
    p.by_rows = geom::FastDiv(p.rows);
    p.g = geom::make_geom(static_cast<uint32_t>(a.T), static_cast<uint32_t>(a.H),
                          static_cast<uint32_t>(a.W), static_cast<uint32_t>(a.ct),
                          static_cast<uint32_t>(a.ch), static_cast<uint32_t>(a.cw));
    p.general = (a.T % a.ct) || (a.H % a.ch) || (a.W % a.cw);
    p.M = static_cast<int32_t>(a.batch * a.T * a.H * a.W);
}

}  // namespace

atlas_status launch_qkv_proj(const ProjArgs &a, cudaStream_t stream) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    Params p{};
    set_rows(p, a);
    p.mode = kModeQKV;
    p.K = a.c_in;
    p.N = 3 * a.heads * a.head_dim;
    p.heads = a.heads;
    p.hd = a.head_dim;
    for (int i = 0; i < 3; ++i) p.out[i] = static_cast<__nv_bfloat16 *>(a.out[i]);
    if (a.rope) {
        const float2 *tab = nullptr;
        atlas_status st = rope_table_for(a.T, a.H, a.W, *a.rope, &tab);
        if (st != ATLAS_OK) return st;
        p.tab = tab;
        p.half[0] = static_cast<uint32_t>(a.rope->d_t / 2);
        p.half[1] = static_cast<uint32_t>(a.rope->d_h / 2);
        p.half[2] = static_cast<uint32_t>(a.rope->d_w / 2);
        p.tab_base[0] = 0;
        p.tab_base[1] = static_cast<uint32_t>(a.T) * p.half[0];
        p.tab_base[2] = p.tab_base[1] + static_cast<uint32_t>(a.H) * p.half[1];
    }
    return launch(p, a.x, a.w, dev, stream);
}

atlas_status launch_out_proj(const ProjArgs &a, cudaStream_t stream) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    Params p{};
    set_rows(p, a);
    p.mode = kModeOut;
    p.K = a.c_in;
    p.N = a.c_out;
    p.out[0] = static_cast<__nv_bfloat16 *>(a.out[0]);
    return launch(p, a.x, a.w, dev, stream);
}

}  // namespace atlas
