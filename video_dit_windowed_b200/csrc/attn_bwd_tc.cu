// attn_bwd_tc.cu -- backward of the asymmetric local-global attention, bf16,
// tcgen05 + TMA + TMEM.
//
// Passages: "Technische Samenvatting: AtlasVid", Methodologie 2 (the
// asymmetric mask; training adapts the attention projections, so the
// attention's gradients are needed). With P the row softmax of
// s = scale*<q,k> over the allowed keys, dO the output gradient and
// delta_i = <dO_i, O_i>:
//   dS = P o (dO V^T - delta),  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
//
// One kernel template, two forms:
//   DQ   -- resident: a 128-row tile of Q and of dO; streamed: K and V tiles
//           of the keys those rows may see (their windows, then the global
//           keys); accumulates dQ.
//   DKDV -- resident: a 128-row tile of K and of V; streamed: Q and dO tiles
//           of the queries that may see those keys (for a detail key, its
//           window's queries; for a global key, the detail queries that see
//           it and every global query); accumulates dV and dK.
// The DQ form keeps its resident Q and dO rows in tensor memory (written by
// the compute threads), so its S and dP MMAs read only the streamed half
// from shared memory (TS form); DKDV has no tensor memory to spare for K and
// V and reads them from shared memory (SS form).
// Resident tiles of detail rows follow the forward's unit forms: windows of
// at least 128 rows get tiles of their own (a fixed number of slots per
// window, the last one partly filled, slots past a shorter window's end
// skipped), so a tile never streams a neighbouring window's rows; shorter
// windows pack 128 consecutive rows. With window offsets the kernel finds the
// longest window itself.
// Either way a streamed tile of 128 rows is taken in two halves of 64, each
// loaded into its own stage of the shared-memory ring (so three halves can
// be in flight while one is used; the streamed queries' LSE and delta ride in
// the same stage, copied by cp.async). For
// half h the MMA warp computes  S_h = X X'_h^T  and  dP_h = Y Y'_h^T  into
// tensor memory (X, Y resident, X', Y' streamed: Q/K and dO/V for DQ, K/Q and
// V/dO for DKDV); the 128 compute threads (one resident row each) turn them
// into P_h and dS_h, written back as bf16 over the first half of their own
// columns; the MMA warp then accumulates from tensor memory:
//   DQ:    dQ += dS_h K_h
//   DKDV:  dV += P_h dO_h,  dK += dS_h Q_h        (P_h, dS_h transposed here)
// and issues the next tile's S_h, dP_h behind them. MMAs issued by one thread
// execute in order, so the next S_h cannot overwrite P_h before it is read,
// and the compute threads work on one half while the tensor core works on
// the other. Two compute warpgroups share the work: thread r of warpgroup g
// takes resident row r and columns 32g .. 32g+31 of each half (and, in the
// epilogue, half of the accumulator columns). Tensor memory:
// S_0 | S_1 | dP_0 | dP_1 (64 columns each) | acc (DQ: dQ, then the
// resident Q and dO; DKDV: dV, dK). Each warpgroup writes its packed P and
// dS over columns of S_h and dP_h that only it reads (group 0: columns 0-15,
// group 1: columns 48-63), so the two groups never wait for each other; the
// accumulating MMAs take their A operand from those two column ranges.
// Every wait is bounded, as in the forward kernel.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "atlas_internal.cuh"
#include "sm100_ptx.cuh"

namespace atlas {
namespace {

constexpr int kRows = 128;            // resident rows per unit = TMEM lanes
constexpr int kHalf = 64;             // streamed rows per half tile
constexpr int kCompute = 256;         // compute threads (warps 0-7: two warpgroups)
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

enum Form { kDQ = 0, kDKDV = 1 };

template <int HD>
struct Smem {
    static constexpr int kTile = kRows * HD * 2;                  // a 128-row bf16 tile
    static constexpr int kHalfTile = kHalf * HD * 2;              // a 64-row bf16 tile
    // streamed (X', Y') half-tile pairs: 128 KB of ring, at most 8 stages
    static constexpr int kStages = (128 * 1024) / (2 * kHalfTile) < 8
                                       ? (128 * 1024) / (2 * kHalfTile) : 8;
    alignas(1024) uint8_t x[kTile];                              // resident X (Q or K)
    alignas(1024) uint8_t y[kTile];                              // resident Y (dO or V)
    alignas(1024) uint8_t xs[kStages][kHalfTile];                // streamed X' (K or Q)
    alignas(1024) uint8_t ys[kStages][kHalfTile];                // streamed Y' (V or dO)
    float lse[kStages][kHalf];    // DKDV: LSE of the streamed queries (natural log)
    float delta[kStages][kHalf];  // DKDV: delta of the streamed queries
    uint64_t x_full, x_empty;
    uint64_t st_full[kStages], st_empty[kStages];
    uint64_t s_full[2], p_full[2];
    uint64_t acc_full, acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int32_t max_len;     // longest window, from the offsets
    volatile int abort;
    uint32_t *err_word;
};

struct Params {
    CUtensorMap tm_q[2], tm_k[2], tm_v[2], tm_do[2];   // 128-row boxes; [0] detail, [1] global
    CUtensorMap hm_q[2], hm_k[2], hm_v[2], hm_do[2];   // the same with 64-row boxes
    __nv_bfloat16 *out0[2], *out1[2];   // DQ: dq (out0); DKDV: dv (out0), dk (out1)
    const __nv_bfloat16 *res_x[2], *res_y[2];   // DQ: Q and dO rows (resident in TMEM)
    const float *lse, *delta;
    uint32_t *err_word;
    int32_t N, L, G, heads, batch;      // N, G: rows of ONE problem
    float scale_log2, scale;
    const int32_t *win_off, *gwin_off;
    int32_t n_win;
    int32_t tiles_d, tiles_g;           // 128-row tiles of one problem's detail / global rows
    int32_t n_long;                     // DKDV: units over global keys (scheduled first)
    int32_t upw;   // detail tiles per window; 0: packed tiles; -1: from the offsets
    int32_t o_v8;  // every output 32-byte aligned: the epilogue stores 32 B at a time
};

// The unit form and counts, the same in every thread of every CTA.
struct Sched {
    int32_t upw, n_dunits, n_units;
};

// max_len: the longest window (clamped ranges of the offsets), when p.upw < 0.
__device__ __forceinline__ Sched make_sched(const Params &p, int32_t max_len) {
    Sched S;
    S.upw = p.upw;
    if (S.upw < 0) {
        // Tiles of their own when windows are long enough, and their slots
        // stay within three times the packed count.
        const int64_t upw = (max_len + kRows - 1) / kRows;
        const int64_t n = static_cast<int64_t>(p.n_win) * upw;
        const bool ok = max_len >= kRows && n <= 3 * static_cast<int64_t>(p.tiles_d) &&
                        (n + p.tiles_g) * p.batch * p.heads <= INT32_MAX;
        S.upw = ok ? static_cast<int32_t>(upw) : 0;
    }
    const int32_t n_win = p.win_off != nullptr ? p.n_win : (p.L > 0 ? p.N / p.L : 0);
    S.n_dunits = S.upw > 0 ? n_win * S.upw : p.tiles_d;
    S.n_units = (S.n_dunits + p.tiles_g) * p.batch * p.heads;
    return S;
}

// ---- window geometry (per problem; as the forward) --------------------------
__device__ __forceinline__ int32_t window_of(const Params &p, int32_t x) {
    if (p.win_off == nullptr) return x / p.L;
    int32_t lo = 0, hi = p.n_win - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (__ldg(p.win_off + mid) <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}
__device__ __forceinline__ int32_t window_start(const Params &p, int32_t w, int32_t x) {
    return p.win_off == nullptr ? w * p.L : min(max(__ldg(p.win_off + w), 0), x);
}
__device__ __forceinline__ int32_t window_end(const Params &p, int32_t w, int32_t x) {
    return p.win_off == nullptr ? min(p.N, (w + 1) * p.L)
                                : max(min(__ldg(p.win_off + w + 1), p.N), x + 1);
}
// Rows of window w without a row to hold (the aligned lookup from a key).
__device__ __forceinline__ void window_rows(const Params &p, int32_t w, int32_t &lo,
                                            int32_t &hi) {
    if (p.win_off == nullptr) {
        lo = w * p.L;
        hi = min(p.N, lo + p.L);
    } else {
        lo = min(max(__ldg(p.win_off + w), 0), p.N);
        hi = min(max(__ldg(p.win_off + w + 1), lo), p.N);
    }
}
__device__ __forceinline__ int32_t global_start(const Params &p, int32_t w) {
    return p.gwin_off == nullptr ? 0 : min(max(__ldg(p.gwin_off + w), 0), p.G);
}
__device__ __forceinline__ int32_t global_end(const Params &p, int32_t w, int32_t start) {
    return p.gwin_off == nullptr ? p.G : min(max(__ldg(p.gwin_off + w + 1), start), p.G);
}
// Aligned variant: the window whose global range holds global row g (-1:
// none).
__device__ __forceinline__ int32_t window_of_global(const Params &p, int32_t g) {
    int32_t lo = 0, hi = p.n_win - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (__ldg(p.gwin_off + mid) <= g) lo = mid; else hi = mid - 1;
    }
    const int32_t s = global_start(p, lo);
    return (s <= g && g < global_end(p, lo, s)) ? lo : -1;
}

// A work unit: one head, one problem, resident rows r0 .. rend-1, and the
// streamed tiles: n_a tiles of detail rows from row a0 (rows up to a_end),
// then n_b tiles of global rows from row b0 (up to b_end); rows within the
// problem. win >= 0: a window tile, whose rows all see the same ranges.
// n_a + n_b == 0: an empty slot.
struct Unit {
    int32_t head, b, detail, r0, rend, a0, n_a, a_end, b0, n_b, b_end, win;
};

// Resident tile `lu` of one problem's detail rows in window form: the
// window's rows are streamed (and, for DQ, its global range).
template <int FORM>
__device__ __forceinline__ void window_tile(const Params &p, const Sched &S, int32_t lu,
                                            Unit &U) {
    const int32_t w = lu / S.upw, sub = lu - w * S.upw;
    int32_t s, e;
    window_rows(p, w, s, e);
    U.win = w;
    U.r0 = s + sub * kRows;
    U.rend = min(U.r0 + kRows, e);
    U.a0 = s;
    U.a_end = e;
    U.n_a = (e - s + kRows - 1) / kRows;
    U.b0 = U.n_b = U.b_end = 0;
    if (FORM == kDQ) {
        const int32_t g0 = global_start(p, w), g1 = global_end(p, w, g0);
        U.b0 = g0;
        U.b_end = g1;
        U.n_b = (g1 - g0 + kRows - 1) / kRows;
    }
    if (U.rend <= U.r0) U.n_a = U.n_b = 0;
}

template <int FORM>
__device__ __forceinline__ Unit decode_unit(const Params &p, const Sched &S, int32_t u) {
    Unit U;
    U.win = -1;
    const int32_t per_prob = S.n_dunits + p.tiles_g;
    if (FORM == kDQ) {
        U.head = u / (per_prob * p.batch);
        int32_t lu = u - U.head * per_prob * p.batch;
        U.b = lu / per_prob;
        lu -= U.b * per_prob;
        U.detail = lu < S.n_dunits;
        if (U.detail && S.upw > 0) {
            window_tile<FORM>(p, S, lu, U);
            return U;
        }
        U.r0 = (U.detail ? lu : lu - S.n_dunits) * kRows;
        U.rend = min(U.r0 + kRows, U.detail ? p.N : p.G);
        U.n_a = 0;
        U.a0 = U.a_end = 0;
        int32_t g0 = 0, g1 = p.G;
        if (U.detail) {
            const int32_t last = U.rend - 1;
            const int32_t w0 = window_of(p, U.r0), w1 = window_of(p, last);
            U.a0 = window_start(p, w0, U.r0);
            U.a_end = window_end(p, w1, last);
            U.n_a = (U.a_end - U.a0 + kRows - 1) / kRows;
            if (p.gwin_off != nullptr) {
                g0 = global_start(p, w0);
                g1 = max(global_end(p, w1, g0), g0);
            }
        }
        U.b0 = g0;
        U.b_end = g1;
        U.n_b = (g1 - g0 + kRows - 1) / kRows;
    } else {
        // global-key units first (they stream every query that sees them)
        const bool long_unit = u < p.n_long;
        const int32_t span = long_unit ? p.tiles_g : S.n_dunits;
        const int32_t v = long_unit ? u : u - p.n_long;
        U.head = v / (span * p.batch);
        int32_t lv = v - U.head * span * p.batch;
        U.b = lv / span;
        lv -= U.b * span;
        U.detail = !long_unit;
        if (U.detail && S.upw > 0) {
            window_tile<FORM>(p, S, lv, U);
            return U;
        }
        U.r0 = lv * kRows;
        U.rend = min(U.r0 + kRows, U.detail ? p.N : p.G);
        const int32_t last = U.rend - 1;
        if (U.detail) {
            const int32_t w0 = window_of(p, U.r0), w1 = window_of(p, last);
            U.a0 = window_start(p, w0, U.r0);
            U.a_end = window_end(p, w1, last);
            U.n_a = (U.a_end - U.a0 + kRows - 1) / kRows;
            U.b0 = U.b_end = 0;
            U.n_b = 0;
        } else {
            int32_t q0 = 0, q1 = p.N;
            if (p.gwin_off != nullptr && p.N > 0) {
                // windows whose global ranges hold the first and last key
                int32_t wa = -1, wb = -1;
                for (int32_t g = U.r0; g <= last && wa < 0; ++g) wa = window_of_global(p, g);
                for (int32_t g = last; g >= U.r0 && wb < 0; --g) wb = window_of_global(p, g);
                if (wa < 0) {
                    q0 = q1 = 0;
                } else {
                    int32_t lo, hi;
                    window_rows(p, wa, q0, hi);
                    window_rows(p, wb, lo, q1);
                    q1 = max(q1, q0);
                }
            }
            U.a0 = q0;
            U.a_end = q1;
            U.n_a = (q1 - q0 + kRows - 1) / kRows;
            U.b0 = 0;
            U.b_end = p.G;
            U.n_b = p.tiles_g;
        }
    }
    return U;
}

// Bounded wait (as the forward): false after flagging `err` when the phase
// did not complete within the limit, or when another role aborted.
template <int HD>
__device__ __forceinline__ bool wait_phase(Smem<HD> &sm, uint64_t &bar, uint32_t parity,
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

// Streamed tile j of unit U: detail rows (true) or global rows, and its first
// row within the problem.
__device__ __forceinline__ bool streamed_detail(const Unit &U, int32_t j) { return j < U.n_a; }
__device__ __forceinline__ int32_t streamed_row(const Unit &U, int32_t j) {
    return j < U.n_a ? U.a0 + j * kRows : U.b0 + (j - U.n_a) * kRows;
}

// ---------------------------------------------------------------------------
// Producer warp: resident X, Y once per unit; then the streamed tiles as
// 64-row halves, (X'_h, Y'_h) per ring stage, with (DKDV) the streamed
// queries' LSE and delta copied by cp.async and tracked by the same stage
// barrier.
// ---------------------------------------------------------------------------
template <int HD, int FORM>
__device__ void producer(const Params &p, const Sched &S, Smem<HD> &sm) {
    constexpr int kStages = Smem<HD>::kStages;
    constexpr uint32_t kTile = Smem<HD>::kTile, kHalfTile = Smem<HD>::kHalfTile;
    constexpr uint32_t kAll = 0xffffffffu;
    const uint32_t lane = threadIdx.x & 31;
    uint32_t it = 0, unit_iter = 0, x_armed = 0;
    uint32_t armed[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) armed[s] = 0;
    bool ok = true;
    // One tile of `rows_box` rows: HD/64 boxes of 64 channels.
    auto tile = [&](uint8_t *dst, const CUtensorMap *map, uint32_t bar, int32_t head,
                    int32_t row, uint32_t box_bytes) {
#pragma unroll
        for (int db = 0; db < HD / 64; ++db)
            ptx::tma_load_3d(ptx::smem_addr(dst + db * box_bytes), map, bar, db * 64, head,
                             row);
    };
    for (int32_t u = blockIdx.x; u < S.n_units && ok; u += gridDim.x) {
        const Unit U = decode_unit<FORM>(p, S, u);
        if (U.n_a + U.n_b == 0) continue;
        // Every lane waits and the warp agrees, so the lanes never diverge
        // around the warp-wide steps below. (DQ: the compute warps put the
        // resident Q and dO rows in tensor memory themselves.)
        if (FORM == kDKDV && unit_iter > 0 &&
            !(ok = __all_sync(kAll, wait_phase(sm, sm.x_empty, (unit_iter - 1) & 1,
                                               kErrTimeoutProducer))))
            break;
        const int side = U.detail ? 0 : 1;
        const int32_t rbase = U.b * (U.detail ? p.N : p.G);
        if (FORM == kDKDV && lane == 0) {
            const uint32_t bar = ptx::smem_addr(&sm.x_full);
            ptx::mbar_arrive_expect_tx(bar, 2 * kTile);
            tile(sm.x, FORM == kDQ ? &p.tm_q[side] : &p.tm_k[side], bar, U.head, rbase + U.r0,
                 kRows * 128);
            tile(sm.y, FORM == kDQ ? &p.tm_do[side] : &p.tm_v[side], bar, U.head, rbase + U.r0,
                 kRows * 128);
        }
        if (FORM == kDKDV) x_armed = unit_iter + 1;
        const int32_t n = 2 * (U.n_a + U.n_b);   // half tiles
        for (int32_t jh = 0; jh < n && ok; ++jh, ++it) {
            const uint32_t s = it % kStages, round = it / kStages;
            if (round > 0 &&
                !(ok = __all_sync(kAll, wait_phase(sm, sm.st_empty[s], (round - 1) & 1,
                                                   kErrTimeoutProducer))))
                break;
            const int32_t j = jh >> 1;
            const bool det = streamed_detail(U, j);
            const int32_t row = streamed_row(U, j) + (jh & 1) * kHalf;   // in the problem
            const int sside = det ? 0 : 1;
            const uint32_t bar = ptx::smem_addr(&sm.st_full[s]);
            if (FORM == kDKDV) {
                // LSE and delta of the 64 streamed queries. Rows past the
                // problem copy the last row's values: those columns are
                // masked by the compute warps.
                const int32_t nrows = det ? p.N : p.G;
                const int64_t col0 = (static_cast<int64_t>(U.b) * p.heads + U.head) *
                                         (p.N + p.G) + (det ? 0 : p.N);
#pragma unroll
                for (int i = 0; i < kHalf / 32; ++i) {
                    const int32_t c = i * 32 + lane, q = min(row + c, nrows - 1);
                    ptx::cp_async_4(ptx::smem_addr(&sm.lse[s][c]), p.lse + col0 + q);
                    ptx::cp_async_4(ptx::smem_addr(&sm.delta[s][c]), p.delta + col0 + q);
                }
                ptx::cp_async_mbar_arrive(bar);
                __syncwarp();
            }
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(bar, 2 * kHalfTile);
                const int32_t srow = (det ? U.b * p.N : U.b * p.G) + row;
                tile(sm.xs[s], FORM == kDQ ? &p.hm_k[sside] : &p.hm_q[sside], bar, U.head, srow,
                     kHalf * 128);
                tile(sm.ys[s], FORM == kDQ ? &p.hm_v[sside] : &p.hm_do[sside], bar, U.head,
                     srow, kHalf * 128);
            }
#pragma unroll
            for (int t = 0; t < kStages; ++t)
                if (t == static_cast<int>(s)) armed[t] = round + 1;
        }
        ++unit_iter;
    }
    if (!ok && lane == 0) {
        // Let every copy already issued land before the CTA can exit.
        if (x_armed) wait_phase(sm, sm.x_full, (x_armed - 1) & 1, kErrTimeoutTeardown, false);
        for (int t = 0; t < kStages; ++t)
            if (armed[t])
                wait_phase(sm, sm.st_full[t], (armed[t] - 1) & 1, kErrTimeoutTeardown, false);
    }
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread). Per unit: S_0, dP_0, S_1, dP_1 of tile 0; then per
// half h of tile j: acc += (P_h, dS_h)(j), release the half's stage, and
// S_h, dP_h of tile j+1.
// ---------------------------------------------------------------------------
template <int HD, int FORM>
__device__ void mma_issuer(const Params &p, const Sched &S, Smem<HD> &sm, uint32_t tmem) {
    constexpr int kStages = Smem<HD>::kStages;
    constexpr uint32_t kH16 = Smem<HD>::kHalfTile >> 4;
    constexpr uint32_t kIdS = ptx::idesc_bf16_f32(kRows, kHalf, 0);   // S_h, dP_h
    constexpr uint32_t kIdAcc = ptx::idesc_bf16_f32(kRows, HD, 1);    // acc += A(tmem) B
    constexpr uint32_t kHi = ptx::desc_sw128_hi(1024);
    const uint32_t x_lo = ptx::desc_sw128_lo(ptx::smem_addr(sm.x), 16);
    const uint32_t y_lo = ptx::desc_sw128_lo(ptx::smem_addr(sm.y), 16);
    const uint32_t xs_lo = ptx::desc_sw128_lo(ptx::smem_addr(sm.xs[0]), 16);
    const uint32_t ys_lo = ptx::desc_sw128_lo(ptx::smem_addr(sm.ys[0]), 16);
    // The same streamed half tiles as MN-major B operands of the
    // accumulation (64-channel blocks kHalf * 128 bytes apart).
    const uint32_t xs_mn = ptx::desc_sw128_lo(ptx::smem_addr(sm.xs[0]), kHalf * 128);
    const uint32_t ys_mn = ptx::desc_sw128_lo(ptx::smem_addr(sm.ys[0]), kHalf * 128);
    const uint32_t t_s = tmem, t_dp = tmem + 2 * kHalf, t_acc = tmem + 4 * kHalf;
    uint32_t it = 0, unit_iter = 0;
    uint32_t p_cnt = 0;
    bool ok = true;

    const uint32_t t_x = t_acc + HD, t_y = t_x + HD / 2;   // DQ: resident Q, dO (packed)
    // S_h = X X'^T and dP_h = Y Y'^T from the half tile in stage s; commit.
    // DKDV reads X, Y from shared memory (SS); DQ from tensor memory (TS), so
    // only the streamed half is read from shared memory.
    auto issue_sdp = [&](int h, uint32_t s) {
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
            const uint32_t a_off = ((ks / 4) * (kRows * 128) + (ks % 4) * 32) >> 4;
            const uint32_t b_off = ((ks / 4) * (kHalf * 128) + (ks % 4) * 32) >> 4;
            if (FORM == kDQ) {
                ptx::mma_ts(t_s + h * kHalf, t_x + ks * 8,
                            ptx::desc_join(xs_lo + s * kH16 + b_off, kHi), kIdS, ks > 0);
                ptx::mma_ts(t_dp + h * kHalf, t_y + ks * 8,
                            ptx::desc_join(ys_lo + s * kH16 + b_off, kHi), kIdS, ks > 0);
            } else {
                ptx::mma_ss(t_s + h * kHalf, ptx::desc_join(x_lo + a_off, kHi),
                            ptx::desc_join(xs_lo + s * kH16 + b_off, kHi), kIdS, ks > 0);
                ptx::mma_ss(t_dp + h * kHalf, ptx::desc_join(y_lo + a_off, kHi),
                            ptx::desc_join(ys_lo + s * kH16 + b_off, kHi), kIdS, ks > 0);
            }
        }
        ptx::mma_commit(ptx::smem_addr(&sm.s_full[h]));
    };
    // acc += A (tensor memory, 64 streamed rows packed in 32 columns) times
    // the half tile in stage s as an MN-major B operand.
    // The packed rows sit in columns 0-15 (keys 0-31, compute group 0) and
    // 48-63 (keys 32-63, group 1) of the half's 64.
    auto issue_acc = [&](uint32_t d, uint32_t a, uint32_t b_lo, uint32_t s, bool first) {
#pragma unroll
        for (int ks = 0; ks < kHalf / 16; ++ks) {
            const uint32_t off = s * kH16 + ((ks * 16 * 128) >> 4);
            const uint32_t col = ks < 2 ? ks * 8 : 32 + ks * 8;
            ptx::mma_ts(d, a + col, ptx::desc_join(b_lo + off, kHi), kIdAcc,
                        (first && ks == 0) ? 0u : 1u);
        }
    };
    auto next_stage = [&](uint32_t &s) -> bool {
        s = it % kStages;
        const bool r = wait_phase(sm, sm.st_full[s], (it / kStages) & 1, kErrTimeoutMma);
        ++it;
        ptx::tc_fence_after();
        return r;
    };

    for (int32_t u = blockIdx.x; u < S.n_units && ok; u += gridDim.x) {
        const Unit U = decode_unit<FORM>(p, S, u);
        const int32_t n = U.n_a + U.n_b;
        if (n == 0) continue;
        if (!(ok = wait_phase(sm, sm.x_full, unit_iter & 1, kErrTimeoutMma))) break;
        ptx::tc_fence_after();
        uint32_t st[2];   // stages of the current tile's halves
        if (!(ok = next_stage(st[0]))) break;
        issue_sdp(0, st[0]);
        if (!(ok = next_stage(st[1]))) break;
        issue_sdp(1, st[1]);
        // The resident rows are read by S and dP only: once the unit's last
        // S/dP are issued, a commit frees them for the next unit's rows.
        if (n == 1) ptx::mma_commit(ptx::smem_addr(&sm.x_empty));
        for (int32_t j = 0; j < n && ok; ++j) {
            const bool more = j + 1 < n;
            for (int h = 0; h < 2 && ok; ++h) {
                if (!(ok = wait_phase(sm, sm.p_full[h], p_cnt & 1, kErrTimeoutMma))) break;
                if (j == 0 && h == 0 && unit_iter > 0 &&
                    !(ok = wait_phase(sm, sm.acc_empty, (unit_iter - 1) & 1, kErrTimeoutMma)))
                    break;
                ptx::tc_fence_after();
                const bool first = j == 0 && h == 0;
                if (FORM == kDQ) {
                    issue_acc(t_acc, t_dp + h * kHalf, xs_mn, st[h], first);        // dQ
                } else {
                    issue_acc(t_acc, t_s + h * kHalf, ys_mn, st[h], first);       // dV
                    issue_acc(t_acc + HD, t_dp + h * kHalf, xs_mn, st[h], first);  // dK
                }
                ptx::mma_commit(ptx::smem_addr(&sm.st_empty[st[h]]));
                if (more) {
                    if (!(ok = next_stage(st[h]))) break;
                    issue_sdp(h, st[h]);
                    if (h == 1 && j + 2 == n) ptx::mma_commit(ptx::smem_addr(&sm.x_empty));
                }
            }
            ++p_cnt;
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&sm.acc_full));
        ++unit_iter;
    }
    // Drain: every MMA issued must finish before tensor memory is freed.
    ptx::mma_commit(ptx::smem_addr(&sm.drain));
    wait_phase(sm, sm.drain, 0, kErrTimeoutTeardown, false);
}

// ---------------------------------------------------------------------------
// Compute warps: thread = resident row = tensor-memory lane.
// ---------------------------------------------------------------------------
template <int HD, int FORM>
__device__ void compute(const Params &p, const Sched &S, Smem<HD> &sm, uint32_t tmem) {
    constexpr int kStages = Smem<HD>::kStages;
    constexpr int kCols = kHalf / 2;                 // columns of a half per warpgroup
    constexpr uint32_t kAll = 0xffffffffu;
    const uint32_t warp = threadIdx.x / 32, r = threadIdx.x & 127;
    const int part = static_cast<int>(warp / 4);     // warpgroup: column block
    const uint32_t lane_sel = ((warp & 3) * 32u) << 16;
    const uint32_t t_s = tmem + lane_sel, t_dp = tmem + 2 * kHalf + lane_sel;
    const uint32_t t_acc = tmem + 4 * kHalf + lane_sel;
    const uint32_t t_res = t_acc + HD + part * (HD / 2);   // DQ: this group's resident Q or dO
    const float c2 = p.scale_log2;
    uint32_t cnt = 0, unit_iter = 0;

    // DQ: the resident rows of unit V into tensor memory: warpgroup 0 the Q
    // row, warpgroup 1 the dO row (bf16 pairs, element 2c in the low half of
    // column c: the A-operand layout of the TS MMAs). Rows past the unit are
    // zeros. The previous unit's S/dP MMAs must be done (x_empty).
    auto write_resident = [&](const Unit &V) {
        const int32_t vrow = V.r0 + static_cast<int32_t>(r);
        uint32_t rv[HD / 2];
        if (vrow < V.rend) {
            const int64_t abs_row = static_cast<int64_t>(V.b) * (V.detail ? p.N : p.G) + vrow;
            const uint4 *src = reinterpret_cast<const uint4 *>(
                (part == 0 ? p.res_x : p.res_y)[V.detail ? 0 : 1] +
                (abs_row * p.heads + V.head) * HD);
#pragma unroll
            for (int i = 0; i < HD / 8; ++i) {
                const uint4 w4 = __ldg(src + i);
                rv[4 * i] = w4.x;
                rv[4 * i + 1] = w4.y;
                rv[4 * i + 2] = w4.z;
                rv[4 * i + 3] = w4.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < HD / 2; ++i) rv[i] = 0u;
        }
        if constexpr (HD == 128) ptx::tmem_st64(t_res, rv);
        else ptx::tmem_st32(t_res, rv);
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&sm.x_full));
    };
    bool resident_ready = false;   // DQ: this unit's rows were written ahead

    for (int32_t u = blockIdx.x; u < S.n_units; u += gridDim.x) {
        const Unit U = decode_unit<FORM>(p, S, u);
        if (U.n_a + U.n_b == 0) continue;
        const int32_t row = U.r0 + static_cast<int32_t>(r);   // resident row (in problem)
        const bool valid = row < U.rend;
        // Allowed streamed rows: [da, db) of detail tiles, [ga, gb) of global tiles.
        int32_t da = 0, db = 0, ga = 0, gb = 0;
        float lse2_own = 0.f, delta_own = 0.f;
        if (valid) {
            if (FORM == kDQ) {
                ga = 0;
                gb = p.G;
                if (U.detail && U.win >= 0) {
                    da = U.a0;
                    db = U.a_end;
                    ga = U.b0;
                    gb = U.b_end;
                } else if (U.detail) {
                    const int32_t w = window_of(p, row);
                    da = window_start(p, w, row);
                    db = window_end(p, w, row);
                    ga = global_start(p, w);
                    gb = global_end(p, w, ga);
                }
                const int64_t col = (static_cast<int64_t>(U.b) * p.heads + U.head) *
                                        (p.N + p.G) + (U.detail ? row : p.N + row);
                lse2_own = __ldg(p.lse + col) * kLog2e;
                delta_own = __ldg(p.delta + col);
            } else if (U.detail && U.win >= 0) {
                da = U.a0;
                db = U.a_end;
            } else if (U.detail) {
                const int32_t w = window_of(p, row);
                da = window_start(p, w, row);
                db = window_end(p, w, row);
            } else {
                db = p.N;
                if (p.gwin_off != nullptr) {
                    const int32_t w = window_of_global(p, row);
                    if (w < 0) db = 0; else window_rows(p, w, da, db);
                }
                gb = p.G;
            }
        } else if (FORM == kDQ) {
            lse2_own = __builtin_huge_valf();
        }
        if (FORM == kDQ && !resident_ready) {
            if (unit_iter > 0 &&
                !__all_sync(kAll, wait_phase(sm, sm.x_empty, (unit_iter - 1) & 1,
                                             kErrTimeoutSoftmax)))
                return;
            write_resident(U);
        }
        resident_ready = false;
        const int32_t n = U.n_a + U.n_b;
        for (int32_t j = 0; j < n; ++j, ++cnt) {
            const bool det = streamed_detail(U, j);
            const int32_t base = streamed_row(U, j);
            const int32_t lo = det ? da : ga, hi = det ? db : gb;
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
                // ring stage of this half tile (the producer's order)
                const uint32_t hc = 2 * cnt + h, stage = hc % kStages, ch = cnt;
                if (FORM == kDKDV &&
                    !__all_sync(kAll, wait_phase(sm, sm.st_full[stage], (hc / kStages) & 1,
                                                 kErrTimeoutSoftmax)))
                    return;
                if (!__all_sync(kAll, wait_phase(sm, sm.s_full[h], ch & 1, kErrTimeoutSoftmax)))
                    return;
                ptx::tc_fence_after();
                uint32_t sv[kCols], dv[kCols];
                ptx::tmem_ld32(t_s + h * kHalf + part * kCols, sv);
                ptx::tmem_ld32(t_dp + h * kHalf + part * kCols, dv);
                const int32_t c0 = base + h * kHalf + part * kCols;   // row of column 0
                const bool partial = c0 < lo || c0 + kCols > hi;
                uint32_t pk_p[kCols / 2], pk_ds[kCols / 2];
#pragma unroll
                for (int e = 0; e < kCols / 2; ++e) {
                    float pv[2], dsv[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int c = 2 * e + k;
                        float l2, de;
                        if (FORM == kDQ) {
                            l2 = lse2_own;
                            de = delta_own;
                        } else {
                            l2 = sm.lse[stage][part * kCols + c] * kLog2e;
                            de = sm.delta[stage][part * kCols + c];
                        }
                        float pr = ptx::ex2(fmaf(__uint_as_float(sv[c]), c2, -l2));
                        if (partial && (c0 + c < lo || c0 + c >= hi)) pr = 0.f;
                        pv[k] = pr;
                        dsv[k] = pr * (__uint_as_float(dv[c]) - de);
                    }
                    pk_p[e] = ptx::pack_bf16x2(pv[0], pv[1]);
                    pk_ds[e] = ptx::pack_bf16x2(dsv[0], dsv[1]);
                }
                // Packed pairs go into this warpgroup's own columns (the first
                // 16 of group 0's 32, the last 16 of group 1's), which the
                // other group never reads: no meeting between the groups.
                if (FORM == kDKDV) ptx::tmem_st16_nowait(t_s + h * kHalf + part * 48, pk_p);
                ptx::tmem_st16_nowait(t_dp + h * kHalf + part * 48, pk_ds);
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                ptx::mbar_arrive(ptx::smem_addr(&sm.p_full[h]));
            }
        }
        if (FORM == kDQ) {
            // The next unit's resident rows go in as soon as this unit's
            // S/dP are done, so its first S/dP run during this epilogue.
            int32_t u2 = u + gridDim.x;
            Unit V;
            for (; u2 < S.n_units; u2 += gridDim.x) {
                V = decode_unit<FORM>(p, S, u2);
                if (V.n_a + V.n_b != 0) break;
            }
            if (u2 < S.n_units) {
                if (!__all_sync(kAll, wait_phase(sm, sm.x_empty, unit_iter & 1,
                                                 kErrTimeoutSoftmax)))
                    return;
                write_resident(V);
                resident_ready = true;
            }
        }
        // Epilogue: accumulators -> bf16 rows.
        if (!__all_sync(kAll, wait_phase(sm, sm.acc_full, unit_iter & 1, kErrTimeoutSoftmax)))
            return;
        ptx::tc_fence_after();
        const int side = U.detail ? 0 : 1;
        const int64_t out_row = static_cast<int64_t>(U.b) * (U.detail ? p.N : p.G) +
                                (valid ? row : 0);
        // DQ: warpgroup g stores columns [g*HD/2, (g+1)*HD/2) of dQ * scale;
        // DKDV: warpgroup 0 stores dV, warpgroup 1 stores dK * scale.
        {
            const int a = FORM == kDQ ? 0 : part;
            const float f = (FORM == kDQ || a == 1) ? p.scale : 1.f;
            __nv_bfloat16 *out = (a == 0 ? p.out0[side] : p.out1[side]);
            const int col0 = FORM == kDQ ? part * (HD / 2) : 0;
            const int ncol = FORM == kDQ ? HD / 2 : HD;
            uint4 *dst = reinterpret_cast<uint4 *>(out + (out_row * p.heads + U.head) * HD +
                                                   col0);
#pragma unroll 1
            for (int c = 0; c < ncol / 32; ++c) {
                uint32_t o[32];
                ptx::tmem_ld32(t_acc + a * HD + col0 + c * 32, o);
                if (valid && p.o_v8) {
                    // two 32-byte stores per 32 columns: whole sectors
#pragma unroll
                    for (int v = 0; v < 2; ++v) {
                        uint32_t w8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            w8[e] = ptx::pack_bf16x2(__uint_as_float(o[16 * v + 2 * e]) * f,
                                                     __uint_as_float(o[16 * v + 2 * e + 1]) * f);
                        ptx::st_global_v8(reinterpret_cast<uint8_t *>(dst) + c * 64 + v * 32, w8);
                    }
                } else if (valid) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 0]) * f,
                                               __uint_as_float(o[8 * v + 1]) * f);
                        w.y = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * f,
                                               __uint_as_float(o[8 * v + 3]) * f);
                        w.z = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * f,
                                               __uint_as_float(o[8 * v + 5]) * f);
                        w.w = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * f,
                                               __uint_as_float(o[8 * v + 7]) * f);
                        dst[c * 4 + v] = w;
                    }
                }
            }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&sm.acc_empty));
        ++unit_iter;
    }
}

template <int HD, int FORM>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem<HD> &sm = *reinterpret_cast<Smem<HD> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        ptx::mbar_init(ptx::smem_addr(&sm.x_full), FORM == kDQ ? kCompute : 1);
        ptx::mbar_init(ptx::smem_addr(&sm.x_empty), 1);
        for (int s = 0; s < Smem<HD>::kStages; ++s) {
            ptx::mbar_init(ptx::smem_addr(&sm.st_full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.st_empty[s]), 1);
        }
        for (int h = 0; h < 2; ++h) {
            ptx::mbar_init(ptx::smem_addr(&sm.s_full[h]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.p_full[h]), kCompute);
        }
        ptx::mbar_init(ptx::smem_addr(&sm.acc_full), 1);
        ptx::mbar_init(ptx::smem_addr(&sm.acc_empty), kCompute);
        ptx::mbar_init(ptx::smem_addr(&sm.drain), 1);
        sm.abort = 0;
        sm.max_len = 0;
        sm.err_word = p.err_word;
        ptx::fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_addr(&sm.tmem_base), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::prefetch_tmap(&p.tm_q[i]);
            ptx::prefetch_tmap(&p.tm_k[i]);
            ptx::prefetch_tmap(&p.tm_v[i]);
            ptx::prefetch_tmap(&p.tm_do[i]);
            ptx::prefetch_tmap(&p.hm_q[i]);
            ptx::prefetch_tmap(&p.hm_k[i]);
            ptx::prefetch_tmap(&p.hm_v[i]);
            ptx::prefetch_tmap(&p.hm_do[i]);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (p.upw < 0) {
        // The longest window: one pass over the offsets per CTA.
        int32_t m = 0;
        for (int32_t w = threadIdx.x; w < p.n_win; w += kThreads) {
            int32_t s, e;
            window_rows(p, w, s, e);
            m = max(m, e - s);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) atomicMax(&sm.max_len, m);
        __syncthreads();
    }
    const Sched S = make_sched(p, sm.max_len);
    const uint32_t tmem = sm.tmem_base;
    const bool tmem_ok = tmem == 0;   // a 512-column allocation starts at column 0
    if (!tmem_ok && threadIdx.x == 0) atomicOr(p.err_word, kErrTmemAlloc);
    if (tmem_ok) {
        if (warp < 8) compute<HD, FORM>(p, S, sm, tmem);
        else if (warp == kProducerWarp) producer<HD, FORM>(p, S, sm);
        else if (lane == 0) mma_issuer<HD, FORM>(p, S, sm, tmem);
    }
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
template <int HD, int FORM>
atlas_status launch_form(Params p, const DeviceInfo &dev, cudaStream_t stream) {
    const size_t smem = sizeof(Smem<HD>) + 1024;
    if (!set_smem_limit(reinterpret_cast<const void *>(attn_bwd_tc_kernel<HD, FORM>),
                        static_cast<int>(smem)))
        return ATLAS_ERR_CUDA;
    const int64_t per_prob = static_cast<int64_t>(p.tiles_d) + p.tiles_g;
    int64_t units = per_prob * p.batch * p.heads;
    if (units == 0) return ATLAS_OK;
    if (units > INT32_MAX) return ATLAS_ERR_SHAPE;
    // Unit form: tiles of their own for windows of at least 128 rows. Fixed
    // windows decide here (their slots never exceed three times the packed
    // count); offsets are read by the kernel only.
    if (p.N == 0) {
        p.upw = 0;
    } else if (p.win_off != nullptr) {
        p.upw = -1;
        units = std::max<int64_t>(units, dev.sm_count);
    } else {
        p.upw = p.L >= kRows ? (p.L + kRows - 1) / kRows : 0;
        if (p.upw > 0)
            units = (static_cast<int64_t>(p.N / p.L) * p.upw + p.tiles_g) * p.batch * p.heads;
        if (units > INT32_MAX) return ATLAS_ERR_SHAPE;
    }
    p.n_long = FORM == kDKDV ? p.tiles_g * p.batch * p.heads : 0;
    uintptr_t ptr_bits = 0;
    for (int i = 0; i < 2; ++i)
        ptr_bits |= reinterpret_cast<uintptr_t>(p.out0[i]) |
                    (FORM == kDKDV ? reinterpret_cast<uintptr_t>(p.out1[i]) : 0);
    p.o_v8 = (ptr_bits & 31) == 0;
    const int grid = static_cast<int>(std::min<int64_t>(units, dev.sm_count));
    if (log_enabled())
        log_launch(FORM == kDQ ? "attn_bwd_tc_kernel<dQ>" : "attn_bwd_tc_kernel<dK/dV>", grid,
                   kThreads, smem, "head_dim %d units %lld (global-key units %d) batch %d heads %d "
                   "n_detail %d n_global %d", HD, static_cast<long long>(units), p.n_long, p.batch,
                   p.heads, p.N, p.G);
    attn_bwd_tc_kernel<HD, FORM><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

template <int HD>
atlas_status launch_hd(const AttnBwdArgs &b, const DeviceInfo &dev, cudaStream_t stream) {
    const AttnArgs &a = b.fwd;
    Params p{};
    const bool has_d = a.n_detail > 0, has_g = a.n_global > 0;
    const int64_t nd = a.n_detail * a.batch, ng = a.n_global * a.batch;
    // Maps of an absent side point at the other side; they are never used.
    const void *src[2][4] = {{a.q_d, a.k_d, a.v_d, b.do_d}, {a.q_g, a.k_g, a.v_g, b.do_g}};
    const int64_t rows[2] = {nd, ng};
    CUtensorMap *maps[4] = {p.tm_q, p.tm_k, p.tm_v, p.tm_do};
    CUtensorMap *half_maps[4] = {p.hm_q, p.hm_k, p.hm_v, p.hm_do};
    for (int side = 0; side < 2; ++side) {
        const int use = (side == 0 ? has_d : has_g) ? side : 1 - side;
        for (int t = 0; t < 4; ++t)
            if (!make_rows_map(&maps[t][side], src[use][t], rows[use], a.heads, HD, kRows) ||
                !make_rows_map(&half_maps[t][side], src[use][t], rows[use], a.heads, HD, kHalf))
                return ATLAS_ERR_CUDA;
    }
    p.lse = a.lse;
    p.delta = b.delta;
    p.err_word = device_error_word();
    if (!p.err_word) return ATLAS_ERR_CUDA;
    p.N = static_cast<int32_t>(a.n_detail);
    p.L = static_cast<int32_t>(has_d ? a.window_len : 1);
    p.G = static_cast<int32_t>(a.n_global);
    p.heads = a.heads;
    p.batch = static_cast<int32_t>(a.batch);
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.win_off = a.win_off;
    p.gwin_off = a.gwin_off;
    p.n_win = static_cast<int32_t>(a.win_off ? a.n_win : a.n_gwin);
    p.tiles_d = static_cast<int32_t>((a.n_detail + kRows - 1) / kRows);
    p.tiles_g = static_cast<int32_t>((a.n_global + kRows - 1) / kRows);
    Params pq = p;
    pq.out0[0] = static_cast<__nv_bfloat16 *>(b.dq_d);
    pq.out0[1] = static_cast<__nv_bfloat16 *>(b.dq_g);
    pq.res_x[0] = static_cast<const __nv_bfloat16 *>(a.q_d);
    pq.res_x[1] = static_cast<const __nv_bfloat16 *>(a.q_g);
    pq.res_y[0] = static_cast<const __nv_bfloat16 *>(b.do_d);
    pq.res_y[1] = static_cast<const __nv_bfloat16 *>(b.do_g);
    atlas_status st = launch_form<HD, kDQ>(pq, dev, stream);
    if (st != ATLAS_OK) return st;
    Params pk = p;
    pk.out0[0] = static_cast<__nv_bfloat16 *>(b.dv_d);
    pk.out0[1] = static_cast<__nv_bfloat16 *>(b.dv_g);
    pk.out1[0] = static_cast<__nv_bfloat16 *>(b.dk_d);
    pk.out1[1] = static_cast<__nv_bfloat16 *>(b.dk_g);
    return launch_form<HD, kDKDV>(pk, dev, stream);
}

}  // namespace

atlas_status launch_attn_bwd_tc_bf16(const AttnBwdArgs &b, cudaStream_t stream) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    if (b.fwd.head_dim == 128) return launch_hd<128>(b, dev, stream);
    if (b.fwd.head_dim == 64) return launch_hd<64>(b, dev, stream);
    return ATLAS_ERR_UNSUPPORTED;
}

}  // namespace atlas
