// attn_tc.cu -- asymmetric local-global attention, bf16, tcgen05 + TMA + TMEM.
//
// Passages: "Technische Samenvatting: AtlasVid" (gist.science), Methodologie
// 1, Fase 2 (window attention over the cube-reordered sequence) and
// Methodologie 2 (asymmetric hierarchical attention: a detail query sees the
// keys of its own cube and every global-proxy key; a global query sees only
// global keys; global -> detail is masked with -inf).
//
// One softmax per query row over its allowed keys, flash style:
//   * a work unit is one head of one problem (a batch stacks problems along
//     the rows) and up to 256 query rows (two 128-row Q tiles), either detail
//     rows (cube order) or global rows;
//   * windows of at least 128 rows get units of their own ("window units"):
//     a fixed number of 256-row slots per window, the last one partly filled,
//     slots past a shorter window's end skipped, so a unit never reads keys
//     of a neighbouring window even when windows are not multiples of 256
//     rows (partial cubes shift every later window off the 256-row grid);
//     shorter windows pack 256 consecutive rows per unit, and the key list
//     is then the union of their windows, cut by per-row masks;
//   * a unit's key list is its window's detail rows (128-key tiles from the
//     window's start), then the global keys of its problem: all of them, or
//     in the aligned variant its window's range (the union of its windows'
//     ranges for packed units);
//   * windows are L rows or the ranges of an offsets array (partial cubes);
//     ranges from offsets are clamped so that any offsets keep every access
//     in bounds; with offsets the kernel finds the longest window itself
//     (every CTA scans the offsets once) and chooses the unit form;
//   * persistent CTAs (one per SM) walk the units head-major, so the CTAs in
//     flight share one head's global K/V in L2.
// Warp roles per CTA (384 threads):
//   warps 0-3 / 4-7  softmax + epilogue of Q tile 0 / 1 (thread = one row =
//                    one TMEM lane),
//   warp 8           TMA producer (Q tiles, then K and V tiles into a ring of
//                    shared-memory slots, in the order the MMAs use them),
//   warp 9           tensor-memory owner and MMA issuer (one thread),
//   warps 10-11      idle (complete the third warpgroup for the register split).
// Tensor memory (512 columns): S0 | S1 | O0 | O1 (fp32). The softmax writes
// P (bf16) over the first half of its S columns and the P*V MMA reads it from
// tensor memory, so P costs no shared-memory traffic. The MMA issue order per
// key tile j is
//   O0 += P0(j) V(j), S0(j+1), O1 += P1(j) V(j), S1(j+1).
// MMAs issued by one thread execute in order: S_i(j+1) overwrites P_i(j) only
// after O_i += P_i(j) V(j) has read it, and a commit after S_i(j+1) also
// covers O_i += P_i(j) V(j). Each softmax therefore has the time of the other
// tile's two MMAs to produce its P. A key tile whose keys end within its first
// 32 or 64 columns for every row of the unit gets S and P*V MMAs of that width
// only (and, in the NARROW form of the kernel, a softmax of that width). The Q tiles are released right after the unit's last S MMA, so the
// next unit's Q loads during the last P*V and the epilogue.
// Every wait is bounded: on expiry a bit is set in the device error word,
// the CTA drains its in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>
#include <type_traits>

#include "atlas_internal.cuh"
#include "sm100_ptx.cuh"

namespace atlas {

// ---------------------------------------------------------------------------
// Tensor maps (host).
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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
    return fn;
}

bool make_rows_map(CUtensorMap *m, const void *base, int64_t rows, int heads, int hd,
                   int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(hd), static_cast<cuuint64_t>(heads),
                          static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(hd) * 2,
                             static_cast<cuuint64_t>(heads) * hd * 2};
    cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

namespace {

constexpr int kBM = 128;          // query rows per Q tile
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kQTiles = 2;        // Q tiles per CTA (one per softmax warpgroup)
constexpr int kUnitRows = kBM * kQTiles;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 384;     // three warpgroups
// Register split (setmaxnreg): the launch gives 168 per thread (3 warps per
// SM sub-partition x 168 <= 512); the two softmax warpgroups take 200 and the
// third warpgroup (producer, MMA issuer, two idle warps) keeps 104:
// 256*200 + 128*104 = 384*168, and per sub-partition 2*200 + 104 <= 512.
constexpr uint32_t kRegsSoftmax = 200;
constexpr uint32_t kRegsOther = 104;
static_assert(256 * kRegsSoftmax + 128 * kRegsOther == kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays <= 2^8

template <int HD>
struct Smem {
    static constexpr int kTileBytes = kBM * HD * 2;           // one 128-row bf16 tile
    static constexpr int kSlots = (160 * 1024) / kTileBytes;  // K/V ring: 160 KB
    alignas(1024) uint8_t q[kQTiles][kTileBytes];
    alignas(1024) uint8_t kv[kSlots][kTileBytes];
    uint64_t q_full[kQTiles];
    uint64_t q_empty;
    uint64_t kv_full[kSlots];
    uint64_t kv_empty[kSlots];
    uint64_t s_full[kQTiles];    // S_i(j) is in TMEM (and O_i += P_i(j-1)V done)  (commit)
    uint64_t p_full[kQTiles];    // P_i(j) in TMEM, O_i rescaled         (128 arrivals)
    uint64_t o_final[kQTiles];   // every MMA of the unit done           (commit)
    uint64_t drain;
    uint32_t tmem_base;
    int32_t max_len;     // longest window, from the offsets
    volatile int abort;
    uint32_t *err_word;
};

struct Params {
    CUtensorMap tm_qd, tm_kd, tm_vd, tm_qg, tm_kg, tm_vg;
    __nv_bfloat16 *o_d, *o_g;
    float *lse;
    uint32_t *err_word;
    int32_t N, L, G, heads;  // N, G: detail and global rows of ONE problem
    float scale_log2;
    int32_t n_dunits, n_gunits;          // packed-form units of one problem
    int32_t batch, n_gtiles;
    int32_t upw;          // window units per window; 0: packed units; -1: from the offsets
    int32_t stall_unit;   // test hook: this unit's first K tile is never loaded (-1: off)
    int32_t o_v8;         // both outputs 32-byte aligned: the epilogue stores 32 B at a time
    const int32_t *win_off;   // window offsets [n_win + 1] of one problem (NULL: L rows)
    const int32_t *gwin_off;  // global key offsets [n_win + 1] per window (NULL: all keys)
    int32_t n_win;
};

// The window holding detail row x (of one problem).
__device__ __forceinline__ int32_t window_of(const Params &p, int32_t x) {
    if (p.win_off == nullptr) return x / p.L;
    int32_t lo = 0, hi = p.n_win - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (__ldg(p.win_off + mid) <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}
// Row range [start, end) of window w, which holds row x. With offsets the
// range is clamped to [0, N) and to contain x, so that offsets other than
// described still keep every access in bounds.
__device__ __forceinline__ int32_t window_start(const Params &p, int32_t w, int32_t x) {
    return p.win_off == nullptr ? w * p.L : min(max(__ldg(p.win_off + w), 0), x);
}
__device__ __forceinline__ int32_t window_end(const Params &p, int32_t w, int32_t x) {
    return p.win_off == nullptr ? min(p.N, (w + 1) * p.L)
                                : max(min(__ldg(p.win_off + w + 1), p.N), x + 1);
}
// Global keys [start, end) seen by the queries of window w (one problem).
__device__ __forceinline__ int32_t global_start(const Params &p, int32_t w) {
    return p.gwin_off == nullptr ? 0 : min(max(__ldg(p.gwin_off + w), 0), p.G);
}
__device__ __forceinline__ int32_t global_end(const Params &p, int32_t w, int32_t start) {
    return p.gwin_off == nullptr ? p.G : min(max(__ldg(p.gwin_off + w + 1), start), p.G);
}

// The unit form and counts, the same in every thread of every CTA.
struct Sched {
    int32_t upw, n_dunits, units_per_prob, units_per_head, n_units;
};

// max_len: the longest window (clamped ranges of the offsets), when p.upw < 0.
__device__ __forceinline__ Sched make_sched(const Params &p, int32_t max_len) {
    Sched S;
    S.upw = p.upw;
    if (S.upw < 0) {
        // Window units when windows are long enough, and their slots stay
        // within three times the packed count (offsets mixing a long window
        // with many short ones would otherwise make mostly empty units).
        const int64_t upw = (max_len + kUnitRows - 1) / kUnitRows;
        const int64_t n = static_cast<int64_t>(p.n_win) * upw;
        const bool ok = max_len >= kBM && n <= 3 * static_cast<int64_t>(p.n_dunits) &&
                        (n + p.n_gunits) * p.batch * p.heads <= INT32_MAX;
        S.upw = ok ? static_cast<int32_t>(upw) : 0;
    }
    const int32_t n_win = p.win_off != nullptr ? p.n_win : (p.L > 0 ? p.N / p.L : 0);
    S.n_dunits = S.upw > 0 ? n_win * S.upw : p.n_dunits;
    S.units_per_prob = S.n_dunits + p.n_gunits;
    S.units_per_head = S.units_per_prob * p.batch;
    S.n_units = S.units_per_head * p.heads;
    return S;
}

// Work unit: one head, one problem of the batch, up to kUnitRows query rows.
// Rows are per problem: rows q0 .. qend-1 are the unit's; row0 is the
// problem's first row in the stacked tensors; kw0 / kg0 are absolute first
// key rows. A window unit (win >= 0) has one key range for all its rows:
// detail [kw0, whi), global [kg0, ghi). n_tiles == 0: an empty slot.
struct Unit {
    int32_t head, detail, b, q0, qend, row0, kw0, n_wtiles, kg0, n_tiles, win, whi, ghi;
};

__device__ __forceinline__ Unit decode_unit(const Params &p, const Sched &S, int32_t u) {
    Unit U;
    U.head = u / S.units_per_head;
    int32_t lu = u - U.head * S.units_per_head;
    U.b = lu / S.units_per_prob;
    lu -= U.b * S.units_per_prob;
    U.detail = lu < S.n_dunits;
    int32_t n_gtiles = p.n_gtiles;
    U.kg0 = U.b * p.G;
    U.ghi = U.kg0 + p.G;
    U.win = -1;
    U.whi = 0;
    if (U.detail && S.upw > 0) {
        const int32_t w = lu / S.upw, sub = lu - w * S.upw;
        int32_t s, e;
        if (p.win_off != nullptr) {
            s = min(max(__ldg(p.win_off + w), 0), p.N);
            e = min(max(__ldg(p.win_off + w + 1), s), p.N);
        } else {
            s = w * p.L;
            e = min(p.N, s + p.L);
        }
        U.row0 = U.b * p.N;
        U.q0 = s + sub * kUnitRows;
        U.qend = min(U.q0 + kUnitRows, e);
        U.kw0 = U.row0 + s;
        U.whi = U.row0 + e;
        U.n_wtiles = (e - s + kBN - 1) / kBN;
        U.win = w;
        if (p.gwin_off != nullptr) {
            const int32_t g0 = global_start(p, w), g1 = global_end(p, w, g0);
            U.kg0 += g0;
            U.ghi = U.b * p.G + g1;
            n_gtiles = (g1 - g0 + kBN - 1) / kBN;
        }
        if (U.qend <= U.q0) U.n_wtiles = n_gtiles = 0;
    } else if (U.detail) {
        U.q0 = lu * kUnitRows;
        U.qend = min(U.q0 + kUnitRows, p.N);
        U.row0 = U.b * p.N;
        const int32_t q_last = min(U.q0 + kUnitRows, p.N) - 1;
        const int32_t w0 = window_of(p, U.q0), w1 = window_of(p, q_last);
        U.kw0 = U.row0 + window_start(p, w0, U.q0);
        const int32_t kw1 = U.row0 + window_end(p, w1, q_last);
        U.n_wtiles = (kw1 - U.kw0 + kBN - 1) / kBN;
        U.whi = kw1;
        if (p.gwin_off != nullptr) {
            const int32_t g0 = global_start(p, w0), g1 = global_end(p, w1, g0);
            U.kg0 += g0;
            U.ghi = U.b * p.G + g1;
            n_gtiles = (g1 - g0 + kBN - 1) / kBN;
        }
    } else {
        U.q0 = (lu - S.n_dunits) * kUnitRows;
        U.qend = min(U.q0 + kUnitRows, p.G);
        U.row0 = U.b * p.G;
        U.kw0 = 0;
        U.n_wtiles = 0;
    }
    U.n_tiles = U.n_wtiles + n_gtiles;
    return U;
}

// Window units with offsets: bring the offsets decode_unit(u) reads into L1,
// so that decoding the next unit after an epilogue costs no trip to L2.
__device__ __forceinline__ void prefetch_unit(const Params &p, const Sched &S, int32_t u) {
    if (u >= S.n_units || S.upw <= 0 || p.win_off == nullptr) return;
    int32_t lu = u - (u / S.units_per_head) * S.units_per_head;
    lu -= (lu / S.units_per_prob) * S.units_per_prob;
    if (lu >= S.n_dunits) return;
    const int32_t w = lu / S.upw;
    ptx::prefetch_l1(p.win_off + w);
    ptx::prefetch_l1(p.win_off + w + 1);
    if (p.gwin_off != nullptr) {
        ptx::prefetch_l1(p.gwin_off + w);
        ptx::prefetch_l1(p.gwin_off + w + 1);
    }
}

// Bounded wait. Returns false (after flagging `err`) if the phase did not
// complete within the limit or another role of this CTA aborted.
template <int HD>
__device__ __forceinline__ bool wait_phase(Smem<HD> &sm, uint64_t &bar, uint32_t parity,
                                           uint32_t err, bool honor_abort = true) {
    const uint32_t a = ptx::smem_addr(&bar);
    if (ptx::mbar_try_wait(a, parity)) return true;
    uint64_t t0 = global_timer_ns();
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

// Key tile j of unit U: first row and whether it is a window (detail) tile.
__device__ __forceinline__ int32_t key_row(const Unit &U, int32_t j) {
    return j < U.n_wtiles ? U.kw0 + j * kBN : U.kg0 + (j - U.n_wtiles) * kBN;
}
// Columns of key tile j that can hold a key allowed to some row of the unit:
// 32, 64 or all kBN. A narrow tile's S = Q K^T is computed for those columns
// only and its P*V reads only them; the S columns beyond are stale and never
// read.
__device__ __forceinline__ int32_t tile_cols(const Unit &U, int32_t j) {
    const int32_t n = j < U.n_wtiles ? U.whi - (U.kw0 + j * kBN)
                                      : U.ghi - (U.kg0 + (j - U.n_wtiles) * kBN);
    return n <= 32 ? 32 : (n <= 64 ? 64 : kBN);
}

// ---------------------------------------------------------------------------
// Producer: Q tiles once per unit, then K(0), V(0), K(1), V(1), ... in the
// order the MMAs consume them.
// ---------------------------------------------------------------------------
template <int HD>
__device__ void producer(const Params &p, const Sched &S, Smem<HD> &sm) {
    constexpr uint32_t kBytes = Smem<HD>::kTileBytes;
    constexpr int kSlots = Smem<HD>::kSlots;
    uint32_t it = 0, unit_iter = 0;
    uint32_t q_armed = 0;
    uint32_t armed[kSlots];
#pragma unroll
    for (int s = 0; s < kSlots; ++s) armed[s] = 0;
    bool ok = true;

    auto load = [&](const CUtensorMap *map, int32_t head, int32_t row) -> bool {
        const uint32_t slot = it % kSlots, round = it / kSlots;
        if (round > 0 &&
            !wait_phase(sm, sm.kv_empty[slot], (round - 1) & 1, kErrTimeoutProducer))
            return false;
        const uint32_t bar = ptx::smem_addr(&sm.kv_full[slot]);
        ptx::mbar_arrive_expect_tx(bar, kBytes);
#pragma unroll
        for (int db = 0; db < HD / 64; ++db)
            ptx::tma_load_3d(ptx::smem_addr(sm.kv[slot] + db * kBN * 128), map, bar, db * 64,
                             head, row);
#pragma unroll
        for (int s = 0; s < kSlots; ++s)
            if (s == static_cast<int>(slot)) armed[s] = round + 1;
        ++it;
        return true;
    };

    for (int32_t u = blockIdx.x; u < S.n_units && ok; u += gridDim.x) {
        const Unit U = decode_unit(p, S, u);
        if (U.n_tiles == 0) continue;
        if (unit_iter > 0 && !(ok = wait_phase(sm, sm.q_empty, (unit_iter - 1) & 1,
                                               kErrTimeoutProducer)))
            break;
        const CUtensorMap *tq = U.detail ? &p.tm_qd : &p.tm_qg;
#pragma unroll
        for (int i = 0; i < kQTiles; ++i) {
            uint32_t bar = ptx::smem_addr(&sm.q_full[i]);
            ptx::mbar_arrive_expect_tx(bar, kBytes);
#pragma unroll
            for (int db = 0; db < HD / 64; ++db)
                ptx::tma_load_3d(ptx::smem_addr(sm.q[i] + db * kBM * 128), tq, bar, db * 64,
                                 U.head, U.row0 + U.q0 + i * kBM);
        }
        q_armed = unit_iter + 1;
        for (int32_t j = 0; j < U.n_tiles && ok; ++j) {
            const bool win = j < U.n_wtiles;
            const int32_t row = key_row(U, j);
            if (j == 0 && u == p.stall_unit) {
                // Failure-path test: leave this slot unarmed so the MMA
                // issuer's bounded wait on it expires.
                ++it;
                ok = load(win ? &p.tm_vd : &p.tm_vg, U.head, row);
                continue;
            }
            ok = load(win ? &p.tm_kd : &p.tm_kg, U.head, row) &&
                 load(win ? &p.tm_vd : &p.tm_vg, U.head, row);
        }
        ++unit_iter;
    }
    if (!ok) {
        // Let every copy already issued land before the CTA can exit.
        if (q_armed)
            for (int i = 0; i < kQTiles; ++i)
                wait_phase(sm, sm.q_full[i], (q_armed - 1) & 1, kErrTimeoutTeardown, false);
        for (int s = 0; s < kSlots; ++s)
            if (armed[s])
                wait_phase(sm, sm.kv_full[s], (armed[s] - 1) & 1, kErrTimeoutTeardown, false);
    }
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread). Per unit: S0(0), S1(0); then for each key tile j:
// O0 += P0(j)V(j), S0(j+1), O1 += P1(j)V(j), S1(j+1).
// ---------------------------------------------------------------------------
template <int HD>
__device__ void mma_issuer(const Params &p, const Sched &S, Smem<HD> &sm, uint32_t tmem) {
    constexpr int kSlots = Smem<HD>::kSlots;
    constexpr uint32_t kIdescQK = ptx::idesc_bf16_f32(kBM, kBN, 0);
    constexpr uint32_t kIdescQK64 = ptx::idesc_bf16_f32(kBM, 64, 0);
    constexpr uint32_t kIdescQK32 = ptx::idesc_bf16_f32(kBM, 32, 0);
    constexpr uint32_t kIdescPV = ptx::idesc_bf16_f32(kBM, HD, 1);
    uint32_t it = 0, unit_iter = 0;
    uint32_t p_cnt = 0;   // P tiles consumed per Q tile (both tiles move together)
    bool ok = true;

    auto next_slot = [&](uint32_t &slot) -> bool {
        slot = it % kSlots;
        const bool r = wait_phase(sm, sm.kv_full[slot], (it / kSlots) & 1, kErrTimeoutMma);
        ++it;
        ptx::tc_fence_after();
        return r;
    };
    // Descriptor words, computed once: the loops below only add constant
    // offsets (bytes >> 4) to the low word.
    constexpr uint32_t kHi = ptx::desc_sw128_hi(1024);
    const uint32_t q_lo0 = ptx::desc_sw128_lo(ptx::smem_addr(sm.q[0]), 16);
    const uint32_t k_lo0 = ptx::desc_sw128_lo(ptx::smem_addr(sm.kv[0]), 16);
    const uint32_t v_lo0 = ptx::desc_sw128_lo(ptx::smem_addr(sm.kv[0]), kBN * 128);
    constexpr uint32_t kTile16 = Smem<HD>::kTileBytes >> 4;
    // S_i = Q_i K^T from the K tile in `slot`, for the tile's first nc keys
    // (the K-major operand's first nc rows: the same descriptors).
    auto issue_s = [&](int i, uint32_t k_slot, int32_t nc) {
        const uint32_t q_lo = q_lo0 + i * kTile16, k_lo = k_lo0 + k_slot * kTile16;
        const uint32_t d_s = tmem + i * kBN;
        const uint32_t idesc = nc == kBN ? kIdescQK : (nc == 64 ? kIdescQK64 : kIdescQK32);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
            const uint32_t off = ((ks / 4) * (kBM * 128) + (ks % 4) * 32) >> 4;
            ptx::mma_ss(d_s, ptx::desc_join(q_lo + off, kHi), ptx::desc_join(k_lo + off, kHi),
                        idesc, ks > 0);
        }
        ptx::mma_commit(ptx::smem_addr(&sm.s_full[i]));
    };
    // O_i += P_i V, P_i from tensor memory, from the V tile in `slot`; the
    // first nc keys only (nc / 16 steps of K = 16).
    auto issue_pv = [&](int i, uint32_t v_slot, bool first, int32_t nc) -> bool {
        if (!wait_phase(sm, sm.p_full[i], p_cnt & 1, kErrTimeoutMma)) return false;
        ptx::tc_fence_after();
        const uint32_t v_lo = v_lo0 + v_slot * kTile16;
        const uint32_t d_o = tmem + 2 * kBN + i * HD, a_p = tmem + i * kBN;
        ptx::mma_ts(d_o, a_p, ptx::desc_join(v_lo, kHi), kIdescPV, first ? 0u : 1u);
        if (nc == kBN) {
#pragma unroll
            for (int ks = 1; ks < kBN / 16; ++ks)
                ptx::mma_ts(d_o, a_p + ks * 8,
                            ptx::desc_join(v_lo + ((ks * 16 * 128) >> 4), kHi), kIdescPV, 1u);
        } else {
#pragma unroll 1
            for (int ks = 1; ks * 16 < nc; ++ks)
                ptx::mma_ts(d_o, a_p + ks * 8,
                            ptx::desc_join(v_lo + ((ks * 16 * 128) >> 4), kHi), kIdescPV, 1u);
        }
        return true;
    };

    for (int32_t u = blockIdx.x; u < S.n_units && ok; u += gridDim.x) {
        const Unit U = decode_unit(p, S, u);
        if (U.n_tiles == 0) continue;
        for (int i = 0; i < kQTiles && ok; ++i)
            ok = wait_phase(sm, sm.q_full[i], unit_iter & 1, kErrTimeoutMma);
        if (!ok) break;
        ptx::tc_fence_after();
        uint32_t k_slot, v_slot;
        if (!(ok = next_slot(k_slot))) break;
        int32_t nc = tile_cols(U, 0);
        issue_s(0, k_slot, nc);
        issue_s(1, k_slot, nc);
        ptx::mma_commit(ptx::smem_addr(&sm.kv_empty[k_slot]));
        // Q is read by the S MMAs only: once the unit's last S is issued, a
        // commit frees it, and the next unit's Q loads during the last P*V
        // and this unit's epilogue.
        if (U.n_tiles == 1) ptx::mma_commit(ptx::smem_addr(&sm.q_empty));
        for (int32_t j = 0; j < U.n_tiles && ok; ++j) {
            const bool more = j + 1 < U.n_tiles;
            const int32_t nc_next = more ? tile_cols(U, j + 1) : 0;
            // ring order: V(j) was loaded before K(j+1)
            if (!(ok = next_slot(v_slot)) || !(ok = issue_pv(0, v_slot, j == 0, nc))) break;
            if (more) {
                if (!(ok = next_slot(k_slot))) break;
                issue_s(0, k_slot, nc_next);
            }
            if (!(ok = issue_pv(1, v_slot, j == 0, nc))) break;
            if (more) {
                issue_s(1, k_slot, nc_next);
                ptx::mma_commit(ptx::smem_addr(&sm.kv_empty[k_slot]));
                if (j + 2 == U.n_tiles) ptx::mma_commit(ptx::smem_addr(&sm.q_empty));
            }
            nc = nc_next;
            ptx::mma_commit(ptx::smem_addr(&sm.kv_empty[v_slot]));
            ++p_cnt;
        }
        if (!ok) break;
        prefetch_unit(p, S, u + gridDim.x);
        for (int i = 0; i < kQTiles; ++i) ptx::mma_commit(ptx::smem_addr(&sm.o_final[i]));
        ++unit_iter;
    }
    // Drain: every MMA issued must finish before tensor memory is freed.
    ptx::mma_commit(ptx::smem_addr(&sm.drain));
    wait_phase(sm, sm.drain, 0, kErrTimeoutTeardown, false);
}

// ---------------------------------------------------------------------------
// Softmax + epilogue of Q tile `qt`; 128 threads, thread = row = TMEM lane.
// ---------------------------------------------------------------------------
// NARROW: the softmax has 64- and 32-column forms for narrow tiles (their
// exponentials skipped); without it a narrow tile's softmax takes all 128
// columns (the masked ones give P = 0) and only its MMAs are narrow. The
// extra forms cost about 1 % on layouts whose narrow tiles are rare.
template <int HD, bool NARROW>
__device__ void softmax_epilogue(const Params &p, const Sched &S, Smem<HD> &sm, uint32_t tmem,
                                 int qt) {
    const uint32_t warp = (threadIdx.x / 32) & 3;
    const uint32_t r = threadIdx.x & 127;                 // row within the tile
    const uint32_t lane_sel = (warp * 32u) << 16;         // TMEM lane field
    const uint32_t t_s = tmem + qt * kBN + lane_sel;      // S, then P over its first half
    const uint32_t t_o = tmem + 2 * kBN + qt * HD + lane_sel;
    const uint32_t err = kErrTimeoutSoftmax;
    const float sc = p.scale_log2;
    constexpr uint32_t kAll = 0xffffffffu;

    // P = exp2(S*scale*log2e - m) of the NC columns in `sr`, as bf16 pairs
    // into tensor memory (stores of 32 packed columns; one of 16 for a
    // 32-column tile); returns the row sum of the fp32 P. WithMax: the row
    // maximum of the raw S is taken in the same pass, into mx. `between` runs
    // after the first group's store, before the second group is read.
    auto exp_store = [&](auto with_max, const auto &sr, float m, float &mx,
                         auto &&between) -> float {
        constexpr bool kWithMax = decltype(with_max)::value;
        constexpr int NC = static_cast<int>(sizeof(sr) / sizeof(uint32_t));
        constexpr int kPer = NC >= 64 ? 32 : 16;
        float sum8[8], m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            sum8[k] = 0.f;
            m8[k] = kNegInf;
        }
#pragma unroll
        for (int g = 0; g < NC / (2 * kPer); ++g) {
            uint32_t pk[kPer];
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
                const int c = g * 2 * kPer + 2 * e;
                const float s0 = __uint_as_float(sr[c]), s1 = __uint_as_float(sr[c + 1]);
                if constexpr (kWithMax) m8[e & 7] = ptx::max3(m8[e & 7], s0, s1);
                const float p0 = ptx::ex2(fmaf(s0, sc, -m));
                const float p1 = ptx::ex2(fmaf(s1, sc, -m));
                sum8[e & 7] += p0 + p1;
                pk[e] = ptx::pack_bf16x2(p0, p1);
            }
            if constexpr (kPer == 32)
                ptx::tmem_st32_nowait(t_s + g * 32, pk);
            else
                ptx::tmem_st16_nowait(t_s + g * 16, pk);
            if (g == 0) between();
        }
        ptx::tmem_wait_st();
#pragma unroll
        for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
            for (int k = 0; k < w; ++k) {
                sum8[k] += sum8[k + w];
                if constexpr (kWithMax) m8[k] = fmaxf(m8[k], m8[k + w]);
            }
        if constexpr (kWithMax) mx = m8[0];
        return sum8[0];
    };
    // Row maximum of the NC columns in `sr` (NC a multiple of 16).
    auto row_max = [&](const auto &sr) -> float {
        constexpr int NC = static_cast<int>(sizeof(sr) / sizeof(uint32_t));
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = __uint_as_float(sr[k]);
#pragma unroll
        for (int c = 8; c + 16 <= NC; c += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k)
                m8[k] = ptx::max3(m8[k], __uint_as_float(sr[c + k]), __uint_as_float(sr[c + 8 + k]));
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], __uint_as_float(sr[NC - 8 + k]));
        return ptx::max3(ptx::max3(m8[0], m8[1], m8[2]), ptx::max3(m8[3], m8[4], m8[5]),
                         fmaxf(m8[6], m8[7]));
    };
    // O *= alpha (only warps where some row moved its reference). The P*V of
    // the previous key tile has completed: the commit that signalled this S
    // covers it.
    auto rescale_o = [&](bool need, float alpha) {
        if (!__any_sync(kAll, need)) return;
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
            uint32_t o[32];
            ptx::tmem_ld32(t_o + c * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            ptx::tmem_st32(t_o + c * 32, o);
        }
    };

    uint32_t cnt = 0, unit_iter = 0;   // key tiles processed (all units)
    for (int32_t u = blockIdx.x; u < S.n_units; u += gridDim.x) {
        const Unit U = decode_unit(p, S, u);
        if (U.n_tiles == 0) continue;
        const int32_t q = U.q0 + qt * kBM + static_cast<int32_t>(r);
        const bool row_valid = q < U.qend;
        // Allowed keys (absolute rows): detail [lo, hi), global [glo, ghi).
        int32_t lo = U.kw0, hi = U.whi, glo = U.kg0, ghi = U.ghi;
        if (U.detail && U.win < 0) {
            glo = U.b * p.G;
            ghi = glo + p.G;
            const int32_t qc = min(q, p.N - 1);
            const int32_t w = window_of(p, qc);
            lo = U.row0 + window_start(p, w, qc);
            hi = U.row0 + window_end(p, w, qc);
            if (p.gwin_off != nullptr) {
                const int32_t g0 = global_start(p, w);
                ghi = U.b * p.G + global_end(p, w, g0);
                glo = U.b * p.G + g0;
            }
        }
        float m_run = kNegInf, l_run = 0.f;
        for (int32_t j = 0; j < U.n_tiles; ++j, ++cnt) {
            if (!__all_sync(kAll, wait_phase(sm, sm.s_full[qt], cnt & 1, err))) return;
            ptx::tc_fence_after();
            // Mask keys outside this row's allowed range.
            const int32_t k0 = key_row(U, j);
            const int32_t klo = j < U.n_wtiles ? lo : glo;
            const int32_t khi = j < U.n_wtiles ? hi : ghi;
            const bool row_masked = k0 < klo || k0 + kBN > khi;
            // One key tile of NC columns (all 128, or the first 64 or 32 of a
            // narrow tile: the others hold no allowed key of any row).
            auto tile = [&](auto ncw) -> float {
                constexpr int NC = decltype(ncw)::value;
                // A full tile loads its second 64 columns while the first
                // 64 are exponentiated (fast path), else before anything.
                uint32_t sr[NC];
                if constexpr (NC == 128) {
                    ptx::tmem_ld64(t_s, *reinterpret_cast<uint32_t(*)[64]>(&sr[0]));
                    ptx::tmem_ld64_nowait(t_s + 64, *reinterpret_cast<uint32_t(*)[64]>(&sr[64]));
                } else if constexpr (NC == 64) {
                    ptx::tmem_ld64(t_s, sr);
                } else {
                    ptx::tmem_ld32(t_s, sr);
                }
                auto wait_hi = [&] {
                    if constexpr (NC == 128)
                        ptx::tmem_wait_ld(*reinterpret_cast<uint32_t(*)[64]>(&sr[64]));
                };
                auto nothing = [] {};
                float sum, mx;
                if (__any_sync(kAll, m_run == kNegInf || row_masked)) {
                    wait_hi();
                    if (row_masked) {
#pragma unroll
                        for (int c = 0; c < NC; ++c)
                            if (k0 + c < klo || k0 + c >= khi) sr[c] = __float_as_uint(kNegInf);
                    }
                    // No reference yet, or masked keys: row max first. The
                    // reference moves only when the tile's max exceeds it by
                    // more than the threshold (exact either way: O and l
                    // share it).
                    const float mx2 = row_max(sr) * sc;
                    const bool need = (m_run == kNegInf) ? (mx2 != kNegInf)
                                                         : (mx2 > m_run + kRescaleThreshold);
                    float alpha = 1.f;
                    if (need) {
                        alpha = (m_run == kNegInf) ? 0.f : ptx::ex2(m_run - mx2);
                        m_run = mx2;
                    }
                    l_run *= alpha;
                    if (j > 0) rescale_o(need, alpha);
                    sum = exp_store(std::false_type{}, sr, m_run == kNegInf ? 0.f : m_run, mx,
                                    nothing);
                } else {
                    // Exponentials against the running reference right away,
                    // the tile max in the same pass; redo the (rare) rows
                    // whose max moved past the threshold.
                    sum = exp_store(std::true_type{}, sr, m_run, mx, wait_hi);
                    const float mx2 = mx * sc;
                    const bool need = mx2 > m_run + kRescaleThreshold;
                    if (__any_sync(kAll, need)) {
                        const float alpha = need ? ptx::ex2(m_run - mx2) : 1.f;
                        if (need) m_run = mx2;
                        l_run *= alpha;
                        rescale_o(need, alpha);
                        sum = exp_store(std::false_type{}, sr, m_run, mx, nothing);
                    }
                }
                return sum;
            };
            float sum;
            if constexpr (NARROW) {
                const int32_t nc = tile_cols(U, j);
                sum = nc == kBN ? tile(std::integral_constant<int, kBN>{})
                      : nc == 64 ? tile(std::integral_constant<int, 64>{})
                                 : tile(std::integral_constant<int, 32>{});
            } else {
                sum = tile(std::integral_constant<int, kBN>{});
            }
            l_run += sum;
            ptx::tc_fence_before();
            ptx::mbar_arrive(ptx::smem_addr(&sm.p_full[qt]));
        }
        // Epilogue: O / l -> bf16 rows; LSE.
        if (r == 0) prefetch_unit(p, S, u + gridDim.x);
        if (!__all_sync(0xffffffffu, wait_phase(sm, sm.o_final[qt], unit_iter & 1, err)))
            return;
        ptx::tc_fence_after();
        const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
        __nv_bfloat16 *out = U.detail ? p.o_d : p.o_g;
        uint4 *dst = reinterpret_cast<uint4 *>(
            out + (static_cast<int64_t>(U.row0 + (row_valid ? q : 0)) * p.heads + U.head) * HD);
        // The whole O row in one load and one wait, then bf16 stores.
        uint32_t o[HD];
        if constexpr (HD == 128)
            ptx::tmem_ld128(t_o, o);
        else
            ptx::tmem_ld64(t_o, o);
        if (row_valid && p.o_v8) {
            // 32-byte stores: whole sectors
#pragma unroll
            for (int v = 0; v < HD / 16; ++v) {
                uint32_t w8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w8[e] = ptx::pack_bf16x2(__uint_as_float(o[16 * v + 2 * e]) * inv_l,
                                             __uint_as_float(o[16 * v + 2 * e + 1]) * inv_l);
                ptx::st_global_v8(reinterpret_cast<uint8_t *>(dst) + v * 32, w8);
            }
        } else if (row_valid) {
#pragma unroll
            for (int v = 0; v < HD / 8; ++v) {
                uint4 w;
                w.x = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l,
                                       __uint_as_float(o[8 * v + 1]) * inv_l);
                w.y = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l,
                                       __uint_as_float(o[8 * v + 3]) * inv_l);
                w.z = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l,
                                       __uint_as_float(o[8 * v + 5]) * inv_l);
                w.w = ptx::pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l,
                                       __uint_as_float(o[8 * v + 7]) * inv_l);
                dst[v] = w;
            }
        }
        if (p.lse != nullptr && row_valid) {
            const int64_t col = U.detail ? q : static_cast<int64_t>(p.N) + q;
            p.lse[(static_cast<int64_t>(U.b) * p.heads + U.head) * (p.N + p.G) + col] =
                (m_run + __log2f(l_run)) * 0.69314718055994531f;
        }
        ptx::tc_fence_before();
        ++unit_iter;
    }
}

template <int HD, bool NARROW>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem<HD> &sm = *reinterpret_cast<Smem<HD> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t warp = threadIdx.x / 32, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kQTiles; ++i) {
            ptx::mbar_init(ptx::smem_addr(&sm.q_full[i]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.s_full[i]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.p_full[i]), kBM);
            ptx::mbar_init(ptx::smem_addr(&sm.o_final[i]), 1);
        }
        ptx::mbar_init(ptx::smem_addr(&sm.q_empty), 1);
        for (int s = 0; s < Smem<HD>::kSlots; ++s) {
            ptx::mbar_init(ptx::smem_addr(&sm.kv_full[s]), 1);
            ptx::mbar_init(ptx::smem_addr(&sm.kv_empty[s]), 1);
        }
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
        ptx::prefetch_tmap(&p.tm_qd);
        ptx::prefetch_tmap(&p.tm_kd);
        ptx::prefetch_tmap(&p.tm_vd);
        ptx::prefetch_tmap(&p.tm_qg);
        ptx::prefetch_tmap(&p.tm_kg);
        ptx::prefetch_tmap(&p.tm_vg);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (p.upw < 0) {
        // The longest window: one pass over the offsets per CTA.
        int32_t m = 0;
        for (int32_t w = threadIdx.x; w < p.n_win; w += kThreads) {
            const int32_t s = min(max(__ldg(p.win_off + w), 0), p.N);
            m = max(m, min(max(__ldg(p.win_off + w + 1), s), p.N) - s);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) atomicMax(&sm.max_len, m);
        __syncthreads();
    }
    const Sched S = make_sched(p, sm.max_len);
    const uint32_t tmem = sm.tmem_base;
    // A 512-column allocation always starts at column 0 of lane 0.
    const bool tmem_ok = tmem == 0;
    if (!tmem_ok && threadIdx.x == 0) {
        atomicOr(p.err_word, kErrTmemAlloc);
    }

    if (warp < 8) {
        ptx::setmaxnreg_inc<kRegsSoftmax>();
        if (tmem_ok) softmax_epilogue<HD, NARROW>(p, S, sm, tmem, warp / 4);
    } else {
        ptx::setmaxnreg_dec<kRegsOther>();
        if (tmem_ok && lane == 0) {
            if (warp == kProducerWarp) producer<HD>(p, S, sm);
            if (warp == kMmaWarp) mma_issuer<HD>(p, S, sm, tmem);
        }
    }
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

template <int HD>
atlas_status launch_hd(const AttnArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    Params p{};
    const bool has_d = a.n_detail > 0, has_g = a.n_global > 0;
    // Maps for an absent side point at the other side; they are never used.
    const void *qd = has_d ? a.q_d : a.q_g, *kd = has_d ? a.k_d : a.k_g,
               *vd = has_d ? a.v_d : a.v_g;
    const void *qg = has_g ? a.q_g : a.q_d, *kg = has_g ? a.k_g : a.k_d,
               *vg = has_g ? a.v_g : a.v_d;
    const int64_t nd = (has_d ? a.n_detail : a.n_global) * a.batch,
                  ng = (has_g ? a.n_global : a.n_detail) * a.batch;
    if (!make_rows_map(&p.tm_qd, qd, nd, a.heads, HD) ||
        !make_rows_map(&p.tm_kd, kd, nd, a.heads, HD) ||
        !make_rows_map(&p.tm_vd, vd, nd, a.heads, HD) ||
        !make_rows_map(&p.tm_qg, qg, ng, a.heads, HD) ||
        !make_rows_map(&p.tm_kg, kg, ng, a.heads, HD) ||
        !make_rows_map(&p.tm_vg, vg, ng, a.heads, HD))
        return ATLAS_ERR_CUDA;
    p.o_d = static_cast<__nv_bfloat16 *>(a.o_d);
    p.o_g = static_cast<__nv_bfloat16 *>(a.o_g);
    p.lse = a.lse;
    p.err_word = device_error_word();
    if (!p.err_word) return ATLAS_ERR_CUDA;
    p.N = static_cast<int32_t>(a.n_detail);
    p.L = static_cast<int32_t>(has_d ? a.window_len : 1);
    p.G = static_cast<int32_t>(a.n_global);
    p.heads = a.heads;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.n_dunits = static_cast<int32_t>((a.n_detail + kUnitRows - 1) / kUnitRows);
    p.n_gunits = static_cast<int32_t>((a.n_global + kUnitRows - 1) / kUnitRows);
    const int64_t packed_units = static_cast<int64_t>(p.n_dunits) + p.n_gunits;
    if (packed_units == 0) return ATLAS_OK;
    if (packed_units * a.batch * a.heads > INT32_MAX) return ATLAS_ERR_SHAPE;
    p.batch = static_cast<int32_t>(a.batch);
    p.n_gtiles = static_cast<int32_t>((a.n_global + kBN - 1) / kBN);
    p.stall_unit = take_stall_request() ? 0 : -1;
    p.o_v8 = ((reinterpret_cast<uintptr_t>(a.o_d) | reinterpret_cast<uintptr_t>(a.o_g)) & 31) == 0;
    p.win_off = a.win_off;
    p.gwin_off = a.gwin_off;
    p.n_win = static_cast<int32_t>(a.win_off ? a.n_win : a.n_gwin);
    // Unit form: window units for windows of at least one Q tile. Fixed
    // windows decide here (their slots never exceed three times the packed
    // count); offsets are read by the kernel only.
    int64_t n_units = packed_units * a.batch * a.heads;
    if (!has_d) {
        p.upw = 0;
    } else if (a.win_off != nullptr) {
        p.upw = -1;
        n_units = std::max<int64_t>(n_units, dev.sm_count);
    } else {
        p.upw = p.L >= kBM ? (p.L + kUnitRows - 1) / kUnitRows : 0;
        if (p.upw > 0)
            n_units = (static_cast<int64_t>(p.N / p.L) * p.upw + p.n_gunits) * a.batch * a.heads;
        if (n_units > INT32_MAX) return ATLAS_ERR_SHAPE;
    }
    // Narrow softmax forms where narrow tiles are frequent: per-window global
    // ranges (aligned proxy tokens) or variable windows (partial cubes).
    const bool narrow = a.win_off != nullptr || a.gwin_off != nullptr;
    const void *fn = narrow ? reinterpret_cast<const void *>(attn_tc_kernel<HD, true>)
                            : reinterpret_cast<const void *>(attn_tc_kernel<HD, false>);
    const size_t smem = sizeof(Smem<HD>) + 1024;
    if (!set_smem_limit(fn, static_cast<int>(smem))) return ATLAS_ERR_CUDA;
    const int grid = static_cast<int>(std::min<int64_t>(n_units, dev.sm_count));
    if (log_enabled())
        log_launch(narrow ? "attn_tc_kernel<NARROW>" : "attn_tc_kernel", grid, kThreads, smem,
                   "head_dim %d units %lld batch %d heads %d n_detail %d window %d n_global %d "
                   "offsets %s global_ranges %s", HD, static_cast<long long>(n_units), p.batch,
                   p.heads, p.N, p.L, p.G, p.win_off ? "yes" : "no", p.gwin_off ? "yes" : "no");
    if (narrow)
        attn_tc_kernel<HD, true><<<grid, kThreads, smem, stream>>>(p);
    else
        attn_tc_kernel<HD, false><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? ATLAS_OK : ATLAS_ERR_CUDA;
}

}  // namespace

atlas_status launch_attn_tc_bf16(const AttnArgs &a, cudaStream_t stream) {
    DeviceInfo dev;
    if (!current_device(&dev)) return ATLAS_ERR_DEVICE;
    if (a.head_dim == 128) return launch_hd<128>(a, dev, stream);
    if (a.head_dim == 64) return launch_hd<64>(a, dev, stream);
    return ATLAS_ERR_UNSUPPORTED;
}

}  // namespace atlas
