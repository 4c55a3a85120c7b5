// atlas_internal.cuh -- shared declarations of libatlas.so (not installed).
//
// Device helpers here are thin inline-PTX wrappers around sm_100a
// instructions (mbarrier, TMA, tcgen05) written for this library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/atlas.h"

#define ATLAS_API extern "C" __attribute__((visibility("default")))

namespace atlas {

// ---------------------------------------------------------------------------
// Device error word: kernels OR bits into it instead of trapping.
// ---------------------------------------------------------------------------
enum DeviceError : uint32_t {
    kErrTimeoutProducer = 1u << 0,   // TMA producer wait expired
    kErrTimeoutMma = 1u << 1,        // MMA issuer wait expired
    kErrTimeoutSoftmax = 1u << 2,    // softmax / epilogue wait expired
    kErrTimeoutTeardown = 1u << 3,   // teardown wait for in-flight work expired
    kErrTmemAlloc = 1u << 4,         // tensor-memory allocation returned bad base
};

// Device address of the error word on the current device (host call; the
// word is a __device__ variable of atlas_api.cu, reached by kernels of other
// translation units through this pointer). NULL if it cannot be resolved.
uint32_t *device_error_word();

// Wall-clock limit of one bounded wait in a kernel, in nanoseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// Host-side helpers shared by the launchers.
// ---------------------------------------------------------------------------
struct DeviceInfo {
    int device = -1;
    int sm_count = 0;
    int major = 0, minor = 0;
    size_t smem_optin = 0;
};

// Current device's properties (cached per device). Returns false if no
// usable device or not compute capability 10.0.
bool current_device(DeviceInfo *out);

// Tracing and logging, both off by default and read once from the
// environment: ATLAS_NVTX=1 opens an NVTX range around every C-ABI call
// (named after the call; visible in Nsight Systems and Nsight Compute
// timelines), ATLAS_LOG=1 prints one line per kernel launch to stderr (the
// kernel, its grid, block and dynamic shared memory, and the work it walks).
bool log_enabled();
struct TraceScope {
    bool on;
    explicit TraceScope(const char *name);
    ~TraceScope();
};
#define ATLAS_TRACE() ::atlas::TraceScope atlas_trace_scope_(__func__)
void log_launch(const char *kernel, int grid, int block, size_t smem, const char *fmt, ...)
    __attribute__((format(printf, 5, 6)));

// Raise `func`'s dynamic shared-memory limit to `bytes` on the current
// device, once per (device, function): the attribute belongs to the device's
// context, so a process driving several GPUs sets it on each.
bool set_smem_limit(const void *func, int bytes);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb) {
    uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Launchers (defined in the kernel files). Arguments are validated by the
// C-ABI layer before these run.
struct PermuteArgs {
    const void *src;
    void *dst;
    int64_t T, H, W;
    int32_t ct, ch, cw;
    int32_t heads, head_dim, elem_bytes;
    int mode;               // 0 reorder (raster -> cube), 1 unorder, 2 raster RoPE,
                            // 5 / 6 to / from the aligned order of global tokens
    const atlas_rope *rope; // may be NULL (pure permutation)
    int64_t batch = 1;      // problems of this grid stacked along the rows
    int64_t DT = 0, DH = 0, DW = 0;   // modes 5 / 6: the detail grid (T, H, W: the global)
};
atlas_status launch_permute_rope(const PermuteArgs &a, cudaStream_t stream);
atlas_status release_rope_tables();
int64_t cached_rope_tables();
// The cached cos/sin table of `rope` on a T x H x W grid, current device
// (layout: axis t [t][k], then h, then w; fp64 angles rounded to fp32).
atlas_status rope_table_for(int64_t T, int64_t H, int64_t W, const atlas_rope &rope,
                            const float2 **out);

// Projections with the path's permutation in the GEMM epilogue (bf16).
struct ProjArgs {
    const void *x, *w;          // x [batch*T*H*W, c_in]; w [n_out, c_in]
    int64_t batch, T, H, W;
    int32_t ct, ch, cw;
    int32_t c_in, c_out;        // c_out: OUT only
    int32_t heads, head_dim;    // QKV only
    const atlas_rope *rope;     // QKV only, may be NULL
    void *out[3];               // QKV: q, k, v; OUT: y
};
atlas_status launch_qkv_proj(const ProjArgs &a, cudaStream_t stream);
atlas_status launch_out_proj(const ProjArgs &a, cudaStream_t stream);
// Reorder (+RoPE) with the cos/sin table in a fixed device array (no
// allocation); ATLAS_ERR_CAPACITY if the table would not fit.
atlas_status launch_permute_rope_noalloc(const PermuteArgs &a, cudaStream_t stream);

struct AttnArgs {
    const void *q_d, *k_d, *v_d;
    int64_t n_detail, window_len;
    const void *q_g, *k_g, *v_g;
    int64_t n_global;
    int32_t heads, head_dim;
    float scale;
    void *o_d, *o_g;
    float *lse;
    const int32_t *win_off = nullptr;  // window offsets (device), NULL: windows of window_len
    int64_t n_win = 0;                 // windows of win_off
    int64_t batch = 1;                 // problems stacked along the rows; n_detail, n_global
                                       // and the offsets are per problem
    const int32_t *gwin_off = nullptr; // per-window global key offsets (device), NULL: all
    int64_t n_gwin = 0;                // window count (with gwin_off)
};
atlas_status launch_attn_tc_bf16(const AttnArgs &a, cudaStream_t stream);
// [rows, heads, hd] bf16 viewed as a 3-D tensor (hd, heads, rows) with a box
// of 64 channels x 1 head x box_rows rows and 128-byte swizzle (defined in
// attn_tc.cu). False if the driver entry point is missing or encoding fails.
bool make_rows_map(CUtensorMap *m, const void *base, int64_t rows, int heads, int hd,
                   int box_rows = 128);
// One-shot request (atlas_debug_stall_next_attention): true once, for the
// next bf16 attention launch, which then leaves one K tile unloaded.
bool take_stall_request();
atlas_status launch_attn_simt_f32(const AttnArgs &a, cudaStream_t stream);

// Backward: the forward's arguments (fwd.o_d / fwd.o_g hold the forward's
// outputs O, fwd.lse its LSE; all are inputs here) plus dO, the delta
// workspace and the gradient outputs.
struct AttnBwdArgs {
    AttnArgs fwd;
    const void *do_d, *do_g;
    float *delta;
    void *dq_d, *dk_d, *dv_d, *dq_g, *dk_g, *dv_g;
    int elem_bytes;
};
// delta_i = <dO_i, O_i> for every row and head, into bwd.delta.
atlas_status launch_attn_bwd_delta(const AttnBwdArgs &a, cudaStream_t stream);
atlas_status launch_attn_bwd_simt_f32(const AttnBwdArgs &a, cudaStream_t stream);
atlas_status launch_attn_bwd_tc_bf16(const AttnBwdArgs &a, cudaStream_t stream);

}  // namespace atlas
