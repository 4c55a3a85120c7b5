/*
 * atlas.h -- C-ABI of libatlas.so: the B200 (sm_100a) hot path of AtlasVid's
 * detail-branch hierarchical locality-preserving attention.
 *
 * The path has four steps (page titles and sections cited at each call):
 *   (1) cube reorder of the latent token grid, and its exact inverse;
 *   (2) 3D rotary position embedding with per-axis position scales (the
 *       temporal scale r_t; global-proxy coordinates mapped onto the detail
 *       grid);
 *   (3) window attention over the reordered sequence, and
 *   (4) the asymmetric global-local attention,
 * where (3) and (4) are one call sharing one softmax per query row.
 *
 * Conventions for every call:
 *   - Tensors are row-major [rows, heads, head_dim], batch 1, contiguous.
 *     A detail grid T x H x W is stored in raster order, row
 *     r = (t*H + h)*W + w, unless the call says "cube order".
 *   - Every pointer is a device pointer owned by the caller, 16-byte
 *     aligned. The library allocates no tensor memory. It caches RoPE
 *     cos/sin tables in device memory (freed by atlas_release_caches) and
 *     keeps one device error word.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *     A status other than ATLAS_OK means nothing was launched, except
 *     ATLAS_ERR_CUDA, which reports a failed launch or copy.
 *   - The library runs on compute capability 10.0 (B200, sm_100a) only.
 */
#ifndef ATLAS_H
#define ATLAS_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *atlas_stream_t;

typedef enum {
    ATLAS_OK = 0,
    ATLAS_ERR_NULL = 1,        /* a required pointer is NULL                      */
    ATLAS_ERR_SHAPE = 2,       /* sizes inconsistent (cube does not divide grid,  */
                               /* n_detail not a multiple of window_len, <0 ...)  */
    ATLAS_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned                */
    ATLAS_ERR_UNSUPPORTED = 4, /* dtype / head_dim / RoPE split not supported     */
    ATLAS_ERR_ALIAS = 5,       /* input and output overlap where not allowed      */
    ATLAS_ERR_CUDA = 6,        /* a CUDA runtime call or a launch failed          */
    ATLAS_ERR_TIMEOUT = 7,     /* a kernel's bounded wait expired (device word)   */
    ATLAS_ERR_DEVICE = 8,      /* no usable device, or not compute capability 10.0 */
    ATLAS_ERR_CAPACITY = 9     /* a fixed-size internal buffer is too small (see  */
                               /* atlas_cube_reorder_noalloc)                     */
} atlas_status;

typedef enum {
    ATLAS_BF16 = 0,            /* bfloat16 I/O, fp32 arithmetic                   */
    ATLAS_FP32 = 1             /* float32 I/O, fp32 arithmetic                    */
} atlas_dtype;

/* Extents of a token grid: T frames, H rows, W columns. */
typedef struct { int64_t T, H, W; } atlas_grid3;

/* Extents of one spatiotemporal cube (window). */
typedef struct { int32_t ct, ch, cw; } atlas_cube3;

/* 3D RoPE parameters. head_dim = d_t + d_h + d_w, each even and > 0 or 0.
 * The segments are contiguous in that order. A token at grid index (t,h,w)
 * has position (t*scale_t, h*scale_h, w*scale_w). Channel pair (2k, 2k+1)
 * of a segment of width d rotates by angle position * theta^(-2k/d). */
typedef struct {
    double theta;
    int32_t d_t, d_h, d_w;
    double scale_t, scale_h, scale_w;
} atlas_rope;

/*
 * atlas_cube_reorder -- step (1), with step (2) fused when rope != NULL.
 *
 * Passage: "Technische Samenvatting: AtlasVid" (gist.science; same text in
 * the French and Portuguese editions), Methodologie 1, Fase 2: the latent
 * video volume is cut into spatiotemporal cubes and the tokens are reordered
 * so the tokens of one cube are contiguous. With rope != NULL the rows are
 * also rotated by 3D RoPE (Methodologie 1, Fase 1: temporal index times
 * r_t; Methodologie 2, position alignment: coordinates times the resolution
 * ratios), at the token's grid position.
 *
 * src: [T*H*W, heads, head_dim] in raster order. dst: same size, cube order:
 * cubes in raster order over the ceil(T/ct) x ceil(H/ch) x ceil(W/cw) cube
 * grid, the tokens of a cube in raster order over the cube, contiguous. When
 * the cube divides the grid, position j = cube*L + local with L = ct*ch*cw.
 * Otherwise the last cube along such an axis is partial (it keeps only the
 * tokens that exist) and windows have variable length: see
 * atlas_cube_window_offsets. Without rope the copy is bit-exact. With rope the
 * rotation runs in fp32 on fp64-built, fp32-rounded cos/sin and rounds once
 * to dtype (round to nearest even).
 * Errors: NULL pointers; a cube extent < 1 (SHAPE); head_dim not even or the RoPE split not summing to head_dim
 * or odd (UNSUPPORTED); rows not a multiple of 16 bytes, or misaligned
 * pointers (ALIGN); src and dst overlapping (ALIAS).
 */
atlas_status atlas_cube_reorder(const void *src, void *dst, atlas_grid3 grid,
                                atlas_cube3 cube, int32_t heads,
                                int32_t head_dim, atlas_dtype dtype,
                                const atlas_rope *rope, atlas_stream_t stream);

/*
 * atlas_cube_unorder -- the exact inverse of step (1).
 *
 * Passage: as atlas_cube_reorder (the permutation is undone after the
 * attention so the output is back in raster order).
 * src: cube order, dst: raster order, both [T*H*W, heads, head_dim]. A
 * byte copy: unorder(reorder(x)) == x for every bit pattern.
 * Errors: as atlas_cube_reorder (no RoPE).
 */
atlas_status atlas_cube_unorder(const void *src, void *dst, atlas_grid3 grid,
                                atlas_cube3 cube, int32_t heads,
                                int32_t head_dim, atlas_dtype dtype,
                                atlas_stream_t stream);

/*
 * atlas_rope3d -- step (2) on raster-ordered tokens (the global proxy).
 *
 * Passage: "Technische Samenvatting: AtlasVid", Methodologie 1, Fase 1
 * (temporally scaled RoPE, factor r_t) and Methodologie 2, position
 * alignment (global-proxy RoPE coordinates scaled by W/w, H/h, T/t onto the
 * high-resolution grid); abstract of "AtlasVid: Efficient Ultra-High-
 * Resolution Long Video Generation via Decoupled Global-Local Modeling".
 *
 * src, dst: [T*H*W, heads, head_dim], raster order. dst may equal src
 * (in place); partial overlap is ALIAS. Numerics as atlas_cube_reorder.
 */
atlas_status atlas_rope3d(const void *src, void *dst, atlas_grid3 grid,
                          int32_t heads, int32_t head_dim, atlas_dtype dtype,
                          const atlas_rope *rope, atlas_stream_t stream);

/*
 * atlas_local_global_attn -- steps (3) and (4) in one pass.
 *
 * Passages: "Technische Samenvatting: AtlasVid", Methodologie 1, Fase 2
 * (window attention over the reordered sequence, windows = geometric
 * neighbourhoods) and Methodologie 2, asymmetric hierarchical attention
 * (X_global and X_detail concatenated; X_global attends only to itself;
 * X_detail attends to its own neighbourhood and to the global tokens;
 * global -> detail masked with -inf).
 *
 * One softmax per query row over its allowed keys:
 *   detail row q (0 <= q < n_detail, cube order): detail keys of its own
 *     window [floor(q/window_len)*window_len, +window_len) and all
 *     n_global global keys;
 *   global row g: all n_global global keys, no detail key.
 * q_d, k_d, v_d: [n_detail, heads, head_dim] in cube order (n_detail may be
 *   0; the pointers are then ignored). n_detail % window_len == 0.
 * q_g, k_g, v_g: [n_global, heads, head_dim] (n_global may be 0).
 * o_d, o_g: outputs, same shapes and order as q_d, q_g.
 * lse: optional (NULL to skip), fp32 [heads, n_detail + n_global]: natural
 *   log of each row's softmax denominator over logits scale*<q,k>; detail
 *   rows first (cube order), then global rows.
 * softmax_scale <= 0 selects 1/sqrt(head_dim).
 * dtype BF16: tcgen05 tensor-core kernel; S and O accumulate in fp32, P is
 *   rounded to bf16 before the P*V product, O rounded to bf16 RNE.
 * dtype FP32: SIMT fp32 kernel.
 * head_dim must be 64 or 128.
 * Errors: NULL (required pointer), SHAPE, ALIGN, UNSUPPORTED; a kernel
 * whose bounded internal wait expires sets the device error word (read it
 * with atlas_last_device_error) and finishes without completing the rows.
 */
atlas_status atlas_local_global_attn(
    const void *q_d, const void *k_d, const void *v_d, int64_t n_detail,
    int64_t window_len, const void *q_g, const void *k_g, const void *v_g,
    int64_t n_global, int32_t heads, int32_t head_dim, float softmax_scale,
    atlas_dtype dtype, void *o_d, void *o_g, float *lse,
    atlas_stream_t stream);

/*
 * atlas_cube_reorder_noalloc -- atlas_cube_reorder without any device
 * memory allocation. The paper has no counterpart: this is a library
 * concern. Some callers cannot let a library call cudaMalloc: a serving
 * process whose device memory is reserved up front by its own allocator and
 * budget, or a latency-critical loop where cudaMalloc's implicit device-wide
 * synchronisation is not acceptable. atlas_cube_reorder caches its RoPE
 * cos/sin table in memory it allocates on first use; this variant keeps the
 * table in a fixed array compiled into the library instead.
 *
 * Arguments, layout, numerics and results are those of atlas_cube_reorder.
 * Differences:
 *   - The table lives in one file-scope device array of 32768 (cos, sin)
 *     pairs (256 KB), held by every GPU that loads the library until the
 *     process exits. A RoPE needs T*(d_t/2) + H*(d_h/2) + W*(d_w/2) pairs;
 *     more than 32768 returns ATLAS_ERR_CAPACITY and launches nothing.
 *   - A call whose grid extents or RoPE differ from those the device's
 *     array was last filled with builds the table on the host, in a host
 *     staging buffer that every call reuses, and copies it into the array
 *     on `stream` (from pageable memory: the call returns once the copy has
 *     been staged). A call with the same extents and RoPE as the last fill
 *     skips both and reads the array as it stands. Then the kernel is
 *     launched on `stream`.
 *   - Every call on a device shares the array and overwrites it: calls whose
 *     work overlaps on the GPU (for example on two streams) race; issue
 *     them on one stream or otherwise order them.
 *   - The first call on each device resolves the array's device address
 *     (cudaGetSymbolAddress, with that device current) and reads the device
 *     properties.
 *   - No cudaMalloc, cudaFree or other allocating routine is called.
 * Without rope the call is a pure permutation and touches no table.
 */
atlas_status atlas_cube_reorder_noalloc(const void *src, void *dst, atlas_grid3 grid,
                                        atlas_cube3 cube, int32_t heads,
                                        int32_t head_dim, atlas_dtype dtype,
                                        const atlas_rope *rope,
                                        atlas_stream_t stream);

/*
 * atlas_cube_window_offsets -- window boundaries of the cube order (host).
 *
 * Passage: as atlas_cube_reorder. Cube c (raster order over the cube grid)
 * occupies cube-order positions [offsets[c], offsets[c+1]); offsets[n] =
 * T*H*W. Partial cubes at the far edges are shorter windows.
 * offsets: host array of `capacity` int32, or NULL to only query the count.
 * *n_windows receives the number of cubes. Errors: NULL n_windows (NULL),
 * a non-positive extent or more than 2^31-1 tokens (SHAPE), capacity <
 * n_windows+1 (CAPACITY). Host only: no device work, no allocation.
 */
atlas_status atlas_cube_window_offsets(atlas_grid3 grid, atlas_cube3 cube,
                                       int32_t *offsets, int64_t capacity,
                                       int64_t *n_windows);

/*
 * atlas_local_global_attn_windows -- steps (3) and (4) with windows of
 * variable length (for example the partial cubes of a grid the cube does
 * not divide).
 *
 * Passages: as atlas_local_global_attn. Detail row q sees the detail keys of
 * the window w with window_offsets[w] <= q < window_offsets[w+1], and every
 * global key. window_offsets: DEVICE array of n_windows+1 int32, increasing,
 * window_offsets[0] = 0 and window_offsets[n_windows] = n_detail (the
 * library does not read it on the host; other contents give undefined rows
 * but no out-of-bounds access). Everything else as atlas_local_global_attn.
 * Errors: NULL window_offsets with n_detail > 0 (NULL), n_windows < 1 or >
 * n_detail (SHAPE), offsets not 4-byte aligned (ALIGN), as
 * atlas_local_global_attn otherwise.
 */
atlas_status atlas_local_global_attn_windows(
    const void *q_d, const void *k_d, const void *v_d, int64_t n_detail,
    const int32_t *window_offsets, int64_t n_windows, const void *q_g,
    const void *k_g, const void *v_g, int64_t n_global, int32_t heads,
    int32_t head_dim, float softmax_scale, atlas_dtype dtype, void *o_d,
    void *o_g, float *lse, atlas_stream_t stream);

/*
 * Layout of a call to atlas_local_global_attn_ex.
 *
 * batch: number of problems of the same shape stacked along the rows (>= 1).
 *   Detail tensors hold batch*n_detail rows (problem b at rows
 *   [b*n_detail, (b+1)*n_detail)), global tensors batch*n_global rows. A
 *   query sees only keys of its own problem.
 * Detail windows, the same for every problem:
 *   window_offsets == NULL: windows of window_len rows (n_detail %
 *     window_len == 0);
 *   window_offsets != NULL: DEVICE array of n_windows+1 int32 offsets over
 *     one problem's rows, increasing, [0] = 0, [n_windows] = n_detail
 *     (window_len is ignored).
 * global_window_offsets: NULL: a detail query sees every global key of its
 *   problem. Otherwise the "aligned proxy tokens only" variant: DEVICE array
 *   of n_windows+1 int32 offsets over one problem's global rows,
 *   non-decreasing, [0] = 0, [n_windows] = n_global; the queries of window
 *   w see the global keys [global_window_offsets[w],
 *   global_window_offsets[w+1]) of their problem. n_windows must then be the
 *   window count (n_detail / window_len without window_offsets). Global
 *   queries always see every global key of their problem.
 * The library never reads the offset arrays on the host. Contents other
 * than described give undefined rows, but every access stays inside the
 * tensors: a detail row always sees its own key, and ranges are clamped.
 */
typedef struct {
    int64_t batch;
    int64_t window_len;
    const int32_t *window_offsets;
    int64_t n_windows;
    const int32_t *global_window_offsets;
} atlas_attn_layout;

/*
 * atlas_local_global_attn_ex -- steps (3) and (4), general layout: batch of
 * problems, windows of fixed or variable length, and the all-global-keys or
 * the aligned-global-keys variant.
 *
 * Passages: as atlas_local_global_attn; for the aligned variant also
 * Methodologie 2, position alignment (global token (tg, hg, wg) of a t x h x w
 * grid sits at detail-grid position (tg*T/t, hg*H/h, wg*W/w); it is aligned
 * with the cube holding that point). When the ratios T/t, H/h, W/w are
 * integers dividing the cube sizes, the aligned global tokens of cube c are
 * cube c of the global grid cut into atlas_aligned_global_cube's cube: reorder
 * the global Q/K/V with atlas_cube_reorder using that cube, pass
 * atlas_cube_window_offsets of it as global_window_offsets, and unorder o_g.
 *
 * n_detail, n_global: rows of ONE problem. layout: see atlas_attn_layout
 * (NULL is an error). lse: optional fp32 [batch, heads, n_detail +
 * n_global], per problem detail rows first, then global rows. Everything
 * else as atlas_local_global_attn.
 * Errors: NULL layout or required pointer (NULL); batch < 1, inconsistent
 * windows, more than 2^31-1 rows in a tensor (SHAPE); misaligned offsets
 * (ALIGN); as atlas_local_global_attn otherwise.
 */
atlas_status atlas_local_global_attn_ex(
    const void *q_d, const void *k_d, const void *v_d, int64_t n_detail,
    const void *q_g, const void *k_g, const void *v_g, int64_t n_global,
    const atlas_attn_layout *layout, int32_t heads, int32_t head_dim,
    float softmax_scale, atlas_dtype dtype, void *o_d, void *o_g, float *lse,
    atlas_stream_t stream);

/*
 * atlas_local_global_attn_bwd -- gradients of steps (3) and (4).
 *
 * Passages: as atlas_local_global_attn_ex; the pages train the attention
 * projections with LoRA ("Technische Samenvatting: AtlasVid", Methodologie
 * 2, training strategy), which needs the gradients of the attention. With P
 * the row softmax of the allowed logits s = scale*<q,k> and dO the gradient
 * of the loss w.r.t. the output O:
 *   delta_i = sum_d dO_id O_id   (= sum_j P_ij <dO_i, v_j>),
 *   dS_ij = P_ij (<dO_i, v_j> - delta_i),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dO_i,
 * over the same allowed pairs as the forward (same layout, windows, batch
 * and variant). P is recomputed from q, k and the forward's lse.
 *
 * q_*, k_*, v_*: the forward's inputs; o_*: its outputs; do_*: gradients
 * w.r.t. o_* (same shapes and order). lse: the forward's LSE, fp32 [batch,
 * heads, n_detail + n_global] (required). delta: caller-owned fp32
 * workspace of the same shape, overwritten with delta_i. dq_*, dk_*, dv_*:
 * outputs, same shapes and dtype as q_*; they may not overlap any input.
 * dtype BF16: tcgen05 kernels (P and dS rounded to bf16 before their
 * products, fp32 accumulation, gradients rounded to bf16 RNE); FP32: SIMT
 * fp32 kernels. head_dim 64 or 128.
 * Errors: as atlas_local_global_attn_ex; NULL lse, delta or a required
 * gradient pointer (NULL); lse or delta not 4-byte aligned (ALIGN).
 */
atlas_status atlas_local_global_attn_bwd(
    const void *q_d, const void *k_d, const void *v_d, const void *o_d,
    const void *do_d, int64_t n_detail, const void *q_g, const void *k_g,
    const void *v_g, const void *o_g, const void *do_g, int64_t n_global,
    const atlas_attn_layout *layout, int32_t heads, int32_t head_dim,
    float softmax_scale, atlas_dtype dtype, const float *lse, float *delta,
    void *dq_d, void *dk_d, void *dv_d, void *dq_g, void *dk_g, void *dv_g,
    atlas_stream_t stream);

/*
 * atlas_aligned_global_reorder / atlas_aligned_global_unorder -- the global
 * proxy's tokens to and from the aligned order, for any grid ratios.
 *
 * Passage: Methodologie 2, position alignment. Reading: global index x of an
 * axis of e tokens sits at detail position x*E/e of the detail axis (E
 * tokens) and is aligned with the detail cube (c tokens) holding that point,
 * box(x) = floor(x*E / (c*e)); box b spans global indices [ceil(b*c*e/E),
 * ceil((b+1)*c*e/E)) (possibly empty), and the box triples partition the
 * global grid by the detail cube each token is aligned with. The aligned
 * order lists the tokens box by box in the cube grid's raster order (raster
 * order inside a box), so the aligned keys of detail window w are one range
 * [offsets[w], offsets[w+1]) (atlas_aligned_global_offsets): pass it as
 * atlas_attn_layout.global_window_offsets. When the ratios are integers
 * dividing the cube this is the cube order of atlas_aligned_global_cube.
 *
 * src, dst: [batch * t*h*w, heads, head_dim] of the global grid (raster order
 * for the reorder's input and the unorder's output); grid and cube are the
 * detail grid and its cube. rope: rotation at each token's global raster
 * position (NULL: none; for the unorder, the transpose with negated scales
 * maps gradients back). Errors as atlas_cube_reorder_batched.
 */
atlas_status atlas_aligned_global_reorder(const void *src, void *dst, int64_t batch,
                                          atlas_grid3 grid, atlas_cube3 cube,
                                          atlas_grid3 global_grid, int32_t heads,
                                          int32_t head_dim, atlas_dtype dtype,
                                          const atlas_rope *rope, atlas_stream_t stream);
atlas_status atlas_aligned_global_unorder(const void *src, void *dst, int64_t batch,
                                          atlas_grid3 grid, atlas_cube3 cube,
                                          atlas_grid3 global_grid, int32_t heads,
                                          int32_t head_dim, atlas_dtype dtype,
                                          const atlas_rope *rope, atlas_stream_t stream);

/*
 * atlas_aligned_global_offsets -- the global key range of every detail window
 * in the aligned order (host). offsets: host array of `capacity` int32, or
 * NULL to query the count; *n_windows receives the number of detail cubes
 * (windows, raster order over the cube grid); offsets[n_windows] = t*h*w.
 * Errors: NULL n_windows (NULL), non-positive extents or too many tokens
 * (SHAPE), capacity < n_windows+1 (CAPACITY). No device work.
 */
atlas_status atlas_aligned_global_offsets(atlas_grid3 grid, atlas_cube3 cube,
                                          atlas_grid3 global_grid, int32_t *offsets,
                                          int64_t capacity, int64_t *n_windows);

/*
 * atlas_aligned_global_cube -- the global-grid cube whose cubes are the
 * aligned sets of the detail cubes (host).
 *
 * Passage: Methodologie 2, position alignment (see atlas_local_global_attn_ex).
 * With ratios r = (T/t, H/h, W/w) integral and dividing (ct, ch, cw), global
 * cube c of the global grid cut into (ct/r_t, ch/r_h, cw/r_w) holds exactly
 * the global tokens aligned with detail cube c, partial cubes included, and
 * both grids have the same number of cubes. *global_cube receives that cube.
 * Errors: NULL global_cube (NULL); non-positive extents (SHAPE); ratios not
 * integral or not dividing the cube (UNSUPPORTED). Host only.
 */
atlas_status atlas_aligned_global_cube(atlas_grid3 grid, atlas_cube3 cube,
                                       atlas_grid3 global_grid,
                                       atlas_cube3 *global_cube);

/*
 * Batched permutations: `batch` problems of the same grid stacked along the
 * rows ([batch * T*H*W, heads, head_dim]); each problem is permuted (and
 * rotated) on its own, exactly as the unbatched call would. batch >= 1;
 * batch * T*H*W must stay below 2^31. Errors as the unbatched calls, SHAPE
 * for batch < 1.
 */
atlas_status atlas_cube_reorder_batched(const void *src, void *dst, int64_t batch,
                                        atlas_grid3 grid, atlas_cube3 cube,
                                        int32_t heads, int32_t head_dim,
                                        atlas_dtype dtype, const atlas_rope *rope,
                                        atlas_stream_t stream);
atlas_status atlas_cube_unorder_batched(const void *src, void *dst, int64_t batch,
                                        atlas_grid3 grid, atlas_cube3 cube,
                                        int32_t heads, int32_t head_dim,
                                        atlas_dtype dtype, atlas_stream_t stream);
atlas_status atlas_rope3d_batched(const void *src, void *dst, int64_t batch,
                                  atlas_grid3 grid, int32_t heads, int32_t head_dim,
                                  atlas_dtype dtype, const atlas_rope *rope,
                                  atlas_stream_t stream);

/*
 * atlas_cube_unorder_rope -- cube order -> raster order with each row rotated
 * by the RoPE of its raster position: dst[r] = R_rope(r) src[pi(r)].
 *
 * Passages: as atlas_cube_reorder. Its use is the backward of step (1)+(2):
 * R is orthogonal and rotating by -phi is its transpose, so with `rope`'s
 * scales negated this maps the gradient w.r.t. the reordered, rotated
 * tokens to the gradient w.r.t. the raster inputs of atlas_cube_reorder.
 * Batch, layout and errors as atlas_cube_unorder_batched; NULL rope (NULL).
 */
atlas_status atlas_cube_unorder_rope(const void *src, void *dst, int64_t batch,
                                     atlas_grid3 grid, atlas_cube3 cube, int32_t heads,
                                     int32_t head_dim, atlas_dtype dtype,
                                     const atlas_rope *rope, atlas_stream_t stream);

/*
 * atlas_qkv_proj_reorder -- the QKV projection with steps (1) and (2) in its
 * epilogue: [Q | K | V] = x w^T, Q and K rotated by 3D RoPE at each token's
 * grid position, all three written in cube order.
 *
 * Passages: as atlas_cube_reorder; the projection is the attention layer's
 * linear map (the summary's training strategy adapts the attention
 * projections). A GEMM acts on rows independently, so writing its rows at
 * their cube positions equals reordering its result. The rotation uses the
 * fp32 accumulator: each output is rounded to bf16 once.
 * x: [batch*T*H*W, c_in] bf16, raster order per problem. w: [3*heads*
 * head_dim, c_in] bf16 (rows of W_q, then W_k, then W_v). q, k, v: outputs
 * [batch*T*H*W, heads, head_dim] in cube order. rope: NULL for no rotation
 * (the global proxy takes a 1x1x1 cube and its own scales). tcgen05 GEMM,
 * fp32 accumulation.
 * Requirements: dtype BF16; c_in a multiple of 64; heads*head_dim a multiple
 * of 256; head_dim a multiple of 32; 16-byte aligned pointers.
 * Errors: NULL, SHAPE, ALIGN, UNSUPPORTED, ALIAS (an output overlapping an
 * input or another output), DEVICE, CUDA.
 */
atlas_status atlas_qkv_proj_reorder(const void *x, const void *w, int64_t batch,
                                    atlas_grid3 grid, atlas_cube3 cube, int32_t c_in,
                                    int32_t heads, int32_t head_dim, atlas_dtype dtype,
                                    const atlas_rope *rope, void *q, void *k, void *v,
                                    atlas_stream_t stream);

/*
 * atlas_out_proj_unorder -- the output projection with the exact inverse of
 * step (1) in its epilogue: y = unorder(o) w^T, computed as o w^T with each
 * row written at its raster position.
 *
 * o: [batch*T*H*W, c_in] bf16 in cube order (c_in = heads*head_dim, the
 * attention output viewed as rows). w: [c_out, c_in] bf16. y: [batch*T*H*W,
 * c_out] bf16, raster order. Requirements: dtype BF16; c_in a multiple of 64;
 * c_out a multiple of 256; 16-byte aligned pointers. Errors as
 * atlas_qkv_proj_reorder.
 */
atlas_status atlas_out_proj_unorder(const void *o, const void *w, int64_t batch,
                                    atlas_grid3 grid, atlas_cube3 cube, int32_t c_in,
                                    int32_t c_out, atlas_dtype dtype, void *y,
                                    atlas_stream_t stream);

/* Human-readable name of a status. Never NULL. */
const char *atlas_status_string(atlas_status status);

/*
 * Synchronise `stream`, then read and clear the device error word of the
 * current device into *code (0 = no kernel reported an error). Returns
 * ATLAS_ERR_TIMEOUT when the word is non-zero, ATLAS_ERR_CUDA when the
 * synchronisation itself failed, ATLAS_OK otherwise.
 */
atlas_status atlas_last_device_error(atlas_stream_t stream, uint32_t *code);

/*
 * Failure-path test hook. The next bf16 atlas_local_global_attn launch (any
 * thread, any device) leaves the first K tile of its first work unit
 * unloaded. The waits that depend on it expire after their bounded limit
 * (about 2 s): that CTA records ATLAS_ERR_TIMEOUT bits in the device error
 * word, drains its in-flight copies and MMAs, frees tensor memory and exits,
 * and its output rows are left incomplete. No fault, trap or hang is
 * involved, and the context stays usable. atlas_last_device_error then
 * returns ATLAS_ERR_TIMEOUT. One-shot; always ATLAS_OK.
 */
atlas_status atlas_debug_stall_next_attention(void);

/* Free the cached RoPE tables of every device (synchronises the device). */
atlas_status atlas_release_caches(void);

/* Number of RoPE cos/sin tables the library holds, over all devices, in
 * device memory it allocated itself (the cache of atlas_cube_reorder and the
 * other rotating calls; emptied by atlas_release_caches). The fixed array
 * of atlas_cube_reorder_noalloc is not counted. Host only; never fails. */
int64_t atlas_cached_rope_tables(void);

/* Library version, major*10000 + minor*100 + patch. */
int32_t atlas_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATLAS_H */
