/*
 * atlas_oracle.c -- plain, slow, fp64 CPU oracle for the detail branch's
 * hierarchical locality-preserving attention of AtlasVid.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA library never
 * calls it and shares no code, header, table or constant with it.
 *
 * Sources (page title, then section):
 *   [TS]  "Technische Samenvatting: AtlasVid" (gist.science, Dutch), with
 *         the same text as "Resume Technique : AtlasVid" (French) and
 *         "Resumo Tecnico: AtlasVid" (Portuguese):
 *           Methodologie 1, Fase 1 -- RoPE with temporal indices scaled by r_t;
 *           Methodologie 1, Fase 2 -- latent volume cut into spatiotemporal
 *               cubes, tokens reordered so each cube is contiguous, window
 *               attention over the reordered sequence;
 *           Methodologie 2 -- asymmetric hierarchical attention over the
 *               concatenated [X_global; X_detail] set (global sees only
 *               global; detail sees its own neighbourhood plus the global
 *               tokens; global->detail masked with -inf) and position
 *               alignment (global RoPE coordinates scaled by W/w, H/h, T/t).
 *   [AB]  "AtlasVid: Efficient Ultra-High-Resolution Long Video Generation
 *         via Decoupled Global-Local Modeling", abstract (arxivdaily.com):
 *         reordered spatiotemporal windows, asymmetric global-local
 *         attention, temporally scaled RoPE.
 *
 * The pages give no formulas for any of these steps. Where they are silent
 * this file takes the plainest reading, stated at each function:
 *   - tokens are stored in raster order r = (t*H + h)*W + w, one row of
 *     heads*head_dim values per token;
 *   - cubes are numbered in raster order over the cube grid, and the tokens
 *     of one cube in raster order over the cube's own extent; where the cube
 *     size does not divide an axis, the last cube along it is partial (keeps
 *     only the tokens that exist), so windows have variable length;
 *   - RoPE splits head_dim into contiguous [t | h | w] segments and rotates
 *     interleaved channel pairs (2k, 2k+1) of a segment of width d by the
 *     angle p * theta^(-2k/d), p = index * scale for that axis;
 *   - one joint softmax per query row over every allowed key; a detail
 *     query is allowed the keys of its own cube and every global key; a
 *     global query is allowed every global key and no detail key;
 *   - in the "aligned proxy tokens only" variant a detail query is allowed,
 *     of the global keys, only those whose scaled position falls inside its
 *     cube (see atlas_oracle_attention_head_aligned).
 *
 * Arithmetic is fp64 throughout, with no intermediate rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Cube reorder ([TS] Methodologie 1, Fase 2; [AB] "reordered windows")     */
/* ------------------------------------------------------------------------ */

/* Cubes along an axis of extent E cut into cubes of c tokens: ceil(E/c)
 * cubes, all of c tokens except the last, which keeps what is left. */
static int64_t cube_extent(int64_t E, int64_t c, int64_t b)
{
    return (b + 1) * c <= E ? c : E - b * c;
}

/* Position j, in the cube-contiguous sequence, of the token at raster index
 * r of a T x H x W grid cut into ct x ch x cw cubes. Cubes are taken in
 * raster order over the cube grid; a cube at the far edge of an axis the
 * cube size does not divide keeps only the tokens that exist (a partial
 * cube). Each cube's tokens are contiguous, in raster order over the cube's
 * own extent. The tokens before cube (bt, bh, bw) are: every whole slab of
 * bt*ct frames, then bh rows of cubes of that slab (bh*ch rows of the grid,
 * et frames deep), then bw cubes of that row (bw*cw columns, et x eh deep).
 * When the cube divides the grid this is cube*L + local with L = ct*ch*cw. */
int64_t atlas_oracle_cube_position(int64_t T, int64_t H, int64_t W,
                                   int64_t ct, int64_t ch, int64_t cw,
                                   int64_t r)
{
    int64_t t = r / (H * W);
    int64_t h = (r / W) % H;
    int64_t w = r % W;
    int64_t bt = t / ct, bh = h / ch, bw = w / cw;
    int64_t et = cube_extent(T, ct, bt);
    int64_t eh = cube_extent(H, ch, bh);
    int64_t ew = cube_extent(W, cw, bw);
    int64_t before = bt * ct * H * W + et * (bh * ch) * W + et * eh * (bw * cw);
    int64_t local = ((t - bt * ct) * eh + (h - bh * ch)) * ew + (w - bw * cw);
    return before + local;
}

/* Window (cube) boundaries of the cube-contiguous sequence: offsets[c] is
 * the first position of cube c (raster order over the cube grid) and
 * offsets[n_cubes] = T*H*W. Returns n_cubes; offsets must hold n_cubes+1. */
int64_t atlas_oracle_cube_windows(int64_t T, int64_t H, int64_t W,
                                  int64_t ct, int64_t ch, int64_t cw,
                                  int64_t *offsets)
{
    int64_t nt = (T + ct - 1) / ct, nh = (H + ch - 1) / ch, nw = (W + cw - 1) / cw;
    int64_t n = 0, pos = 0;
    for (int64_t bt = 0; bt < nt; ++bt)
        for (int64_t bh = 0; bh < nh; ++bh)
            for (int64_t bw = 0; bw < nw; ++bw) {
                offsets[n++] = pos;
                pos += cube_extent(T, ct, bt) * cube_extent(H, ch, bh) *
                       cube_extent(W, cw, bw);
            }
    offsets[n] = pos;
    return n;
}

/* Fill pos[r] = cube position of raster token r, for every r < T*H*W. */
void atlas_oracle_cube_positions(int64_t T, int64_t H, int64_t W,
                                 int64_t ct, int64_t ch, int64_t cw,
                                 int64_t *pos)
{
    int64_t n = T * H * W;
    for (int64_t r = 0; r < n; ++r)
        pos[r] = atlas_oracle_cube_position(T, H, W, ct, ch, cw, r);
}

/* dst[position(r)] = src[r], row by row, as a byte copy: every bit pattern
 * survives, so the inverse below restores the input exactly. Returns 0, or
 * 3 if a position falls outside the grid (defensive; cannot happen with a
 * correct position map). */
int atlas_oracle_cube_reorder(const unsigned char *src, unsigned char *dst,
                              int64_t T, int64_t H, int64_t W,
                              int64_t ct, int64_t ch, int64_t cw,
                              int64_t row_bytes)
{
    int64_t n = T * H * W;
    for (int64_t r = 0; r < n; ++r) {
        int64_t j = atlas_oracle_cube_position(T, H, W, ct, ch, cw, r);
        if (j < 0 || j >= n) return 3;
        memcpy(dst + j * row_bytes, src + r * row_bytes, (size_t)row_bytes);
    }
    return 0;
}

/* The exact inverse: dst[r] = src[position(r)]. Returns as the reorder. */
int atlas_oracle_cube_unorder(const unsigned char *src, unsigned char *dst,
                              int64_t T, int64_t H, int64_t W,
                              int64_t ct, int64_t ch, int64_t cw,
                              int64_t row_bytes)
{
    int64_t n = T * H * W;
    for (int64_t r = 0; r < n; ++r) {
        int64_t j = atlas_oracle_cube_position(T, H, W, ct, ch, cw, r);
        if (j < 0 || j >= n) return 3;
        memcpy(dst + r * row_bytes, src + j * row_bytes, (size_t)row_bytes);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* 3D RoPE ([TS] Methodologie 1, Fase 1: temporal index times r_t;          */
/*          [TS] Methodologie 2, position alignment: global coordinates     */
/*          scaled by the resolution ratios)                                */
/* ------------------------------------------------------------------------ */

/* Rotate one segment of one head: channels [off, off + d) of x, as pairs
 * (2k, 2k+1), by angle p * theta^(-2k/d). */
static void rope_segment(const double *x, double *y, int64_t off, int64_t d,
                         double p, double theta)
{
    for (int64_t k = 0; k < d / 2; ++k) {
        double omega = pow(theta, -2.0 * (double)k / (double)d);
        double phi = p * omega;
        double c = cos(phi), s = sin(phi);
        double x0 = x[off + 2 * k], x1 = x[off + 2 * k + 1];
        y[off + 2 * k] = x0 * c - x1 * s;
        y[off + 2 * k + 1] = x0 * s + x1 * c;
    }
}

/* Apply 3D RoPE to n_rows token rows. Row i of x (heads*head_dim values)
 * is the token at raster index raster_idx[i] of a T x H x W grid; its
 * position is p = (t*s_t, h*s_h, w*s_w). head_dim = d_t + d_h + d_w, each
 * even; the t segment comes first, then h, then w. */
void atlas_oracle_rope3d_rows(const double *x, double *y, int64_t n_rows,
                              const int64_t *raster_idx,
                              int64_t T, int64_t H, int64_t W,
                              int64_t heads, int64_t head_dim, double theta,
                              int64_t d_t, int64_t d_h, int64_t d_w,
                              double s_t, double s_h, double s_w)
{
    (void)T;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = raster_idx[i];
        double p_t = (double)(r / (H * W)) * s_t;
        double p_h = (double)((r / W) % H) * s_h;
        double p_w = (double)(r % W) * s_w;
        for (int64_t hd = 0; hd < heads; ++hd) {
            const double *xr = x + (i * heads + hd) * head_dim;
            double *yr = y + (i * heads + hd) * head_dim;
            rope_segment(xr, yr, 0, d_t, p_t, theta);
            rope_segment(xr, yr, d_t, d_h, p_h, theta);
            rope_segment(xr, yr, d_t + d_h, d_w, p_w, theta);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Asymmetric global-local attention ([TS] Methodologie 1 Fase 2 and 2)     */
/* ------------------------------------------------------------------------ */

/* Key ids run over the concatenated set: 0 .. N-1 are the detail tokens in
 * cube-contiguous order, N .. N+G-1 the global tokens. Query ids likewise.
 * A detail query sees the keys of its own cube (window of L consecutive
 * positions) and every global key; a global query sees every global key and
 * no detail key (mask value -inf). */
/* The window holding detail position x: x / L for windows of L positions,
 * else the last c with win_off[c] <= x (win_off: n_win+1 increasing
 * offsets, win_off[0] = 0, win_off[n_win] = N). */
static int64_t window_of(int64_t x, int64_t L, const int64_t *win_off, int64_t n_win)
{
    if (win_off == NULL) return x / L;
    int64_t lo = 0, hi = n_win - 1;
    while (lo < hi) {
        int64_t mid = (lo + hi + 1) / 2;
        if (win_off[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* "Aligned proxy tokens only" variant ([TS] Methodologie 2: a detail query
 * sees the global tokens aligned with it; position alignment puts global
 * token (tg, hg, wg) of a t x h x w grid at detail-grid coordinates
 * (tg*T/t, hg*H/h, wg*W/w)). Reading: a global key is aligned with a detail
 * cube when that scaled position lies inside the cube, i.e. on each axis
 * a <= tg*T/t < a + e for the cube's start a and extent e, compared exactly
 * as a*t <= tg*T < (a+e)*t. */
struct mask {
    int64_t N, L, n_win;
    const int64_t *win_off;
    int aligned;                 /* 0: a detail query sees every global key */
    int64_t T, H, W, ct, ch, cw; /* aligned only: detail grid and cube */
    int64_t t, h, w;             /* aligned only: global grid */
    const int64_t *cube_of;      /* aligned only: cube id of each detail position */
};

static int axis_aligned(int64_t a, int64_t e, int64_t g, int64_t E, int64_t e_glob)
{
    return a * e_glob <= g * E && g * E < (a + e) * e_glob;
}

static int global_aligned(const struct mask *m, int64_t c, int64_t g)
{
    int64_t nh = (m->H + m->ch - 1) / m->ch, nw = (m->W + m->cw - 1) / m->cw;
    int64_t bt = c / (nh * nw), bh = (c / nw) % nh, bw = c % nw;
    int64_t gt = g / (m->h * m->w), gh = (g / m->w) % m->h, gw = g % m->w;
    return axis_aligned(bt * m->ct, cube_extent(m->T, m->ct, bt), gt, m->T, m->t) &&
           axis_aligned(bh * m->ch, cube_extent(m->H, m->ch, bh), gh, m->H, m->h) &&
           axis_aligned(bw * m->cw, cube_extent(m->W, m->cw, bw), gw, m->W, m->w);
}

static int allowed(const struct mask *m, int64_t q, int64_t k)
{
    int q_detail = q < m->N, k_detail = k < m->N;
    if (q_detail && k_detail) {
        if (m->aligned) return m->cube_of[q] == m->cube_of[k];
        return window_of(q, m->L, m->win_off, m->n_win) ==
               window_of(k, m->L, m->win_off, m->n_win);
    }
    if (q_detail && !k_detail) return m->aligned ? global_aligned(m, m->cube_of[q], k - m->N) : 1;
    if (!q_detail && k_detail) return 0;
    return 1;
}

/* One head. Windows: window_len consecutive detail positions, or, when
 * win_off is not NULL, the n_win ranges [win_off[c], win_off[c+1]).
 * For each of the n_q queries (ids q_ids[i], vectors q[i]),
 * evaluate allowed() against all N+G keys, take logits scale*<q,k> on the
 * allowed ones, then a two-pass softmax (max, then sum of exp) and the
 * weighted sum of V. Outputs o[i] (head_dim values) and lse[i] (natural
 * log of the softmax denominator, logits included, i.e. max + log(sum)).
 *
 * k_d/v_d hold detail rows kd_lo .. kd_hi-1 only (row stride head_dim);
 * k_g/v_g hold all G global rows. If an allowed detail key falls outside
 * the rows supplied the function returns 1 (caller error); 2 on allocation
 * failure; 0 on success. */
static int attention_core(const struct mask *msk, int64_t n_global, int64_t head_dim,
                          double scale, const double *k_d, const double *v_d,
                          int64_t kd_lo, int64_t kd_hi, const double *k_g, const double *v_g,
                          int64_t n_q, const int64_t *q_ids, const double *q, double *o,
                          double *lse, int n_threads)
{
    int64_t N = msk->N, G = n_global, D = head_dim;
    int status = 0;
    if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
    for (int64_t i = 0; i < n_q; ++i) {
        int64_t qid = q_ids[i];
        const double *qi = q + i * D;
        double *oi = o + i * D;
        double *logit = (double *)malloc((size_t)(N + G) * sizeof(double));
        const double **vrow = (const double **)malloc((size_t)(N + G) * sizeof(double *));
        if (!logit || !vrow) {
            free(logit); free(vrow);
#pragma omp atomic write
            status = 2;
            continue;
        }
        int64_t n_allowed = 0;
        int bad = 0;
        for (int64_t kid = 0; kid < N + G; ++kid) {
            if (!allowed(msk, qid, kid)) continue;
            const double *kr, *vr;
            if (kid < N) {
                if (kid < kd_lo || kid >= kd_hi) { bad = 1; break; }
                kr = k_d + (kid - kd_lo) * D;
                vr = v_d + (kid - kd_lo) * D;
            } else {
                kr = k_g + (kid - N) * D;
                vr = v_g + (kid - N) * D;
            }
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d) dot += qi[d] * kr[d];
            logit[n_allowed] = scale * dot;
            vrow[n_allowed] = vr;
            ++n_allowed;
        }
        if (bad) {
            free(logit); free(vrow);
#pragma omp atomic write
            status = 1;
            continue;
        }
        /* pass 1: row maximum */
        double m = -INFINITY;
        for (int64_t a = 0; a < n_allowed; ++a)
            if (logit[a] > m) m = logit[a];
        /* pass 2: denominator and weighted sum of V */
        double sum = 0.0;
        for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
        for (int64_t a = 0; a < n_allowed; ++a) {
            double p = exp(logit[a] - m);
            sum += p;
            for (int64_t d = 0; d < D; ++d) oi[d] += p * vrow[a][d];
        }
        for (int64_t d = 0; d < D; ++d) oi[d] /= sum;
        lse[i] = m + log(sum);
        free(logit);
        free(vrow);
    }
    return status;
}

int atlas_oracle_attention_head_windows(int64_t n_detail, int64_t window_len,
                                        const int64_t *win_off, int64_t n_win,
                                        int64_t n_global, int64_t head_dim,
                                        double scale,
                                        const double *k_d, const double *v_d,
                                        int64_t kd_lo, int64_t kd_hi,
                                        const double *k_g, const double *v_g,
                                        int64_t n_q, const int64_t *q_ids,
                                        const double *q, double *o, double *lse,
                                        int n_threads)
{
    struct mask m;
    memset(&m, 0, sizeof m);
    m.N = n_detail;
    m.L = window_len;
    m.win_off = win_off;
    m.n_win = n_win;
    return attention_core(&m, n_global, head_dim, scale, k_d, v_d, kd_lo, kd_hi, k_g, v_g,
                          n_q, q_ids, q, o, lse, n_threads);
}

/* One head of the aligned variant. Detail grid T x H x W cut into cubes
 * ct x ch x cw (partial cubes at the far edges), detail rows in cube order;
 * global grid t x h x w (G = t*h*w rows, raster order). A detail query sees
 * its own cube and the global keys aligned with that cube; a global query
 * sees every global key. Arguments and return value otherwise as
 * atlas_oracle_attention_head_windows; 3 if the cube positions are not a
 * permutation (defensive; cannot happen with a correct position map). */
int atlas_oracle_attention_head_aligned(int64_t T, int64_t H, int64_t W,
                                        int64_t ct, int64_t ch, int64_t cw,
                                        int64_t t, int64_t h, int64_t w,
                                        int64_t head_dim, double scale,
                                        const double *k_d, const double *v_d,
                                        int64_t kd_lo, int64_t kd_hi,
                                        const double *k_g, const double *v_g,
                                        int64_t n_q, const int64_t *q_ids,
                                        const double *q, double *o, double *lse,
                                        int n_threads)
{
    struct mask m;
    memset(&m, 0, sizeof m);
    m.N = T * H * W;
    m.aligned = 1;
    m.T = T; m.H = H; m.W = W;
    m.ct = ct; m.ch = ch; m.cw = cw;
    m.t = t; m.h = h; m.w = w;
    int64_t *cube_of = (int64_t *)malloc((size_t)(m.N > 0 ? m.N : 1) * sizeof(int64_t));
    if (!cube_of) return 2;
    int64_t nh = (H + ch - 1) / ch, nw = (W + cw - 1) / cw;
    for (int64_t r = 0; r < m.N; ++r) {
        int64_t tt = r / (H * W), hh = (r / W) % H, ww = r % W;
        int64_t j = atlas_oracle_cube_position(T, H, W, ct, ch, cw, r);
        if (j < 0 || j >= m.N) { free(cube_of); return 3; }   /* not a permutation */
        cube_of[j] = ((tt / ct) * nh + hh / ch) * nw + ww / cw;
    }
    m.cube_of = cube_of;
    int st = attention_core(&m, t * h * w, head_dim, scale, k_d, v_d, kd_lo, kd_hi, k_g, v_g,
                            n_q, q_ids, q, o, lse, n_threads);
    free(cube_of);
    return st;
}

/* Windows of window_len consecutive detail positions (the cube divides the
 * grid). */
int atlas_oracle_attention_head(int64_t n_detail, int64_t window_len,
                                int64_t n_global, int64_t head_dim,
                                double scale,
                                const double *k_d, const double *v_d,
                                int64_t kd_lo, int64_t kd_hi,
                                const double *k_g, const double *v_g,
                                int64_t n_q, const int64_t *q_ids,
                                const double *q, double *o, double *lse,
                                int n_threads)
{
    return atlas_oracle_attention_head_windows(n_detail, window_len, NULL, 0, n_global,
                                               head_dim, scale, k_d, v_d, kd_lo, kd_hi,
                                               k_g, v_g, n_q, q_ids, q, o, lse, n_threads);
}

/* ------------------------------------------------------------------------ */
/* Backward pass (gradients of the attention above; [TS] Methodologie 2      */
/* trains the attention projections with LoRA, which needs dQ, dK and dV)    */
/* ------------------------------------------------------------------------ */

/* One head, all N+G rows. q, k, v, dout: [N+G][D], detail rows first (cube
 * order), then global rows; dout is the gradient of the loss w.r.t. the
 * attention output o. With P the row softmax of the allowed logits
 * s_ij = scale*<q_i,k_j>:
 *   dP_ij = <dout_i, v_j>,  delta_i = sum_j P_ij dP_ij,
 *   dS_ij = P_ij (dP_ij - delta_i)            (softmax Jacobian),
 *   dq_i = scale sum_j dS_ij k_j,  dk_j = scale sum_i dS_ij q_i,
 *   dv_j = sum_i P_ij dout_i.
 * Pass 1 (over query rows) takes each row's softmax (two passes, as the
 * forward), delta_i and dq_i; pass 2 (over key rows) visits every query
 * that is allowed the key and accumulates dk_j and dv_j from the same
 * definitions. Returns 0, or 2 on allocation failure. */
static int attention_bwd_core(const struct mask *msk, int64_t n_global, int64_t D,
                              double scale, const double *q, const double *k,
                              const double *v, const double *dout, double *dq, double *dk,
                              double *dv, int64_t n_qsel, const int64_t *qsel,
                              int64_t n_ksel, const int64_t *ksel, int n_threads)
{
    int64_t R = msk->N + n_global;
    int status = 0;
    double *lse = (double *)malloc((size_t)(R > 0 ? R : 1) * sizeof(double));
    double *delta = (double *)malloc((size_t)(R > 0 ? R : 1) * sizeof(double));
    if (!lse || !delta) { free(lse); free(delta); return 2; }
    if (n_threads < 1) n_threads = 1;
    /* pass 1: every query row's softmax statistics (the selected keys may be
     * seen by any row), and dq for the selected rows (all rows without a
     * selection) */
    int64_t n_dq = qsel ? n_qsel : R;
    char *want_dq = (char *)calloc((size_t)(R > 0 ? R : 1), 1);
    int64_t *dq_slot = (int64_t *)malloc((size_t)(R > 0 ? R : 1) * sizeof(int64_t));
    if (!want_dq || !dq_slot) { free(lse); free(delta); free(want_dq); free(dq_slot); return 2; }
    for (int64_t a = 0; a < n_dq; ++a) {
        int64_t i = qsel ? qsel[a] : a;
        want_dq[i] = 1;
        dq_slot[i] = a;
    }
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
    for (int64_t i = 0; i < R; ++i) {
        const double *qi = q + i * D, *gi = dout + i * D;
        double *logit = (double *)malloc((size_t)R * sizeof(double));
        double *dp = (double *)malloc((size_t)R * sizeof(double));
        int64_t *key = (int64_t *)malloc((size_t)R * sizeof(int64_t));
        if (!logit || !dp || !key) {
            free(logit); free(dp); free(key);
#pragma omp atomic write
            status = 2;
            continue;
        }
        int64_t n = 0;
        for (int64_t j = 0; j < R; ++j) {
            if (!allowed(msk, i, j)) continue;
            double dot = 0.0, dpo = 0.0;
            for (int64_t d = 0; d < D; ++d) {
                dot += qi[d] * k[j * D + d];
                dpo += gi[d] * v[j * D + d];
            }
            logit[n] = scale * dot;
            dp[n] = dpo;
            key[n] = j;
            ++n;
        }
        double m = -INFINITY;
        for (int64_t a = 0; a < n; ++a)
            if (logit[a] > m) m = logit[a];
        double sum = 0.0;
        for (int64_t a = 0; a < n; ++a) sum += exp(logit[a] - m);
        lse[i] = log(sum) + m;
        double dl = 0.0;
        for (int64_t a = 0; a < n; ++a) dl += exp(logit[a] - lse[i]) * dp[a];
        delta[i] = dl;
        if (want_dq[i]) {
            double *dqi = dq + dq_slot[i] * D;
            for (int64_t d = 0; d < D; ++d) dqi[d] = 0.0;
            for (int64_t a = 0; a < n; ++a) {
                double ds = exp(logit[a] - lse[i]) * (dp[a] - dl);
                for (int64_t d = 0; d < D; ++d) dqi[d] += scale * ds * k[key[a] * D + d];
            }
        }
        free(logit); free(dp); free(key);
    }
    /* pass 2: dk and dv of the selected key rows (all rows without a
     * selection), over every query allowed to see the key */
    int64_t n_dk = ksel ? n_ksel : R;
    if (status == 0) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
        for (int64_t a = 0; a < n_dk; ++a) {
            int64_t j = ksel ? ksel[a] : a;
            const double *kj = k + j * D, *vj = v + j * D;
            double *dkj = dk + a * D, *dvj = dv + a * D;
            for (int64_t d = 0; d < D; ++d) { dkj[d] = 0.0; dvj[d] = 0.0; }
            for (int64_t i = 0; i < R; ++i) {
                if (!allowed(msk, i, j)) continue;
                double dot = 0.0, dpo = 0.0;
                for (int64_t d = 0; d < D; ++d) {
                    dot += q[i * D + d] * kj[d];
                    dpo += dout[i * D + d] * vj[d];
                }
                double p = exp(scale * dot - lse[i]);
                double ds = p * (dpo - delta[i]);
                for (int64_t d = 0; d < D; ++d) {
                    dkj[d] += scale * ds * q[i * D + d];
                    dvj[d] += p * dout[i * D + d];
                }
            }
        }
    }
    free(lse);
    free(delta);
    free(want_dq);
    free(dq_slot);
    return status;
}

/* Backward of one head with windows of window_len rows, or of the ranges
 * of win_off when not NULL; every global key allowed to detail queries. */
int atlas_oracle_attention_bwd_head_windows(int64_t n_detail, int64_t window_len,
                                            const int64_t *win_off, int64_t n_win,
                                            int64_t n_global, int64_t head_dim, double scale,
                                            const double *q, const double *k, const double *v,
                                            const double *dout, double *dq, double *dk,
                                            double *dv, int n_threads)
{
    struct mask m;
    memset(&m, 0, sizeof m);
    m.N = n_detail;
    m.L = window_len;
    m.win_off = win_off;
    m.n_win = n_win;
    return attention_bwd_core(&m, n_global, head_dim, scale, q, k, v, dout, dq, dk, dv, 0, NULL,
                              0, NULL, n_threads);
}

/* Backward of one head, windows form, for selected rows only: dq for the
 * n_qsel query rows qsel (written as n_qsel rows), dk and dv for the n_ksel
 * key rows ksel. Inputs hold all N+G rows. Every row's softmax statistics
 * are taken first, as the full version does. */
int atlas_oracle_attention_bwd_head_sampled(int64_t n_detail, int64_t window_len,
                                            const int64_t *win_off, int64_t n_win,
                                            int64_t n_global, int64_t head_dim, double scale,
                                            const double *q, const double *k, const double *v,
                                            const double *dout, int64_t n_qsel,
                                            const int64_t *qsel, int64_t n_ksel,
                                            const int64_t *ksel, double *dq, double *dk,
                                            double *dv, int n_threads)
{
    struct mask m;
    memset(&m, 0, sizeof m);
    m.N = n_detail;
    m.L = window_len;
    m.win_off = win_off;
    m.n_win = n_win;
    return attention_bwd_core(&m, n_global, head_dim, scale, q, k, v, dout, dq, dk, dv, n_qsel,
                              qsel, n_ksel, ksel, n_threads);
}

/* Backward of one head of the aligned variant (geometry as
 * atlas_oracle_attention_head_aligned). Returns 0, 2 (allocation) or 3. */
int atlas_oracle_attention_bwd_head_aligned(int64_t T, int64_t H, int64_t W,
                                            int64_t ct, int64_t ch, int64_t cw,
                                            int64_t t, int64_t h, int64_t w,
                                            int64_t head_dim, double scale,
                                            const double *q, const double *k, const double *v,
                                            const double *dout, double *dq, double *dk,
                                            double *dv, int n_threads)
{
    struct mask m;
    memset(&m, 0, sizeof m);
    m.N = T * H * W;
    m.aligned = 1;
    m.T = T; m.H = H; m.W = W;
    m.ct = ct; m.ch = ch; m.cw = cw;
    m.t = t; m.h = h; m.w = w;
    int64_t *cube_of = (int64_t *)malloc((size_t)(m.N > 0 ? m.N : 1) * sizeof(int64_t));
    if (!cube_of) return 2;
    int64_t nh = (H + ch - 1) / ch, nw = (W + cw - 1) / cw;
    for (int64_t r = 0; r < m.N; ++r) {
        int64_t tt = r / (H * W), hh = (r / W) % H, ww = r % W;
        int64_t j = atlas_oracle_cube_position(T, H, W, ct, ch, cw, r);
        if (j < 0 || j >= m.N) { free(cube_of); return 3; }
        cube_of[j] = ((tt / ct) * nh + hh / ch) * nw + ww / cw;
    }
    m.cube_of = cube_of;
    int st = attention_bwd_core(&m, t * h * w, head_dim, scale, q, k, v, dout, dq, dk, dv, 0,
                                NULL, 0, NULL, n_threads);
    free(cube_of);
    return st;
}

/* Number of threads an OpenMP parallel region of this library would use by
 * default (reported beside CPU timings). */
int atlas_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
