/*
 * attn_oracle.c -- plain fp64 CPU oracle for grouped-KV scaled-dot-product
 * attention (forward only).
 *
 * TEST INFRASTRUCTURE. This file is the reference the CUDA kernels are
 * checked against. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg may load it. It shares no code, header, table or helper
 * with the CUDA library, and it never calls into it.
 *
 * What it computes (the plain definition, not the tiled algorithm):
 *
 *   For batch b, query head h, query row i, with G = n_q / n_kv and the
 *   key/value head g = floor(h / G):
 *     s_j   = scale * <q[b,h,i,:], k[b,g,j,:]>            for j in V(i)
 *     m     = max_j s_j
 *     l     = sum_j exp(s_j - m)
 *     o[c]  = (sum_j exp(s_j - m) * v[b,g,j,c]) / l
 *     lse   = m + ln(l)
 *
 *   Sources:
 *   - "Attention, Worked Out by Hand (Part 2)" (j33.ai), "The recap": the
 *     five steps score, scale, mask, softmax, mix; and the FlashAttention
 *     section: every exponent taken relative to the running maximum (the
 *     numerically stable softmax, here in its two-pass form).
 *   - "Attention Engineering: From MHA to GQA, MLA & FlashAttention"
 *     (arman1o1.github.io), section 2, Grouped-Query Attention Formulation:
 *     the G query heads of group g share K_g and V_g; the zero-copy view
 *     [B, n_kv, G, S, D] puts query head h in group floor(h / G).
 *   - "2.4 Multi-Head Attention, MQA, GQA & MLA" (llm-stack-book), section
 *     "Implementing the MHA -> GQA conversion": query head j reads KV head
 *     j // n_rep.
 *   - Same "Attention Engineering" page, section 4: the log-sum-exp kept
 *     per row is L = m + log(l) in natural log of the scaled scores.
 *
 *   Visible set V(i):
 *   - causal prefill: keys j <= i + (Skv - Sq). The pages show only
 *     Sq == Skv, where this is the upper-triangular -inf mask of "Attention
 *     Engineering" section 2; for Sq < Skv the query rows are taken to be
 *     the last Sq positions (bottom-right alignment), the reading that makes
 *     a one-row query the decode step against a cache.
 *   - non-causal: all Skv keys.
 *   - decode (seqlens given): keys 0 .. seqlens[b]-1, no other mask
 *     ("2.4 Multi-Head Attention, MQA, GQA & MLA", exercise decode_step,
 *     which calls SDPA with is_causal=False for the lone query).
 *   - an empty visible set gives o = 0 and lse = -inf (the pages are
 *     silent; this is the limit of an empty sum).
 *   - sliding window (window W > 0): of the keys above, only those with
 *     p - j < W stay, p being the query's own position (the last visible
 *     key: i + Skv - Sq in causal prefill, seqlens[b] - 1 in decode),
 *     "Attention deep dive" (askaiml.pages.dev) section 6, mask (j <= i)
 *     AND (i - j < W); plus the first n_sink keys, which stay visible to
 *     every query ("Attention Engineering" section 5, failure mode 2: keep
 *     the initial sink tokens in a rolling window). W = 0: no window.
 *
 * The online mode follows the FlashAttention-2 exact tiled rescaling
 * recurrence of "Attention Engineering" section 4 (running m, l, O~ per row,
 * rescale by exp(m_old - m_new), divide by l once at the end), with key tiles
 * of B_c columns and query blocks of B_r rows; causal key tiles to the right
 * of a query block's last row are never visited.
 *
 * Layouts (all fp64, element strides):
 *   q   [B, n_q, Sq, d_qk] contiguous
 *   k   element (b, g, j, c) at k[b*k_sb + g*k_sh + j*k_ss + c]
 *   v   element (b, g, j, c) at v[b*v_sb + g*v_sh + j*v_ss + c]
 *   o   [B, n_q, Sq, d_v] contiguous
 *   lse [B, n_q, Sq] contiguous
 * K and V may alias (the MLA latent cache: key = first d_qk columns of a row,
 * value = first d_v columns of the same row).
 *
 * Return value: 0 on success, -1 on invalid arguments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    const double *k, *v;
    int64_t k_sb, k_sh, k_ss, v_sb, v_sh, v_ss;
    int n_q, n_kv, Sq, Skv, d_qk, d_v;
    const int32_t *seqlens;
    int causal;
    double scale;
    int64_t window, n_sink;   /* window 0: every key up to the end is visible */
} problem_t;

static int check_problem(const problem_t *p, int B)
{
    if (B < 0 || p->n_q <= 0 || p->n_kv <= 0 || p->Sq < 0 || p->Skv < 0) return -1;
    if (p->d_qk <= 0 || p->d_v <= 0) return -1;
    if (p->n_q % p->n_kv != 0) return -1;
    if (p->causal != 0 && p->causal != 1) return -1;
    if (p->window < 0 || p->n_sink < 0) return -1;
    return 0;
}

/* Number of visible keys for query row i of batch b: V(i) = [0, end). */
static int64_t visible_end(const problem_t *p, int b, int64_t i)
{
    if (p->seqlens) {
        int64_t n = p->seqlens[b];
        if (n < 0) n = 0;
        if (n > p->Skv) n = p->Skv;
        return n;
    }
    if (p->causal) {
        int64_t end = i + ((int64_t)p->Skv - (int64_t)p->Sq) + 1;
        if (end < 0) end = 0;
        if (end > p->Skv) end = p->Skv;
        return end;
    }
    return p->Skv;
}

/* Is key j (< end) visible? Only the window and the sinks remove keys. */
static int visible(const problem_t *p, int64_t end, int64_t j)
{
    if (p->window == 0) return 1;
    return (end - 1 - j < p->window) || (j < p->n_sink);
}

/*
 * One query row, the plain definition: score, scale, mask, two-pass softmax,
 * mix. `s` is scratch of at least Skv doubles. `weights` (optional) receives
 * the softmax weights of the visible keys (0 for the others).
 */
static void attend_row(const problem_t *p, int b, int h, int64_t i,
                       const double *q_row, double *o_row, double *lse_out,
                       double *s, double *weights)
{
    const int g = h / (p->n_q / p->n_kv);
    const double *kb = p->k + b * p->k_sb + g * p->k_sh;
    const double *vb = p->v + b * p->v_sb + g * p->v_sh;
    const int64_t end = visible_end(p, b, i);

    for (int c = 0; c < p->d_v; ++c) o_row[c] = 0.0;
    if (end == 0) {
        *lse_out = -INFINITY;
        return;
    }
    /* score and scale (a window keeps the last key, so some key is visible) */
    for (int64_t j = 0; j < end; ++j) {
        if (!visible(p, end, j)) continue;
        const double *kj = kb + j * p->k_ss;
        double acc = 0.0;
        for (int c = 0; c < p->d_qk; ++c) acc += q_row[c] * kj[c];
        s[j] = p->scale * acc;
    }
    /* softmax, pass 1: the row maximum */
    double m = -INFINITY;
    for (int64_t j = 0; j < end; ++j)
        if (visible(p, end, j) && s[j] > m) m = s[j];
    /* softmax, pass 2: exponentials relative to the maximum, their sum, and
       the weighted sum of value rows */
    double l = 0.0;
    for (int64_t j = 0; j < end; ++j) {
        if (!visible(p, end, j)) continue;
        const double e = exp(s[j] - m);
        const double *vj = vb + j * p->v_ss;
        l += e;
        for (int c = 0; c < p->d_v; ++c) o_row[c] += e * vj[c];
    }
    for (int c = 0; c < p->d_v; ++c) o_row[c] /= l;
    *lse_out = m + log(l);
    if (weights) {
        for (int64_t j = 0; j < end; ++j) weights[j] = visible(p, end, j) ? exp(s[j] - m) / l : 0.0;
    }
}

static int set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) return nthreads;
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Full forward over every (b, h, i). */
int oracle_sdpa_fp64(const double *q, const double *k, const double *v,
                     double *o, double *lse,
                     int B, int n_q, int n_kv, int Sq, int Skv, int d_qk, int d_v,
                     int64_t k_sb, int64_t k_sh, int64_t k_ss,
                     int64_t v_sb, int64_t v_sh, int64_t v_ss,
                     const int32_t *seqlens, int causal, double scale, int nthreads)
{
    problem_t p = {k, v, k_sb, k_sh, k_ss, v_sb, v_sh, v_ss,
                   n_q, n_kv, Sq, Skv, d_qk, d_v, seqlens, causal, scale, 0, 0};
    if (check_problem(&p, B)) return -1;
    const int64_t rows = (int64_t)B * n_q * Sq;
    int nt = set_threads(nthreads);
    int err = 0;
#pragma omp parallel num_threads(nt)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t i = r % Sq;
                const int h = (int)((r / Sq) % n_q);
                const int b = (int)(r / ((int64_t)Sq * n_q));
                attend_row(&p, b, h, i, q + r * d_qk, o + r * d_v, lse + r, s, NULL);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/* Full forward with a sliding window of `window` keys (> 0) and `n_sink`
 * always-visible initial keys (see the visible set above). */
int oracle_sdpa_window_fp64(const double *q, const double *k, const double *v,
                            double *o, double *lse,
                            int B, int n_q, int n_kv, int Sq, int Skv, int d_qk, int d_v,
                            int64_t k_sb, int64_t k_sh, int64_t k_ss,
                            int64_t v_sb, int64_t v_sh, int64_t v_ss,
                            const int32_t *seqlens, int causal, int window, int n_sink,
                            double scale, int nthreads)
{
    problem_t p = {k, v, k_sb, k_sh, k_ss, v_sb, v_sh, v_ss,
                   n_q, n_kv, Sq, Skv, d_qk, d_v, seqlens, causal, scale, window, n_sink};
    if (check_problem(&p, B) || window <= 0) return -1;
    const int64_t rows = (int64_t)B * n_q * Sq;
    int nt = set_threads(nthreads);
    int err = 0;
#pragma omp parallel num_threads(nt)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < rows; ++r) {
                const int64_t i = r % Sq;
                const int h = (int)((r / Sq) % n_q);
                const int b = (int)(r / ((int64_t)Sq * n_q));
                attend_row(&p, b, h, i, q + r * d_qk, o + r * d_v, lse + r, s, NULL);
            }
            free(s);
        }
    }
    return err ? -1 : 0;
}

/*
 * Selected rows only: row r is (row_b[r], row_h[r], row_i[r]); its query
 * vector is q_rows[r*d_qk ...] and its outputs go to o_rows[r*d_v ...] and
 * lse_rows[r]. Used for sampled checks at sizes the full oracle cannot reach.
 */
int oracle_sdpa_rows_fp64(const double *q_rows, const double *k, const double *v,
                          double *o_rows, double *lse_rows,
                          const int32_t *row_b, const int32_t *row_h, const int32_t *row_i,
                          int n_rows,
                          int B, int n_q, int n_kv, int Sq, int Skv, int d_qk, int d_v,
                          int64_t k_sb, int64_t k_sh, int64_t k_ss,
                          int64_t v_sb, int64_t v_sh, int64_t v_ss,
                          const int32_t *seqlens, int causal, double scale, int nthreads)
{
    problem_t p = {k, v, k_sb, k_sh, k_ss, v_sb, v_sh, v_ss,
                   n_q, n_kv, Sq, Skv, d_qk, d_v, seqlens, causal, scale, 0, 0};
    if (check_problem(&p, B) || n_rows < 0) return -1;
    for (int r = 0; r < n_rows; ++r) {
        if (row_b[r] < 0 || row_b[r] >= B || row_h[r] < 0 || row_h[r] >= n_q ||
            row_i[r] < 0 || row_i[r] >= Sq)
            return -1;
    }
    int nt = set_threads(nthreads);
    int err = 0;
#pragma omp parallel num_threads(nt)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int r = 0; r < n_rows; ++r)
                attend_row(&p, row_b[r], row_h[r], row_i[r], q_rows + (int64_t)r * d_qk,
                           o_rows + (int64_t)r * d_v, lse_rows + r, s, NULL);
            free(s);
        }
    }
    return err ? -1 : 0;
}

/*
 * One row with its softmax weights exposed: weights[j] for j < n_visible
 * (returned), zero beyond. `weights` must hold Skv doubles.
 */
int64_t oracle_row_weights_fp64(const double *q_row, const double *k, const double *v,
                                double *o_row, double *lse, double *weights,
                                int b, int h, int i,
                                int B, int n_q, int n_kv, int Sq, int Skv, int d_qk, int d_v,
                                int64_t k_sb, int64_t k_sh, int64_t k_ss,
                                int64_t v_sb, int64_t v_sh, int64_t v_ss,
                                const int32_t *seqlens, int causal, double scale)
{
    problem_t p = {k, v, k_sb, k_sh, k_ss, v_sb, v_sh, v_ss,
                   n_q, n_kv, Sq, Skv, d_qk, d_v, seqlens, causal, scale, 0, 0};
    if (check_problem(&p, B) || b < 0 || b >= B || h < 0 || h >= n_q || i < 0 || i >= Sq)
        return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
    if (!s) return -1;
    for (int j = 0; j < Skv; ++j) weights[j] = 0.0;
    attend_row(&p, b, h, i, q_row, o_row, lse, s, weights);
    free(s);
    return visible_end(&p, b, i);
}

/*
 * Online mode: the FlashAttention-2 tiled recurrence, in fp64, with query
 * blocks of block_r rows and key tiles of block_c columns.
 *
 *   m_new  = max(m, rowmax(S_tile))            (masked entries are -inf)
 *   P~     = exp(S_tile - m_new)
 *   l      = exp(m - m_new) * l + rowsum(P~)
 *   O~     = exp(m - m_new) * O~ + P~ V_tile
 * and at the end O = O~ / l, L = m + ln l.
 *
 * A row whose visible set is still empty after a tile keeps m = -inf and
 * adds nothing (exp(-inf - -inf) is taken as the identity rescale 1, the
 * limit the recurrence has when no score has been seen yet).
 */
int oracle_online_fp64(const double *q, const double *k, const double *v,
                       double *o, double *lse,
                       int B, int n_q, int n_kv, int Sq, int Skv, int d_qk, int d_v,
                       int64_t k_sb, int64_t k_sh, int64_t k_ss,
                       int64_t v_sb, int64_t v_sh, int64_t v_ss,
                       const int32_t *seqlens, int causal, double scale,
                       int block_r, int block_c, int nthreads)
{
    problem_t p = {k, v, k_sb, k_sh, k_ss, v_sb, v_sh, v_ss,
                   n_q, n_kv, Sq, Skv, d_qk, d_v, seqlens, causal, scale, 0, 0};
    if (check_problem(&p, B) || block_r <= 0 || block_c <= 0) return -1;
    const int G = n_q / n_kv;
    const int64_t n_blocks = ((int64_t)Sq + block_r - 1) / block_r;
    const int64_t units = (int64_t)B * n_q * n_blocks;
    int nt = set_threads(nthreads);
    int err = 0;
#pragma omp parallel num_threads(nt)
    {
        double *m = (double *)malloc(sizeof(double) * (size_t)block_r);
        double *l = (double *)malloc(sizeof(double) * (size_t)block_r);
        double *acc = (double *)malloc(sizeof(double) * (size_t)block_r * (size_t)d_v);
        double *st = (double *)malloc(sizeof(double) * (size_t)block_r * (size_t)block_c);
        if (!m || !l || !acc || !st) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t u = 0; u < units; ++u) {
                const int64_t blk = u % n_blocks;
                const int h = (int)((u / n_blocks) % n_q);
                const int b = (int)(u / (n_blocks * n_q));
                const int g = h / G;
                const double *kb = k + b * k_sb + g * k_sh;
                const double *vb = v + b * v_sb + g * v_sh;
                const int64_t r0 = blk * block_r;
                const int64_t r1 = (r0 + block_r < Sq) ? r0 + block_r : Sq;
                const int br = (int)(r1 - r0);
                /* key range the block visits: up to the widest visible set of
                   its rows (the last row's, since V(i) only grows with i) */
                const int64_t c_limit = visible_end(&p, b, r1 - 1);
                for (int r = 0; r < br; ++r) {
                    m[r] = -INFINITY;
                    l[r] = 0.0;
                    for (int c = 0; c < d_v; ++c) acc[(int64_t)r * d_v + c] = 0.0;
                }
                for (int64_t c0 = 0; c0 < c_limit; c0 += block_c) {
                    const int64_t c1 = (c0 + block_c < c_limit) ? c0 + block_c : c_limit;
                    const int bc = (int)(c1 - c0);
                    for (int r = 0; r < br; ++r) {
                        const int64_t i = r0 + r;
                        const int64_t end = visible_end(&p, b, i);
                        const double *qi = q + (((int64_t)b * n_q + h) * Sq + i) * d_qk;
                        double *srow = st + (int64_t)r * block_c;
                        /* tile scores, masked entries -inf */
                        double tile_max = -INFINITY;
                        for (int jj = 0; jj < bc; ++jj) {
                            const int64_t j = c0 + jj;
                            if (j >= end) {
                                srow[jj] = -INFINITY;
                                continue;
                            }
                            const double *kj = kb + j * k_ss;
                            double a = 0.0;
                            for (int c = 0; c < d_qk; ++c) a += qi[c] * kj[c];
                            srow[jj] = scale * a;
                            if (srow[jj] > tile_max) tile_max = srow[jj];
                        }
                        const double m_new = (tile_max > m[r]) ? tile_max : m[r];
                        if (m_new == -INFINITY) continue; /* nothing visible yet */
                        const double alpha = exp(m[r] - m_new);
                        double rowsum = 0.0;
                        double *ar = acc + (int64_t)r * d_v;
                        for (int c = 0; c < d_v; ++c) ar[c] *= alpha;
                        for (int jj = 0; jj < bc; ++jj) {
                            if (srow[jj] == -INFINITY) continue;
                            const double pj = exp(srow[jj] - m_new);
                            const double *vj = vb + (c0 + jj) * v_ss;
                            rowsum += pj;
                            for (int c = 0; c < d_v; ++c) ar[c] += pj * vj[c];
                        }
                        l[r] = alpha * l[r] + rowsum;
                        m[r] = m_new;
                    }
                }
                for (int r = 0; r < br; ++r) {
                    const int64_t row = ((int64_t)b * n_q + h) * Sq + r0 + r;
                    double *orow = o + row * d_v;
                    if (m[r] == -INFINITY) {
                        for (int c = 0; c < d_v; ++c) orow[c] = 0.0;
                        lse[row] = -INFINITY;
                        continue;
                    }
                    for (int c = 0; c < d_v; ++c) orow[c] = acc[(int64_t)r * d_v + c] / l[r];
                    lse[row] = m[r] + log(l[r]);
                }
            }
        }
        free(m);
        free(l);
        free(acc);
        free(st);
    }
    return err ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Rotary position embedding ("Attention Engineering: From MHA to GQA, MLA &
 * FlashAttention", section 1, Rotary Position Embeddings: the complex-plane
 * derivation and its real 2x2 block form; section 2, the GQA formulation
 * applies it to the queries and the keys before the scores).
 *
 * The head dimension d is split into d/2 planes (x_{2j}, x_{2j+1}). At
 * position m, plane j turns by the angle m * theta_j with the geometric base
 * frequencies theta_j = base^(-2j/d), j = 0 .. d/2-1.
 * ------------------------------------------------------------------------ */

/* cos_t / sin_t [n_pos][d/2]: cos(m theta_j), sin(m theta_j). */
int oracle_rope_tables_fp64(double *cos_t, double *sin_t, int n_pos, int d, double base) {
    if (n_pos < 0 || d <= 0 || d % 2 != 0 || !(base > 0.0)) return -1;
    const int half = d / 2;
    for (int j = 0; j < half; ++j) {
        const double theta = pow(base, -2.0 * (double)j / (double)d);
        for (int m = 0; m < n_pos; ++m) {
            const double a = (double)m * theta;
            cos_t[(int64_t)m * half + j] = cos(a);
            sin_t[(int64_t)m * half + j] = sin(a);
        }
    }
    return 0;
}

/* x, out [n_vec][d]; vector i sits at position pos[i] (a row of the tables).
 * Each plane is multiplied by the rotation matrix [[c, -s], [s, c]]:
 *   out_{2j}   = x_{2j} c - x_{2j+1} s
 *   out_{2j+1} = x_{2j} s + x_{2j+1} c,   c = cos_t[pos][j], s = sin_t[pos][j]. */
int oracle_rope_fp64(const double *x, double *out, int64_t n_vec, int d, const int32_t *pos,
                     const double *cos_t, const double *sin_t, int n_pos) {
    if (n_vec < 0 || d <= 0 || d % 2 != 0) return -1;
    const int half = d / 2;
    for (int64_t i = 0; i < n_vec; ++i) {
        const int m = pos[i];
        if (m < 0 || m >= n_pos) return -1;
        const double *xi = x + i * d;
        double *oi = out + i * d;
        for (int j = 0; j < half; ++j) {
            const double c = cos_t[(int64_t)m * half + j], s = sin_t[(int64_t)m * half + j];
            const double xe = xi[2 * j], xo = xi[2 * j + 1];
            oi[2 * j] = xe * c - xo * s;
            oi[2 * j + 1] = xe * s + xo * c;
        }
    }
    return 0;
}
