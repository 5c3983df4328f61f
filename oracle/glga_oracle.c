/*
 * glga_oracle.c -- float64 CPU oracle for the gated local-global graph-attention layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct statement of
 * what the layer computes.  Only the test-suite, the smoke check and the CPU-baseline leg
 * of the benchmark load it; the library and its Python binding never do.  It shares no
 * code, header or constant with the CUDA implementation.
 *
 * Everything follows the method page "Gated Local-Global Graph Attention" (synthcore idea
 * 2699), section "Key formulas":
 *   L_i = sum_{j : A_ij = 1} softmax_j(q_i k_j^T / sqrt(r)) v_j,  q = x W_Q, k = x W_K,
 *         v = x W_V
 *   G_i = phi(q_i)^T S / (phi(q_i)^T z + eps),  S = sum_{j=1..N} phi(k_j) v_j^T,
 *         z = sum_{j=1..N} phi(k_j)
 *   g_i = sigmoid(x_i w_g + b_g),  Y_i = g_i L_i + (1 - g_i) G_i
 * with phi = elu + 1 (same page, "Implementation notes", item 2), heads of width r taken
 * as consecutive column blocks and concatenated (tinymesh "Sparse attention experiment",
 * section "Multiple heads are composition"), and the stable softmax that subtracts the
 * per-target maximum (tinymesh page, section "Target softmax").
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - A_ij = 1 <=> the edge list holds j -> i; each stored edge is one softmax term,
 *    duplicates included; self-loops come only from the edge list.
 *  - A target with no in-edges has L_i = 0 (an empty weighted sum).
 *  - S and z sum over all N nodes of the call.
 *  - The 1/sqrt(r) scale uses the per-head width and applies to the local scores only.
 *
 * All arithmetic is double.  Inputs arrive as float32 (bf16 inputs arrive already widened
 * exactly to float32) and are widened to double before any product.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------------------------
 * Topology: target-grouped CSR (rows = targets i, entries = sources j, ascending j).
 * tinymesh page, "Target softmax": both segment reductions traverse destination CSR.
 * ------------------------------------------------------------------------------------- */

static int cmp_i32(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Returns 0 on success, -1 if an endpoint is outside [0, N), -2 if E does not fit int32. */
int oracle_csr_from_coo(int64_t N, int64_t E, const int32_t *src, const int32_t *dst,
                        int32_t *row_ptr, int32_t *col_idx) {
    if (E > 2147483647LL) return -2;
    for (int64_t e = 0; e < E; ++e)
        if (src[e] < 0 || src[e] >= N || dst[e] < 0 || dst[e] >= N) return -1;
    /* counting sort by target */
    for (int64_t i = 0; i <= N; ++i) row_ptr[i] = 0;
    for (int64_t e = 0; e < E; ++e) row_ptr[dst[e] + 1] += 1;
    for (int64_t i = 0; i < N; ++i) row_ptr[i + 1] += row_ptr[i];
    int32_t *fill = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    if (!fill) return -3;
    for (int64_t i = 0; i < N; ++i) fill[i] = row_ptr[i];
    for (int64_t e = 0; e < E; ++e) col_idx[fill[dst[e]]++] = src[e];
    free(fill);
    /* ascending source inside every row */
    for (int64_t i = 0; i < N; ++i) {
        int32_t b = row_ptr[i], n = row_ptr[i + 1] - row_ptr[i];
        if (n > 1) qsort(col_idx + b, (size_t)n, sizeof(int32_t), cmp_i32);
    }
    return 0;
}

/* Degree buckets.  Row i with in-degree deg = row_ptr[i+1] - row_ptr[i] goes to
 *   bucket 0 if deg <= warp_max,
 *   bucket 1 if warp_max < deg <= chunk_edges,
 *   bucket 2 otherwise; a bucket-2 row is cut into ceil(deg / chunk_edges) chunks that
 *   start at row_ptr[i] + c * chunk_edges.
 * Bucket 0 lists its rows by descending degree, ties by ascending row; buckets 1 and 2
 * list rows in ascending order; chunks follow their rows' order, then c.
 * counts[0..2] = bucket sizes, counts[3] = number of chunks.  Passing NULL lists only
 * counts.                                                                               */
static const int32_t *g_sort_row_ptr;
static int cmp_deg_desc(const void *a, const void *b) {
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    const int32_t dx = g_sort_row_ptr[x + 1] - g_sort_row_ptr[x];
    const int32_t dy = g_sort_row_ptr[y + 1] - g_sort_row_ptr[y];
    if (dx != dy) return dx > dy ? -1 : 1;
    return (x > y) - (x < y);
}
int oracle_degree_buckets(int64_t N, const int32_t *row_ptr, int32_t warp_max,
                          int32_t chunk_edges, int64_t *counts, int32_t *warp_rows,
                          int32_t *cta_rows, int32_t *split_rows, int32_t *chunk_row,
                          int32_t *chunk_begin) {
    if (warp_max < 0 || chunk_edges < 1 || warp_max > chunk_edges) return -1;
    int64_t n0 = 0, n1 = 0, n2 = 0, nc = 0;
    for (int64_t i = 0; i < N; ++i) {
        int64_t deg = (int64_t)row_ptr[i + 1] - row_ptr[i];
        if (deg <= warp_max) {
            if (warp_rows) warp_rows[n0] = (int32_t)i;
            n0++;
        } else if (deg <= chunk_edges) {
            if (cta_rows) cta_rows[n1] = (int32_t)i;
            n1++;
        } else {
            if (split_rows) split_rows[n2] = (int32_t)i;
            n2++;
            for (int64_t b = 0; b < deg; b += chunk_edges) {
                if (chunk_row) chunk_row[nc] = (int32_t)i;
                if (chunk_begin) chunk_begin[nc] = (int32_t)(row_ptr[i] + b);
                nc++;
            }
        }
    }
    counts[0] = n0; counts[1] = n1; counts[2] = n2; counts[3] = nc;
    if (warp_rows && n0 > 1) {
        g_sort_row_ptr = row_ptr;
        qsort(warp_rows, (size_t)n0, sizeof(int32_t), cmp_deg_desc);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * Projections.  Method page, "Key formulas": q_i = x_i W_Q, k_j = x_j W_K, v_j = x_j W_V;
 * "Key formulas", gate: the logit x_i w_g.  out[i][c] = sum_k X[i][k] * W[k][c].
 * ------------------------------------------------------------------------------------- */
void oracle_project(int64_t n, int32_t d, int32_t D, const float *X, const float *W,
                    double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double *o = out + i * (int64_t)D;
        for (int32_t c = 0; c < D; ++c) o[c] = 0.0;
        const float *x = X + i * (int64_t)d;
        for (int32_t k = 0; k < d; ++k) {
            double xk = (double)x[k];
            const float *w = W + (int64_t)k * D;
            for (int32_t c = 0; c < D; ++c) o[c] += xk * (double)w[c];
        }
    }
}

void oracle_gate_logit(int64_t n, int32_t d, const float *X, const float *w_g, double *t) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double acc = 0.0;
        const float *x = X + i * (int64_t)d;
        for (int32_t k = 0; k < d; ++k) acc += (double)x[k] * (double)w_g[k];
        t[i] = acc;
    }
}

/* phi = elu + 1 (alpha = 1): x + 1 for x > 0, exp(x) otherwise.
 * Method page, "Implementation notes", item 2 ("PhiQ=elu(Q)+1").                         */
double oracle_phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

/* Global statistics per head h: S_h[a][c] = sum_j phi(k_j[h*r+a]) v_j[h*r+c],
 * z_h[a] = sum_j phi(k_j[h*r+a]), j = 0..N-1 in order.  Method page, "Key formulas".     */
void oracle_global_stats(int64_t N, int32_t H, int32_t r, const double *K, const double *V,
                         double *S, double *z) {
    const int64_t D = (int64_t)H * r;
    memset(S, 0, sizeof(double) * (size_t)(H * r * r));
    memset(z, 0, sizeof(double) * (size_t)(H * r));
    double *pk = (double *)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
    for (int64_t j = 0; j < N; ++j) {
        const double *k = K + j * D, *v = V + j * D;
        for (int32_t h = 0; h < H; ++h) {
            for (int32_t a = 0; a < r; ++a) pk[a] = oracle_phi(k[h * r + a]);
            for (int32_t a = 0; a < r; ++a) {
                z[h * r + a] += pk[a];
                double *Srow = S + ((int64_t)h * r + a) * r;
                for (int32_t c = 0; c < r; ++c) Srow[c] += pk[a] * v[h * r + c];
            }
        }
    }
    free(pk);
}

/* ---------------------------------------------------------------------------------------
 * Per-target outputs for a list of target rows.
 *   Q rows: Qrows[m] is q of target rows[m] (only the listed rows are needed);
 *   K, V: all N nodes; t: gate logit of the listed rows; S, z from oracle_global_stats.
 * Writes L, G (each [n_rows][H*r]), g [n_rows] and Y [n_rows][H*r].
 * Local branch: two-pass stable softmax over the CSR row in stored order (max, then the
 * shifted exponentials), tinymesh page "Target softmax"; method page "Key formulas" L_i.
 * Counters (may be NULL): ops[0] += score multiply-adds (edges * r per head),
 * ops[1] += aggregation multiply-adds, ops[2] += readout multiply-adds (r*(r+1) per head).
 * ------------------------------------------------------------------------------------- */
void oracle_rows(int64_t n_rows, const int64_t *rows, int32_t H, int32_t r,
                 const int32_t *row_ptr, const int32_t *col_idx, const double *Qrows,
                 const double *K, const double *V, const double *t, const double *S,
                 const double *z, double b_g, double eps, double *L, double *G, double *g,
                 double *Y, int64_t *ops) {
    const int64_t D = (int64_t)H * r;
    const double inv_sqrt_r = 1.0 / sqrt((double)r);
    int64_t c_score = 0, c_agg = 0, c_read = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(+ : c_score, c_agg, c_read)
    for (int64_t m = 0; m < n_rows; ++m) {
        const int64_t i = rows[m];
        const double *q = Qrows + m * D;
        const int32_t beg = row_ptr[i], end = row_ptr[i + 1];
        double *Lm = L + m * D, *Gm = G + m * D, *Ym = Y + m * D;
        for (int32_t h = 0; h < H; ++h) {
            /* local branch, head h */
            double mx = -INFINITY;
            for (int32_t e = beg; e < end; ++e) {
                const double *k = K + (int64_t)col_idx[e] * D + (int64_t)h * r;
                double s = 0.0;
                for (int32_t a = 0; a < r; ++a) s += q[h * r + a] * k[a];
                s *= inv_sqrt_r;
                if (s > mx) mx = s;
                c_score += r;
            }
            double den = 0.0;
            for (int32_t c = 0; c < r; ++c) Lm[h * r + c] = 0.0;
            for (int32_t e = beg; e < end; ++e) {
                const int64_t j = col_idx[e];
                const double *k = K + j * D + (int64_t)h * r;
                const double *v = V + j * D + (int64_t)h * r;
                double s = 0.0;
                for (int32_t a = 0; a < r; ++a) s += q[h * r + a] * k[a];
                s *= inv_sqrt_r;
                const double p = exp(s - mx);
                den += p;
                for (int32_t c = 0; c < r; ++c) Lm[h * r + c] += p * v[c];
                c_agg += r;
            }
            if (end > beg)
                for (int32_t c = 0; c < r; ++c) Lm[h * r + c] /= den;
            /* global branch readout, head h */
            const double *Sh = S + (int64_t)h * r * r, *zh = z + (int64_t)h * r;
            double qz = 0.0;
            for (int32_t a = 0; a < r; ++a) qz += oracle_phi(q[h * r + a]) * zh[a];
            for (int32_t c = 0; c < r; ++c) {
                double num = 0.0;
                for (int32_t a = 0; a < r; ++a) num += oracle_phi(q[h * r + a]) * Sh[a * r + c];
                Gm[h * r + c] = num / (qz + eps);
            }
            c_read += (int64_t)r * (r + 1);
        }
        /* gate and blend: method page, "Key formulas", g_i and Y_i */
        const double gi = 1.0 / (1.0 + exp(-(t[m] + b_g)));
        g[m] = gi;
        for (int64_t c = 0; c < D; ++c) Ym[c] = gi * Lm[c] + (1.0 - gi) * Gm[c];
    }
    if (ops) { ops[0] += c_score; ops[1] += c_agg; ops[2] += c_read; }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
