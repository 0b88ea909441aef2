/*
 * moe_oracle.c -- plain fp64 CPU oracle of the top-k routed MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code with the CUDA path and is deliberately slow and literal: every loop
 * below is the definition of the quantity it computes, evaluated one token at
 * a time in double precision from the exact stored input values (bf16 and
 * fp32 inputs are widened exactly to double).
 *
 * Sources (page title, section):
 *   - "OmniMoE" technical summary 2.1 (atomic expert E_i(x) = sigma(x w_in^T)
 *     w_out; Dynamic Expert Assembly; shared dense MLP always active) and 2.2
 *     (Cartesian Product Router over an N_r x N_c grid; Expert-Centric
 *     Scheduling: task collection, grouping by expert id, sorting by token id
 *     within each group).
 *   - "PCoMoE" summary, "The Limitation of Monolithic Expert Selection": the
 *     router selects a fixed set of k experts per token.
 *   - "MoE++" summary, "Approach": zero expert (discard), copy expert
 *     (identity), constant expert (trainable vector mixed with the input),
 *     gating residuals carrying the previous layer's router scores.
 * Readings where the pages are silent (all listed in the design notes):
 *   SwiGLU(x) = W_down (silu(W_gate x) * (W_up x)), silu(a) = a/(1+e^-a);
 *   gates = softmax over the k selected logits; ties go to the lower index;
 *   router bias and previous-layer logits are added to the logits; the
 *   constant expert is a1*x + a2*v with (a1,a2) = softmax(W_c x); the atomic
 *   sigma is the exact erf GELU; the product-key score of expert (r, c) is
 *   s_row[r] + s_col[c], expert id r*N_c + c.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1 };

/* Exact widening of one stored element to double. */
static double ld(const void* p, size_t i, int dt)
{
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* sum_i a[i] * W[row, i] with a in double and W stored (row-major, ld = n) */
static double dot_row(const double* a, const void* W, size_t row, int n, int dt)
{
    double s = 0.0;
    size_t base = row * (size_t)n;
    for (int i = 0; i < n; ++i) s += a[i] * ld(W, base + i, dt);
    return s;
}

static void widen_row(const void* X, size_t row, int n, int dt, double* out)
{
    for (int i = 0; i < n; ++i) out[i] = ld(X, row * (size_t)n + i, dt);
}

static double silu(double a) { return a / (1.0 + exp(-a)); }
static double gelu(double a) { return 0.5 * a * (1.0 + erf(a / sqrt(2.0))); }

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------ router */

/* z[t, e] = sum_i x[t, i] W[e, i] + bias[e] + zprev[t, e]   (bias, zprev nullable) */
void orc_router_logits(int T, int d, int E, int dt, const void* x, const void* W,
                       const float* bias, const float* zprev, double* z)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        widen_row(x, (size_t)t, d, dt, xt);
        for (int e = 0; e < E; ++e) {
            double s = dot_row(xt, W, (size_t)e, d, dt);
            if (bias) s += (double)bias[e];
            if (zprev) s += (double)zprev[(size_t)t * E + e];
            z[(size_t)t * E + e] = s;
        }
        free(xt);
    }
}

/*
 * The k largest of z[0..E) in descending order; among equal values the lower
 * index comes first.  gate[j] = exp(z_sel[j] - z_sel[0]) / sum_j' exp(...),
 * i.e. the softmax over the selected logits.  margin = z_sel[k-1] minus the
 * largest unselected logit (+inf when k == E).
 */
static void topk_one(int E, int k, const double* z, int32_t* idx, double* gate,
                     double* margin, unsigned char* taken)
{
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || z[e] > z[best])) best = e;
        taken[best] = 1;
        idx[j] = best;
    }
    double zmax = z[idx[0]], s = 0.0;
    for (int j = 0; j < k; ++j) s += exp(z[idx[j]] - zmax);
    for (int j = 0; j < k; ++j) gate[j] = exp(z[idx[j]] - zmax) / s;
    if (margin) {
        double rest = -INFINITY;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && z[e] > rest) rest = z[e];
        *margin = (k < E) ? z[idx[k - 1]] - rest : INFINITY;
    }
}

void orc_topk(int T, int E, int k, const double* z, int32_t* idx, double* gate,
              double* margin)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
        topk_one(E, k, z + (size_t)t * E, idx + (size_t)t * k, gate + (size_t)t * k,
                 margin ? margin + t : NULL, taken);
        free(taken);
    }
}

/* -------------------------------------------------- expert-centric ordering */

typedef struct { int32_t e, t, j; } task_t;

static int cmp_task(const void* a, const void* b)
{
    const task_t* x = (const task_t*)a;
    const task_t* y = (const task_t*)b;
    if (x->e != y->e) return x->e < y->e ? -1 : 1;
    if (x->t != y->t) return x->t < y->t ? -1 : 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * Task collection, then grouping by expert id and sorting by token id within
 * each group.  Only tasks whose expert id is < n_grouped take part (FFN or
 * atomic experts; zero-computation experts are not grouped).
 *   counts[e]        number of tasks of expert e               [n_grouped]
 *   offsets[e]       first position of expert e's group        [n_grouped + 1]
 *   row_of[t*k + j]  position of task (t, j), -1 if not grouped [T*k]
 *   token_of[p]      token of the task at position p           [R]
 *   slot_of[p]       slot j of the task at position p          [R] (nullable)
 * Returns R, the number of grouped tasks, or -1 on an out-of-range id.
 */
long orc_group_tasks(int T, int k, const int32_t* idx, int n_grouped, int n_ids,
                     int32_t* counts, int32_t* offsets, int32_t* row_of,
                     int32_t* token_of, int32_t* slot_of)
{
    size_t n = (size_t)T * k, R = 0;
    task_t* tasks = (task_t*)malloc(sizeof(task_t) * (n ? n : 1));
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t e = idx[(size_t)t * k + j];
            if (e < 0 || e >= n_ids) { free(tasks); return -1; }
            row_of[(size_t)t * k + j] = -1;
            if (e < n_grouped) { tasks[R].e = e; tasks[R].t = t; tasks[R].j = j; ++R; }
        }
    qsort(tasks, R, sizeof(task_t), cmp_task);
    for (int e = 0; e < n_grouped; ++e) counts[e] = 0;
    for (size_t p = 0; p < R; ++p) {
        counts[tasks[p].e]++;
        token_of[p] = tasks[p].t;
        if (slot_of) slot_of[p] = tasks[p].j;
        row_of[(size_t)tasks[p].t * k + tasks[p].j] = (int32_t)p;
    }
    offsets[0] = 0;
    for (int e = 0; e < n_grouped; ++e) offsets[e + 1] = offsets[e] + counts[e];
    free(tasks);
    return (long)R;
}

/* --------------------------------------------------------- SwiGLU experts */

/* y += w * W_down (silu(W_gate x) * (W_up x)); W_gate, W_up [H, d], W_down [d, H]. */
static void swiglu_acc(int d, int H, int dt, const void* Wg, const void* Wu,
                       const void* Wd, const double* x, double w, double* y, double* h)
{
    for (int i = 0; i < H; ++i)
        h[i] = silu(dot_row(x, Wg, (size_t)i, d, dt)) * dot_row(x, Wu, (size_t)i, d, dt);
    for (int o = 0; o < d; ++o) y[o] += w * dot_row(h, Wd, (size_t)o, H, dt);
}

typedef struct {
    int T, d, top_k, dt;
    int n_ffn, hidden, n_shared, hidden_shared;
    int n_zero, n_copy, n_const;
} orc_layer;

/*
 * The layer output for the listed tokens:
 *   y_t = sum_s SwiGLU_s(x_t)  +  sum_j g_j O_j
 * with O_j = SwiGLU_e(x_t) for an FFN expert, 0 for a zero expert, x_t for a
 * copy expert and a1 x_t + a2 v_c, (a1, a2) = softmax(W_c,c x_t), for a
 * constant expert.  The routing is computed from the logits unless idx_in
 * (n_tok x k) is given, in which case those experts are used and the gates
 * are the softmax of their logits.
 * Outputs (all n_tok rows): y [n_tok, d], idx [n_tok, k], gate [n_tok, k],
 * margin [n_tok] (nullable).
 */
void orc_moe_tokens(const orc_layer* L, const void* x, const void* w_router,
                    const float* bias, const float* zprev,
                    const void* w_gate, const void* w_up, const void* w_down,
                    const void* ws_gate, const void* ws_up, const void* ws_down,
                    const void* w_const_mix, const void* const_vec,
                    int n_tok, const int32_t* tokens, const int32_t* idx_in,
                    double* y, int32_t* idx, double* gate, double* margin)
{
    const int d = L->d, k = L->top_k, H = L->hidden, Hs = L->hidden_shared;
    const int E = L->n_ffn + L->n_zero + L->n_copy + L->n_const;
    const int zero0 = L->n_ffn, copy0 = zero0 + L->n_zero, const0 = copy0 + L->n_copy;
    const int hmax = H > Hs ? H : Hs;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_tok; ++n) {
        const int t = tokens[n];
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        double* z = (double*)malloc(sizeof(double) * (size_t)E);
        double* h = (double*)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
        double* yt = y + (size_t)n * d;
        int32_t* it = idx + (size_t)n * k;
        double* gt = gate + (size_t)n * k;
        widen_row(x, (size_t)t, d, L->dt, xt);
        for (int e = 0; e < E; ++e) {
            z[e] = dot_row(xt, w_router, (size_t)e, d, L->dt);
            if (bias) z[e] += (double)bias[e];
            if (zprev) z[e] += (double)zprev[(size_t)t * E + e];
        }
        if (idx_in) {
            double zmax = -INFINITY, s = 0.0;
            for (int j = 0; j < k; ++j) {
                it[j] = idx_in[(size_t)n * k + j];
                if (z[it[j]] > zmax) zmax = z[it[j]];
            }
            for (int j = 0; j < k; ++j) s += exp(z[it[j]] - zmax);
            for (int j = 0; j < k; ++j) gt[j] = exp(z[it[j]] - zmax) / s;
            if (margin) margin[n] = NAN;
        } else {
            topk_one(E, k, z, it, gt, margin ? margin + n : NULL, taken);
        }
        for (int o = 0; o < d; ++o) yt[o] = 0.0;
        for (int s = 0; s < L->n_shared; ++s) {
            size_t off_in = (size_t)s * Hs * d;   /* [S, Hs, d] and [S, d, Hs] */
            swiglu_acc(d, Hs, L->dt,
                       (const char*)ws_gate + off_in * (L->dt == ORC_F32 ? 4 : 2),
                       (const char*)ws_up + off_in * (L->dt == ORC_F32 ? 4 : 2),
                       (const char*)ws_down + off_in * (L->dt == ORC_F32 ? 4 : 2),
                       xt, 1.0, yt, h);
        }
        for (int j = 0; j < k; ++j) {
            const int e = it[j];
            const double g = gt[j];
            if (e < zero0) {
                size_t off = (size_t)e * H * d * (L->dt == ORC_F32 ? 4 : 2);
                swiglu_acc(d, H, L->dt, (const char*)w_gate + off, (const char*)w_up + off,
                           (const char*)w_down + off, xt, g, yt, h);
            } else if (e < copy0) {
                /* zero expert: contributes nothing */
            } else if (e < const0) {
                for (int o = 0; o < d; ++o) yt[o] += g * xt[o];
            } else {
                const int c = e - const0;
                double l0 = dot_row(xt, w_const_mix, (size_t)(2 * c), d, L->dt);
                double l1 = dot_row(xt, w_const_mix, (size_t)(2 * c + 1), d, L->dt);
                double m = l0 > l1 ? l0 : l1;
                double a1 = exp(l0 - m), a2 = exp(l1 - m), sa = a1 + a2;
                a1 /= sa;
                a2 /= sa;
                for (int o = 0; o < d; ++o)
                    yt[o] += g * (a1 * xt[o] + a2 * ld(const_vec, (size_t)c * d + o, L->dt));
            }
        }
        free(xt); free(z); free(h); free(taken);
    }
}

/* (a1, a2) = softmax(W_c,c x_t) for every token and constant expert: [T, n_const, 2] */
void orc_const_mix(int T, int d, int n_const, int dt, const void* x,
                   const void* w_const_mix, double* a)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        widen_row(x, (size_t)t, d, dt, xt);
        for (int c = 0; c < n_const; ++c) {
            double l0 = dot_row(xt, w_const_mix, (size_t)(2 * c), d, dt);
            double l1 = dot_row(xt, w_const_mix, (size_t)(2 * c + 1), d, dt);
            double m = l0 > l1 ? l0 : l1;
            double a1 = exp(l0 - m), a2 = exp(l1 - m);
            a[((size_t)t * n_const + c) * 2 + 0] = a1 / (a1 + a2);
            a[((size_t)t * n_const + c) * 2 + 1] = a2 / (a1 + a2);
        }
        free(xt);
    }
}

/* ------------------------------------------- Cartesian-product router */

/*
 * q = W_q x_t  (d_query values, not rounded);
 * s_row[r] = sum_i K_row[r, i] q[i]          for the first d_query/2 dims,
 * s_col[c] = sum_i K_col[c, i] q[d_query/2 + i] for the second half.
 * Outputs: s_row [T, rows], s_col [T, cols], q [T, dq] (nullable).
 */
void orc_pk_scores(int T, int d, int dq, int rows, int cols, int dt, const void* x,
                   const void* w_query, const void* k_row, const void* k_col,
                   double* s_row, double* s_col, double* q_out)
{
    const int half = dq / 2;
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        double* q = (double*)malloc(sizeof(double) * (size_t)dq);
        widen_row(x, (size_t)t, d, dt, xt);
        for (int i = 0; i < dq; ++i) q[i] = dot_row(xt, w_query, (size_t)i, d, dt);
        if (q_out) memcpy(q_out + (size_t)t * dq, q, sizeof(double) * (size_t)dq);
        for (int r = 0; r < rows; ++r) s_row[(size_t)t * rows + r] = dot_row(q, k_row, (size_t)r, half, dt);
        for (int c = 0; c < cols; ++c) s_col[(size_t)t * cols + c] = dot_row(q + half, k_col, (size_t)c, half, dt);
        free(xt); free(q);
    }
}

/*
 * Product-key selection for one token: the top-kh rows of s_row and top-kh
 * columns of s_col (ties to the lower sub-index); the kh*kh candidate experts
 * (r, c) with score s_row[r] + s_col[c] and id r*cols + c; the K best by
 * descending score, ties to the lower id; gates = softmax over the K scores.
 * margins: [0] row kh-th minus (kh+1)-th, [1] same for columns, [2] K-th minus
 * (K+1)-th candidate (+inf where nothing is left out).
 */
static void pk_select_one(int rows, int cols, int kh, int K, const double* sr,
                          const double* sc, int32_t* idx, double* gate, double* mg,
                          int32_t* wr, int32_t* wc, double* cand_s, int32_t* cand_id,
                          unsigned char* taken)
{
    /* top-kh of each half, with the same ordering rule as the router's top-k */
    double* gtmp = (double*)malloc(sizeof(double) * (size_t)(kh > K ? kh : K));
    unsigned char* tk = (unsigned char*)malloc((size_t)(rows > cols ? rows : cols));
    topk_one(rows, kh, sr, wr, gtmp, &mg[0], tk);
    topk_one(cols, kh, sc, wc, gtmp, &mg[1], tk);
    int nc = kh * kh;
    for (int a = 0; a < kh; ++a)
        for (int b = 0; b < kh; ++b) {
            cand_s[a * kh + b] = sr[wr[a]] + sc[wc[b]];
            cand_id[a * kh + b] = wr[a] * cols + wc[b];
        }
    memset(taken, 0, (size_t)nc);
    for (int j = 0; j < K; ++j) {
        int best = -1;
        for (int p = 0; p < nc; ++p) {
            if (taken[p]) continue;
            if (best < 0 || cand_s[p] > cand_s[best] ||
                (cand_s[p] == cand_s[best] && cand_id[p] < cand_id[best]))
                best = p;
        }
        taken[best] = 1;
        idx[j] = cand_id[best];
        gate[j] = cand_s[best];
    }
    double rest = -INFINITY;
    for (int p = 0; p < nc; ++p)
        if (!taken[p] && cand_s[p] > rest) rest = cand_s[p];
    mg[2] = (K < nc) ? gate[K - 1] - rest : INFINITY;
    double m = gate[0], s = 0.0;
    for (int j = 0; j < K; ++j) s += exp(gate[j] - m);
    for (int j = 0; j < K; ++j) gate[j] = exp(gate[j] - m) / s;
    free(gtmp); free(tk);
}

void orc_pk_select(int T, int rows, int cols, int kh, int K, const double* s_row,
                   const double* s_col, int32_t* idx, double* gate, double* margins)
{
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        int32_t* wr = (int32_t*)malloc(sizeof(int32_t) * (size_t)kh);
        int32_t* wc = (int32_t*)malloc(sizeof(int32_t) * (size_t)kh);
        double* cs = (double*)malloc(sizeof(double) * (size_t)kh * kh);
        int32_t* ci = (int32_t*)malloc(sizeof(int32_t) * (size_t)kh * kh);
        unsigned char* taken = (unsigned char*)malloc((size_t)kh * kh);
        pk_select_one(rows, cols, kh, K, s_row + (size_t)t * rows, s_col + (size_t)t * cols,
                      idx + (size_t)t * K, gate + (size_t)t * K, margins + (size_t)t * 3,
                      wr, wc, cs, ci, taken);
        free(wr); free(wc); free(cs); free(ci); free(taken);
    }
}

/*
 * Atomic-expert layer output for the listed tokens, given their routing
 * (idx, gate as K values per listed token):
 *   y_t = sum_j g_j * GELU(u_e . x_t) * v_e,  e = idx[j].
 */
void orc_atomic_tokens(int d, int K, int dt, const void* x, const void* u, const void* v,
                       int n_tok, const int32_t* tokens, const int32_t* idx,
                       const double* gate, double* y)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_tok; ++n) {
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        double* yt = y + (size_t)n * d;
        widen_row(x, (size_t)tokens[n], d, dt, xt);
        for (int o = 0; o < d; ++o) yt[o] = 0.0;
        for (int j = 0; j < K; ++j) {
            const int32_t e = idx[(size_t)n * K + j];
            const double c = gate[(size_t)n * K + j] * gelu(dot_row(xt, u, (size_t)e, d, dt));
            for (int o = 0; o < d; ++o) yt[o] += c * ld(v, (size_t)e * d + o, dt);
        }
        free(xt);
    }
}

/*
 * The full OmniMoE layer ("OmniMoE" 2.1: a shared dense MLP branch, always
 * active, beside the routed atomic experts) for the listed tokens:
 *   y_t = sum_s SwiGLU_s(x_t) + sum_j g_j * GELU(u_e . x_t) * v_e
 * with the shared branches in the layer's SwiGLU form (ws_gate, ws_up
 * [n_shared, Hs, d], ws_down [n_shared, d, Hs]) and weight 1.
 */
void orc_omni_tokens(int d, int K, int dt, const void* x, const void* u, const void* v,
                     int n_shared, int Hs, const void* ws_gate, const void* ws_up, const void* ws_down,
                     int n_tok, const int32_t* tokens, const int32_t* idx, const double* gate, double* y)
{
    orc_atomic_tokens(d, K, dt, x, u, v, n_tok, tokens, idx, gate, y);
    const size_t eb = dt == ORC_F32 ? 4 : 2;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_tok; ++n) {
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        double* h = (double*)malloc(sizeof(double) * (size_t)(Hs > 0 ? Hs : 1));
        widen_row(x, (size_t)tokens[n], d, dt, xt);
        for (int sh = 0; sh < n_shared; ++sh) {
            const size_t off = (size_t)sh * Hs * d * eb;
            swiglu_acc(d, Hs, dt, (const char*)ws_gate + off, (const char*)ws_up + off,
                       (const char*)ws_down + off, xt, 1.0, y + (size_t)n * d, h);
        }
        free(xt);
        free(h);
    }
}

/* ---------------------------------------------------------- FP8 experts */
/*
 * "PCoMoE" summary, "Improvements", 3 (Mixed Precision Execution): the
 * expert computation in FP8, the gating in BF16.  FP8 here is E4M3: sign, 4
 * exponent bits (bias 7), 3 mantissa bits; largest finite value 448,
 * smallest normal 2^-6, subnormals spaced 2^-9; the code with all exponent
 * and mantissa bits set is NaN.
 *   stored expert weights: an e4m3 code per element and an fp32 scale per
 *     output row; the weight is code value * scale (read exactly here);
 *   activations (x, then the hidden h): each row is divided by the smallest
 *     power of two s with 448 s >= max|row| and rounded to the nearest e4m3
 *     value (ties to even); the row is then s * codes.  A power-of-two scale
 *     makes the division exact, so the rounding decisions are those of the
 *     definition whatever the precision of the arithmetic;
 *   the hidden activation is rounded to bf16 (nearest, ties to even) before
 *     its quantization: it is stored so between the two expert GEMMs.
 */

double orc_e4m3_decode(uint8_t b)
{
    const int e = (b >> 3) & 15, m = b & 7;
    const double s = (b & 0x80) ? -1.0 : 1.0;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return s * ldexp((double)m, -9);
    return s * ldexp(1.0 + m / 8.0, e - 7);
}

/* Nearest e4m3 value to v, ties to even mantissa; |v| >= 448 gives +-448. */
double orc_e4m3_round(double v)
{
    if (v != v) return v;
    const double a = fabs(v), sg = v < 0 ? -1.0 : 1.0;
    if (a >= 448.0) return sg * 448.0;
    double q;                                   /* spacing of the e4m3 values around a */
    if (a < ldexp(1.0, -6)) {
        q = ldexp(1.0, -9);
    } else {
        int ex;
        frexp(a, &ex);                          /* a in [2^(ex-1), 2^ex) */
        q = ldexp(1.0, ex - 1 - 3);
    }
    return sg * nearbyint(a / q) * q;           /* a / q exact; nearbyint: ties to even */
}

/* Nearest bf16 value to v (8 significant bits), ties to even. */
static double bf16_round(double v)
{
    if (v == 0.0 || v != v || isinf(v)) return v;
    int ex;
    frexp(fabs(v), &ex);
    if (ex - 1 < -126) ex = -125;               /* subnormal range: fixed spacing 2^-133 */
    const double q = ldexp(1.0, ex - 1 - 7);
    return nearbyint(v / q) * q;
}

/* The smallest power of two s with 448 s >= amax (1 for amax == 0). */
double orc_pow2_scale(double amax)
{
    if (!(amax > 0.0)) return 1.0;
    int ex;
    frexp(amax, &ex);                           /* amax in [2^(ex-1), 2^ex) */
    int e = ex - 9;                             /* 448 * 2^(ex-9) = 0.875 * 2^ex: at or near amax */
    while (448.0 * ldexp(1.0, e) < amax) ++e;
    while (448.0 * ldexp(1.0, e - 1) >= amax) --e;
    return ldexp(1.0, e);
}

/* One row of n values quantized: codes (as values) q[i] and the scale. */
static double quantize_row(const double* v, int n, double* q)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i)
        if (fabs(v[i]) > amax) amax = fabs(v[i]);
    const double s = orc_pow2_scale(amax);
    for (int i = 0; i < n; ++i) q[i] = orc_e4m3_round(v[i] / s);
    return s;
}

/* Rows of x (n rows of d, dtype dt) quantized: q [n, d] (e4m3 values), scale [n]. */
void orc_quantize_rows(int n, int d, int dt, const void* x, double* q, double* scale)
{
    double* row = (double*)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
    for (int r = 0; r < n; ++r) {
        widen_row(x, (size_t)r, d, dt, row);
        scale[r] = quantize_row(row, d, q + (size_t)r * d);
    }
    free(row);
}

/* sum_i a[i] * W[row, i] with W an e4m3 code matrix (row-major, ld = n). */
static double dot_row_e4m3(const double* a, const uint8_t* W, size_t row, int n)
{
    double s = 0.0;
    const uint8_t* w = W + row * (size_t)n;
    for (int i = 0; i < n; ++i) s += a[i] * orc_e4m3_decode(w[i]);
    return s;
}

/*
 * One FP8 SwiGLU expert on one token, y += w * out:
 *   x quantized (sx, x8);  g_i = sx sg_i (x8 . Wg8_i),  u_i = sx su_i (x8 . Wu8_i);
 *   h_i = bf16(silu(g_i) u_i);  h quantized (sh, h8);  out_o = sh sd_o (h8 . Wd8_o).
 * Wg8, Wu8 [H, d], Wd8 [d, H] codes; sg, su [H], sd [d] row scales.
 */
static void swiglu_fp8_acc(int d, int H, const uint8_t* Wg, const float* sg, const uint8_t* Wu, const float* su,
                           const uint8_t* Wd, const float* sd, const double* x8, double sx, double w, double* y,
                           double* h, double* h8)
{
    for (int i = 0; i < H; ++i) {
        const double g = sx * (double)sg[i] * dot_row_e4m3(x8, Wg, (size_t)i, d);
        const double u = sx * (double)su[i] * dot_row_e4m3(x8, Wu, (size_t)i, d);
        h[i] = bf16_round(silu(g) * u);
    }
    const double sh = quantize_row(h, H, h8);
    for (int o = 0; o < d; ++o) y[o] += w * sh * (double)sd[o] * dot_row_e4m3(h8, Wd, (size_t)o, H);
}

/*
 * The layer output for the listed tokens with FP8 experts: routing, zero /
 * copy / constant experts and the combine exactly as orc_moe_tokens (bf16
 * or fp32 x, router and MoE++ tensors of type L->dt); every FFN and shared
 * expert is swiglu_fp8_acc with its codes and row scales (routed [n_ffn, ...],
 * shared [n_shared, ...]).
 */
void orc_fp8_moe_tokens(const orc_layer* L, const void* x, const void* w_router, const float* bias,
                        const float* zprev, const uint8_t* wg8, const float* sg, const uint8_t* wu8,
                        const float* su, const uint8_t* wd8, const float* sd, const uint8_t* sg8,
                        const float* ssg, const uint8_t* su8, const float* ssu, const uint8_t* sd8,
                        const float* ssd, const void* w_const_mix, const void* const_vec, int n_tok,
                        const int32_t* tokens, const int32_t* idx_in, double* y, int32_t* idx, double* gate,
                        double* margin)
{
    const int d = L->d, k = L->top_k, H = L->hidden, Hs = L->hidden_shared;
    const int E = L->n_ffn + L->n_zero + L->n_copy + L->n_const;
    const int zero0 = L->n_ffn, copy0 = zero0 + L->n_zero, const0 = copy0 + L->n_copy;
    const int hmax = H > Hs ? H : Hs;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int n = 0; n < n_tok; ++n) {
        const int t = tokens[n];
        double* xt = (double*)malloc(sizeof(double) * (size_t)d);
        double* x8 = (double*)malloc(sizeof(double) * (size_t)d);
        double* z = (double*)malloc(sizeof(double) * (size_t)E);
        double* h = (double*)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
        double* h8 = (double*)malloc(sizeof(double) * (size_t)(hmax > 0 ? hmax : 1));
        unsigned char* taken = (unsigned char*)malloc((size_t)E);
        double* yt = y + (size_t)n * d;
        int32_t* it = idx + (size_t)n * k;
        double* gt = gate + (size_t)n * k;
        widen_row(x, (size_t)t, d, L->dt, xt);
        for (int e = 0; e < E; ++e) {
            z[e] = dot_row(xt, w_router, (size_t)e, d, L->dt);
            if (bias) z[e] += (double)bias[e];
            if (zprev) z[e] += (double)zprev[(size_t)t * E + e];
        }
        if (idx_in) {
            double zmax = -INFINITY, s = 0.0;
            for (int j = 0; j < k; ++j) {
                it[j] = idx_in[(size_t)n * k + j];
                if (z[it[j]] > zmax) zmax = z[it[j]];
            }
            for (int j = 0; j < k; ++j) s += exp(z[it[j]] - zmax);
            for (int j = 0; j < k; ++j) gt[j] = exp(z[it[j]] - zmax) / s;
            if (margin) margin[n] = NAN;
        } else {
            topk_one(E, k, z, it, gt, margin ? margin + n : NULL, taken);
        }
        const double sx = quantize_row(xt, d, x8);
        for (int o = 0; o < d; ++o) yt[o] = 0.0;
        for (int s = 0; s < L->n_shared; ++s) {
            const size_t wo = (size_t)s * Hs * d;
            swiglu_fp8_acc(d, Hs, sg8 + wo, ssg + (size_t)s * Hs, su8 + wo, ssu + (size_t)s * Hs, sd8 + wo,
                           ssd + (size_t)s * d, x8, sx, 1.0, yt, h, h8);
        }
        for (int j = 0; j < k; ++j) {
            const int e = it[j];
            const double g = gt[j];
            if (e < zero0) {
                const size_t wo = (size_t)e * H * d;
                swiglu_fp8_acc(d, H, wg8 + wo, sg + (size_t)e * H, wu8 + wo, su + (size_t)e * H, wd8 + wo,
                               sd + (size_t)e * d, x8, sx, g, yt, h, h8);
            } else if (e < copy0) {
                /* zero expert: contributes nothing */
            } else if (e < const0) {
                for (int o = 0; o < d; ++o) yt[o] += g * xt[o];
            } else {
                const int c = e - const0;
                double l0 = dot_row(xt, w_const_mix, (size_t)(2 * c), d, L->dt);
                double l1 = dot_row(xt, w_const_mix, (size_t)(2 * c + 1), d, L->dt);
                double m = l0 > l1 ? l0 : l1;
                double a1 = exp(l0 - m), a2 = exp(l1 - m), sa = a1 + a2;
                a1 /= sa;
                a2 /= sa;
                for (int o = 0; o < d; ++o)
                    yt[o] += g * (a1 * xt[o] + a2 * ld(const_vec, (size_t)c * d + o, L->dt));
            }
        }
        free(xt); free(x8); free(z); free(h); free(h8); free(taken);
    }
}
