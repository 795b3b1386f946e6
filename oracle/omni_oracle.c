/*
 * omni_oracle.c -- plain, slow CPU oracle for the routed branch of an OmniMoE
 * layer.  TEST INFRASTRUCTURE ONLY: it is called by tests/, by the smoke check
 * in __graft_entry__.py and by the cpu_baseline leg of bench.py, never by the
 * library.  It shares no code with the CUDA path (no headers, helpers, tables).
 *
 * Sources (cited by page title and section):
 *   [R]  "OmniMoE: An Efficient MoE by Orchestrating Atomic Experts at Scale",
 *        review at paper.rainbus.top, method paragraph.  Step 1: atomic expert
 *        E_i(x) = sigma(x w_in_i^T) w_out_i, global matrices W, V, retrieval
 *        w_x = W[I_x], assembly y = (g_x . sigma(x w_x^T)) v_x + MLP(x).
 *        Step 2: Cartesian product router s_r = x W_r, s_c = x W_c, LogSoftmax
 *        to p_r, p_c, implicit score S_ij = p_r[i] + p_c[j], global top-K.
 *        Step 3: expert-centric scheduling: M = L*K tasks, sorted by expert id,
 *        contiguous groups of B, hierarchical order (group id, token id), then
 *        per active group O_q = (G_q . sigma(X_q W_q^T)) V_q.
 *   [G]  same title, gist.science summary (German edition), section 2.2
 *        "Experten-zentriertes Scheduling": groups are contiguous ranges of
 *        expert ids, tokens sorted inside each group.  Section 2.1
 *        "Kernkomponenten": a standard dense MLP branch, active for every
 *        input, runs beside the routed one.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - sigma is SiLU, z / (1 + exp(-z)) (each expert has a single w_in, so the
 *     SwiGLU named in [R] has no gate vector to multiply).
 *   - expert id n = i * N_c + j for grid cell (i, j).
 *   - g_x is the softmax over the K selected scores S.
 *   - order key of a grid cell: (S desc, p_r[i] desc, p_c[j] desc, n asc);
 *     row and column ranks use (p desc, index asc).
 *   - S_ij is one IEEE fp32 addition of the fp32 log-probabilities.
 *   - group of expert e is q = floor(e / B); inside a group tasks are ordered
 *     by (token, e).
 *   - W_r is stored as N_r rows of d (the transpose of the d x N_r matrix of
 *     [R]), likewise W_c, so s_r[i] = sum_k x[k] * W_r[i][k].
 *   - the shared MLP is the gated (SwiGLU) form with hidden width F:
 *     MLP(x) = (SiLU(x W_g^T) * (x W_u^T)) W_d^T.
 *
 * Floating point: everything is fp64 except where the method fixes fp32 (the
 * log-probabilities that selection runs on, S, and the returned gates).  bf16
 * inputs arrive as uint16 bit patterns and are widened exactly.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (no -ffast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- bf16 bit pattern -> double (exact) -------------------------------- */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- Step 2 of [R]: s = x W^T, p = LogSoftmax(s) -------------------------
 * One axis at a time: Wt is n_out rows of d.  p is computed in fp64 as
 * s - (max + log(sum exp(s - max))) and rounded once to fp32.            */
static void logsoftmax_axis(const uint16_t *x, const uint16_t *Wt, int L, int d,
                            int n_out, float *p) {
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)n_out);
        double *xr = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 4)
        for (int t = 0; t < L; ++t) {
            for (int k = 0; k < d; ++k) xr[k] = bf16_to_double(x[(size_t)t * d + k]);
            double mx = -INFINITY;
            for (int i = 0; i < n_out; ++i) {
                const uint16_t *w = Wt + (size_t)i * d;
                double acc = 0.0;
                for (int k = 0; k < d; ++k) acc += xr[k] * bf16_to_double(w[k]);
                s[i] = acc;
                if (acc > mx) mx = acc;
            }
            double sum = 0.0;
            for (int i = 0; i < n_out; ++i) sum += exp(s[i] - mx);
            double lse = mx + log(sum);
            for (int i = 0; i < n_out; ++i) p[(size_t)t * n_out + i] = (float)(s[i] - lse);
        }
        free(s);
        free(xr);
    }
}

int oracle_router_logprobs(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c,
                           int L, int d, int N_r, int N_c, float *p_r, float *p_c,
                           int nthreads) {
    if (L < 0 || d <= 0 || N_r <= 0 || N_c <= 0) return -1;
    set_threads(nthreads);
    logsoftmax_axis(x, W_r, L, d, N_r, p_r);
    logsoftmax_axis(x, W_c, L, d, N_c, p_c);
    return 0;
}

/* ---- Step 2 of [R]: exact global top-K over the implicit grid ------------ */
typedef struct { float p; int32_t i; } axis_item;

/* rank order on one axis: p desc, index asc */
static int axis_cmp(const void *a, const void *b) {
    const axis_item *u = (const axis_item *)a, *v = (const axis_item *)b;
    if (u->p > v->p) return -1;
    if (u->p < v->p) return 1;
    return (u->i > v->i) - (u->i < v->i);
}

typedef struct { float S, pr, pc; int64_t n; } cell;

/* grid-cell order: S desc, p_r desc, p_c desc, n asc */
static int cell_cmp(const void *a, const void *b) {
    const cell *u = (const cell *)a, *v = (const cell *)b;
    if (u->S > v->S) return -1;
    if (u->S < v->S) return 1;
    if (u->pr > v->pr) return -1;
    if (u->pr < v->pr) return 1;
    if (u->pc > v->pc) return -1;
    if (u->pc < v->pc) return 1;
    return (u->n > v->n) - (u->n < v->n);
}

/* fp32 addition with a single rounding (volatile keeps it in fp32 storage) */
static float add_f32(float a, float b) {
    volatile float s = a + b;
    return s;
}

/*
 * For each token: rank rows by p_r and columns by p_c, keep the first
 * min(K, N_r) rows and min(K, N_c) columns, form every cell (a, b) of that
 * block whose ranks satisfy (a+1)(b+1) <= K, and keep the K best cells by the
 * grid-cell order.  Any cell outside that set has at least K cells that rank
 * above it (all cells dominating it in both ranks), so the K best of the set
 * are the K best of the whole N_r x N_c grid -- the grid is never built.
 * Outputs per token, in grid-cell order: idx = n, score = S, gate = softmax(S).
 * Returns 0, -1 on bad sizes, -2 if a log-probability is NaN or infinite.
 */
int oracle_topk_from_logprobs(const float *p_r, const float *p_c, int L, int N_r, int N_c,
                              int K, int32_t *idx, float *score, float *gate, int nthreads) {
    if (L < 0 || N_r <= 0 || N_c <= 0 || K <= 0) return -1;
    if ((int64_t)K > (int64_t)N_r * (int64_t)N_c) return -1;
    for (int64_t u = 0; u < (int64_t)L * N_r; ++u) if (!isfinite(p_r[u])) return -2;
    for (int64_t u = 0; u < (int64_t)L * N_c; ++u) if (!isfinite(p_c[u])) return -2;
    set_threads(nthreads);
    const int Kr = K < N_r ? K : N_r;
    const int Kc = K < N_c ? K : N_c;
    #pragma omp parallel
    {
        axis_item *rows = (axis_item *)malloc(sizeof(axis_item) * (size_t)N_r);
        axis_item *cols = (axis_item *)malloc(sizeof(axis_item) * (size_t)N_c);
        cell *cand = (cell *)malloc(sizeof(cell) * ((size_t)Kr * (size_t)Kc));
        #pragma omp for schedule(dynamic, 8)
        for (int t = 0; t < L; ++t) {
            for (int i = 0; i < N_r; ++i) { rows[i].p = p_r[(size_t)t * N_r + i]; rows[i].i = i; }
            for (int j = 0; j < N_c; ++j) { cols[j].p = p_c[(size_t)t * N_c + j]; cols[j].i = j; }
            qsort(rows, (size_t)N_r, sizeof(axis_item), axis_cmp);
            qsort(cols, (size_t)N_c, sizeof(axis_item), axis_cmp);
            int nc = 0;
            for (int a = 0; a < Kr; ++a) {
                for (int b = 0; b < Kc; ++b) {
                    if ((int64_t)(a + 1) * (b + 1) > K) break;
                    cell c;
                    c.pr = rows[a].p;
                    c.pc = cols[b].p;
                    c.S = add_f32(c.pr, c.pc);
                    c.n = (int64_t)rows[a].i * N_c + cols[b].i;
                    cand[nc++] = c;
                }
            }
            qsort(cand, (size_t)nc, sizeof(cell), cell_cmp);
            /* gate: softmax over the K selected scores, fp64, rounded once */
            double smax = (double)cand[0].S, den = 0.0;
            for (int k = 0; k < K; ++k) den += exp((double)cand[k].S - smax);
            for (int k = 0; k < K; ++k) {
                idx[(size_t)t * K + k] = (int32_t)cand[k].n;
                score[(size_t)t * K + k] = cand[k].S;
                gate[(size_t)t * K + k] = (float)(exp((double)cand[k].S - smax) / den);
            }
        }
        free(rows);
        free(cols);
        free(cand);
    }
    return 0;
}

/* ---- Step 3 of [R]: expert-centric schedule ------------------------------ */
typedef struct { int64_t q, t, e; float g; } task;

static int task_cmp(const void *a, const void *b) {
    const task *u = (const task *)a, *v = (const task *)b;
    if (u->q != v->q) return u->q < v->q ? -1 : 1;
    if (u->t != v->t) return u->t < v->t ? -1 : 1;
    return (u->e > v->e) - (u->e < v->e);
}

/*
 * Tasks m = t*K + k carry (t, e = idx[t,k], g = gate[t,k]).  They are sorted by
 * (q = e div B, t, e); group_counts[q] is the number of tasks of group q,
 * group_offsets its exclusive prefix sum (G+1 entries), active_groups the
 * groups with a task in ascending order (num_active of them; the rest of the
 * array is left untouched), num_distinct the number of distinct experts.
 * Returns 0, -1 on bad sizes, -3 if an expert id is out of [0, N).
 */
int oracle_schedule(const int32_t *idx, const float *gate, int L, int K, int N, int B,
                    int32_t *task_token, int32_t *task_expert, float *task_gate,
                    int32_t *group_offsets, int32_t *group_counts, int32_t *active_groups,
                    int32_t *num_active, int32_t *num_distinct) {
    if (L < 0 || K <= 0 || N <= 0 || B <= 0) return -1;
    const int64_t M = (int64_t)L * K;
    const int64_t G = ((int64_t)N + B - 1) / B;
    task *ts = (task *)malloc(sizeof(task) * (size_t)(M > 0 ? M : 1));
    unsigned char *seen = (unsigned char *)calloc((size_t)N, 1);
    for (int64_t m = 0; m < M; ++m) {
        int64_t e = idx[m];
        if (e < 0 || e >= N) { free(ts); free(seen); return -3; }
        ts[m].t = m / K;
        ts[m].e = e;
        ts[m].q = e / B;
        ts[m].g = gate[m];
    }
    qsort(ts, (size_t)M, sizeof(task), task_cmp);
    for (int64_t q = 0; q < G; ++q) group_counts[q] = 0;
    int64_t distinct = 0;
    for (int64_t m = 0; m < M; ++m) {
        task_token[m] = (int32_t)ts[m].t;
        task_expert[m] = (int32_t)ts[m].e;
        task_gate[m] = ts[m].g;
        group_counts[ts[m].q] += 1;
        if (!seen[ts[m].e]) { seen[ts[m].e] = 1; ++distinct; }
    }
    int64_t run = 0, na = 0;
    for (int64_t q = 0; q < G; ++q) {
        group_offsets[q] = (int32_t)run;
        run += group_counts[q];
        if (group_counts[q] > 0) active_groups[na++] = (int32_t)q;
    }
    group_offsets[G] = (int32_t)run;
    *num_active = (int32_t)na;
    *num_distinct = (int32_t)distinct;
    free(ts);
    free(seen);
    return 0;
}

/* ---- Step 1 of [R]: DEA assembly, token-centric --------------------------
 * y[r, :] = sum_k g[t,k] * SiLU(x_t . W[e_k]) * V[e_k]  for t = tokens[r],
 * in fp64 over the exact bf16 inputs.  tokens == NULL means r = t = 0..n-1.  */
static double silu(double z) { return z / (1.0 + exp(-z)); }

int oracle_expert_fwd_token_centric(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                    int d, int K, const int32_t *idx, const float *gate,
                                    const int32_t *tokens, int n_tokens, double *y,
                                    int nthreads) {
    if (d <= 0 || K <= 0 || n_tokens < 0) return -1;
    set_threads(nthreads);
    #pragma omp parallel
    {
        double *xr = (double *)malloc(sizeof(double) * (size_t)d);
        #pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < n_tokens; ++r) {
            const int64_t t = tokens ? tokens[r] : r;
            double *yr = y + (size_t)r * d;
            for (int c = 0; c < d; ++c) { xr[c] = bf16_to_double(x[(size_t)t * d + c]); yr[c] = 0.0; }
            for (int k = 0; k < K; ++k) {
                const int64_t e = idx[(size_t)t * K + k];
                const uint16_t *w = W + (size_t)e * d;
                const uint16_t *v = V + (size_t)e * d;
                double h = 0.0;
                for (int c = 0; c < d; ++c) h += xr[c] * bf16_to_double(w[c]);
                const double coef = (double)gate[(size_t)t * K + k] * silu(h);
                for (int c = 0; c < d; ++c) yr[c] += coef * bf16_to_double(v[c]);
            }
        }
        free(xr);
    }
    return 0;
}

/* ---- Step 3 of [R]: DEA assembly, expert-centric -------------------------
 * For each active group q: X_q = rows of its distinct tokens, W_q, V_q = rows of
 * its distinct experts, G_q[t][e] = gate of task (t, e) or 0, and
 * O_q = (G_q . SiLU(X_q W_q^T)) V_q is added into y row by row.  Dense per
 * group, fp64, single-threaded.                                            */
int oracle_expert_fwd_expert_centric(const uint16_t *x, const uint16_t *W, const uint16_t *V,
                                     int L, int d, int N, int B,
                                     const int32_t *task_token, const int32_t *task_expert,
                                     const float *task_gate, const int32_t *group_offsets,
                                     const int32_t *active_groups, int num_active, double *y) {
    if (L < 0 || d <= 0 || N <= 0 || B <= 0) return -1;
    for (int64_t u = 0; u < (int64_t)L * d; ++u) y[u] = 0.0;
    for (int a = 0; a < num_active; ++a) {
        const int64_t q = active_groups[a];
        const int64_t m0 = group_offsets[q], m1 = group_offsets[q + 1];
        /* distinct tokens and experts of the group */
        int64_t nt = 0, ne = 0;
        int64_t *toks = (int64_t *)malloc(sizeof(int64_t) * (size_t)(m1 - m0));
        int64_t *exps = (int64_t *)malloc(sizeof(int64_t) * (size_t)(m1 - m0));
        for (int64_t m = m0; m < m1; ++m) {
            int64_t t = task_token[m], e = task_expert[m], f;
            for (f = 0; f < nt && toks[f] != t; ++f) {}
            if (f == nt) toks[nt++] = t;
            for (f = 0; f < ne && exps[f] != e; ++f) {}
            if (f == ne) exps[ne++] = e;
        }
        double *Gq = (double *)calloc((size_t)(nt * ne), sizeof(double));
        for (int64_t m = m0; m < m1; ++m) {
            int64_t ti = 0, ei = 0;
            while (toks[ti] != task_token[m]) ++ti;
            while (exps[ei] != task_expert[m]) ++ei;
            Gq[ti * ne + ei] = (double)task_gate[m];
        }
        /* P = G_q . SiLU(X_q W_q^T), then O_q = P V_q */
        double *P = (double *)malloc(sizeof(double) * (size_t)(nt * ne));
        for (int64_t ti = 0; ti < nt; ++ti) {
            for (int64_t ei = 0; ei < ne; ++ei) {
                double h = 0.0;
                for (int c = 0; c < d; ++c)
                    h += bf16_to_double(x[(size_t)toks[ti] * d + c]) *
                         bf16_to_double(W[(size_t)exps[ei] * d + c]);
                P[ti * ne + ei] = Gq[ti * ne + ei] * silu(h);
            }
        }
        for (int64_t ti = 0; ti < nt; ++ti) {
            double *yr = y + (size_t)toks[ti] * d;
            for (int c = 0; c < d; ++c) {
                double o = 0.0;
                for (int64_t ei = 0; ei < ne; ++ei)
                    o += P[ti * ne + ei] * bf16_to_double(V[(size_t)exps[ei] * d + c]);
                yr[c] += o;
            }
        }
        free(toks);
        free(exps);
        free(Gq);
        free(P);
    }
    return 0;
}

/* ---- Backward of the routed branch ----------------------------------------
 * The pages give no backward; it is the derivative of the forward above with
 * the top-K selection held fixed (a selection has no gradient).
 *
 * Expert part, for each task (t, k), e = idx[t,k], g = gate[t,k]:
 *   h = x_t . w_e,  a = SiLU(h),  c = dy_t . v_e
 *   dgate[t,k] = a c
 *   dV[e] += g a dy_t
 *   dh = g c SiLU'(h),  SiLU'(h) = s (1 + h (1 - s)),  s = 1 / (1 + exp(-h))
 *   dW[e] += dh x_t,    dx_t += dh w_e
 * W and V may be passed compacted to the rows the tokens use (idx then holds
 * row numbers 0..rows-1); dW and dV are [rows, d].  dx, dW, dV, dgate are
 * overwritten.  fp64, single-threaded (the scatter into dW, dV is ordered). */
static double silu_grad(double z) {
    const double s = 1.0 / (1.0 + exp(-z));
    return s * (1.0 + z * (1.0 - s));
}

int oracle_expert_bwd(const uint16_t *x, const uint16_t *W, const uint16_t *V, int L, int d,
                      int K, int rows, const int32_t *idx, const float *gate, const float *dy,
                      double *dx, double *dW, double *dV, double *dgate) {
    if (L < 0 || d <= 0 || K <= 0 || rows <= 0) return -1;
    for (int64_t u = 0; u < (int64_t)L * d; ++u) dx[u] = 0.0;
    for (int64_t u = 0; u < (int64_t)rows * d; ++u) { dW[u] = 0.0; dV[u] = 0.0; }
    for (int t = 0; t < L; ++t) {
        const uint16_t *xt = x + (size_t)t * d;
        const float *dyt = dy + (size_t)t * d;
        for (int k = 0; k < K; ++k) {
            const int64_t e = idx[(size_t)t * K + k];
            if (e < 0 || e >= rows) return -2;
            const uint16_t *w = W + (size_t)e * d, *v = V + (size_t)e * d;
            const double g = (double)gate[(size_t)t * K + k];
            double h = 0.0, c = 0.0;
            for (int j = 0; j < d; ++j) {
                h += bf16_to_double(xt[j]) * bf16_to_double(w[j]);
                c += (double)dyt[j] * bf16_to_double(v[j]);
            }
            const double a = silu(h);
            dgate[(size_t)t * K + k] = a * c;
            const double dh = g * c * silu_grad(h);
            for (int j = 0; j < d; ++j) {
                dV[(size_t)e * d + j] += g * a * (double)dyt[j];
                dW[(size_t)e * d + j] += dh * bf16_to_double(xt[j]);
                dx[(size_t)t * d + j] += dh * bf16_to_double(w[j]);
            }
        }
    }
    return 0;
}

/* Router part, given dgate:
 *   gates are the softmax over the K selected S:  dS_k = g_k (dgate_k - sum_j g_j dgate_j)
 *   S = p_r[i] + p_c[j], n = i N_c + j:           dp_r[i] += dS_k,  dp_c[j] += dS_k
 *   p = s - logsumexp(s):                          ds = dp - exp(p) * sum(dp)
 *   s_r = x W_r^T:                                 dx_t += sum_i ds_r[i] W_r[i],
 *                                                  dW_r[i] += ds_r[i] x_t   (columns alike)
 * dx is ADDED to (so the expert part can go first); dW_r, dW_c are
 * overwritten.  p_r, p_c are the forward's fp32 log-probabilities.  Dense over
 * the grid axes in fp64, single-threaded.                                  */
int oracle_router_bwd(const uint16_t *x, const uint16_t *W_r, const uint16_t *W_c, int L, int d,
                      int N_r, int N_c, int K, const float *p_r, const float *p_c,
                      const int32_t *idx, const float *gate, const double *dgate, double *dx,
                      double *dW_r, double *dW_c) {
    if (L < 0 || d <= 0 || N_r <= 0 || N_c <= 0 || K <= 0) return -1;
    for (int64_t u = 0; u < (int64_t)N_r * d; ++u) dW_r[u] = 0.0;
    for (int64_t u = 0; u < (int64_t)N_c * d; ++u) dW_c[u] = 0.0;
    double *dp_r = (double *)malloc(sizeof(double) * (size_t)N_r);
    double *dp_c = (double *)malloc(sizeof(double) * (size_t)N_c);
    if (!dp_r || !dp_c) { free(dp_r); free(dp_c); return -3; }
    for (int t = 0; t < L; ++t) {
        double sgd = 0.0;
        for (int k = 0; k < K; ++k) sgd += (double)gate[(size_t)t * K + k] * dgate[(size_t)t * K + k];
        for (int i = 0; i < N_r; ++i) dp_r[i] = 0.0;
        for (int j = 0; j < N_c; ++j) dp_c[j] = 0.0;
        for (int k = 0; k < K; ++k) {
            const int64_t n = idx[(size_t)t * K + k];
            if (n < 0 || n >= (int64_t)N_r * N_c) { free(dp_r); free(dp_c); return -2; }
            const double dS = (double)gate[(size_t)t * K + k] * (dgate[(size_t)t * K + k] - sgd);
            dp_r[n / N_c] += dS;
            dp_c[n % N_c] += dS;
        }
        double sr = 0.0, sc = 0.0;
        for (int i = 0; i < N_r; ++i) sr += dp_r[i];
        for (int j = 0; j < N_c; ++j) sc += dp_c[j];
        const uint16_t *xt = x + (size_t)t * d;
        for (int i = 0; i < N_r; ++i) {
            const double ds = dp_r[i] - exp((double)p_r[(size_t)t * N_r + i]) * sr;
            if (ds == 0.0) continue;
            for (int j = 0; j < d; ++j) {
                dx[(size_t)t * d + j] += ds * bf16_to_double(W_r[(size_t)i * d + j]);
                dW_r[(size_t)i * d + j] += ds * bf16_to_double(xt[j]);
            }
        }
        for (int i = 0; i < N_c; ++i) {
            const double ds = dp_c[i] - exp((double)p_c[(size_t)t * N_c + i]) * sc;
            if (ds == 0.0) continue;
            for (int j = 0; j < d; ++j) {
                dx[(size_t)t * d + j] += ds * bf16_to_double(W_c[(size_t)i * d + j]);
                dW_c[(size_t)i * d + j] += ds * bf16_to_double(xt[j]);
            }
        }
    }
    free(dp_r);
    free(dp_c);
    return 0;
}

/* ---- The shared dense MLP of [R] step 1 / [G] section 2.1 ----------------
 * The pages call it a standard dense MLP and give no form; the reading here is
 * the gated one, SwiGLU being the activation [R] names for the layer:
 *   a_f = x_t . W_g[f],  b_f = x_t . W_u[f]            (f < F)
 *   h_f = SiLU(a_f) * b_f
 *   out[r, c] = sum_f h_f * W_d[c][f]                   (c < d)
 * W_g and W_u are F rows of d, W_d is d rows of F (each the K-major operand of
 * its product).  fp64 over the exact bf16 inputs; row r is token
 * t = tokens[r] (r itself when tokens is NULL).                            */
int oracle_shared_mlp(const uint16_t *x, const uint16_t *W_g, const uint16_t *W_u,
                      const uint16_t *W_d, int d, int F, const int32_t *tokens, int n_tokens,
                      double *out, int nthreads) {
    if (d <= 0 || F <= 0 || n_tokens < 0) return -1;
    set_threads(nthreads);
    #pragma omp parallel
    {
        double *xr = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        #pragma omp for schedule(dynamic, 4)
        for (int r = 0; r < n_tokens; ++r) {
            const int64_t t = tokens ? tokens[r] : r;
            for (int c = 0; c < d; ++c) xr[c] = bf16_to_double(x[(size_t)t * d + c]);
            for (int f = 0; f < F; ++f) {
                double a = 0.0, b = 0.0;
                for (int c = 0; c < d; ++c) {
                    a += xr[c] * bf16_to_double(W_g[(size_t)f * d + c]);
                    b += xr[c] * bf16_to_double(W_u[(size_t)f * d + c]);
                }
                h[f] = silu(a) * b;
            }
            double *o = out + (size_t)r * d;
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int f = 0; f < F; ++f) acc += h[f] * bf16_to_double(W_d[(size_t)c * F + f]);
                o[c] = acc;
            }
        }
        free(xr);
        free(h);
    }
    return 0;
}
