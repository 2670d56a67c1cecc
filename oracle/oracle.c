/*
 * oracle.c -- plain, slow, fp64 CPU exact attention.  TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference legs may load
 * this library.  The CUDA product path never calls it and shares no code with it.
 *
 * What it computes is the plain definition of attention given on the FlashAttention pages
 * (FlashAttention (DE), section "Problematik der Standard-Attention", the one formula
 * Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V; the same formula in the Russian article's
 * section on the problem of standard attention).  The pages state that FlashAttention returns
 * exactly this result (FlashAttention (DE), "Online-Softmax-Berechnung": "exaktes Ergebnis";
 * flash-attention glossary page, "Hoe werkt het?": exact attention), so the oracle is the
 * definition written out, NOT the tiled online algorithm:
 *
 *   J_i   = { j : j < L  and (not causal or j <= i) }       (mask reading: top-left causal,
 *                                                            key padding at j >= L)
 *   s_ij  = scale * sum_k q_ik k_jk                 for j in J_i
 *   m_i   = max_j s_ij,  l_i = sum_j exp(s_ij - m_i),  lse_i = m_i + ln l_i
 *   P_ij  = exp(s_ij - lse_i)                       (two passes over the row)
 *   O_i   = sum_j P_ij v_j
 *
 * The backward pass is the ordinary derivative of that formula (the pages print no gradient;
 * the glossary page's "Herberekening" item only says that training keeps the normalisation
 * values and recomputes the blocks).  With dO the gradient of the loss w.r.t. O:
 *
 *   dP_ij = dO_i . v_j,   D_i = dO_i . O_i,   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij k_j,   dK_j = scale sum_i dS_ij q_i,   dV_j = sum_i P_ij dO_i
 *
 * Entries with j outside J_i have P = dS = 0.  A row with an empty J_i (unreachable when
 * every L >= 1) gets O = 0, lse = -inf and no gradient.
 *
 * Every function works on ONE head: q, k, v, dO are row-major [N][d] fp64 arrays holding the
 * exact values of the bf16 inputs (the caller upcasts, which is exact).  Rows are spread over
 * plain pthreads; no BLAS, no blocking, no reordering beyond the sums written above.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

static int g_threads = 0;

void oracle_set_threads(int n) { g_threads = n; }

int oracle_get_threads(void) {
    if (g_threads > 0) return g_threads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* ---- a tiny parallel-for over [0, n) with a static round-robin split ---- */
typedef void (*row_fn)(void* ctx, int index, double* scratch);

struct pf_job {
    row_fn fn;
    void* ctx;
    int n, stride, first, scratch_len;
};

static void* pf_worker(void* arg) {
    struct pf_job* job = (struct pf_job*)arg;
    double* scratch = (double*)malloc(sizeof(double) * (size_t)(job->scratch_len > 0 ? job->scratch_len : 1));
    if (!scratch) return (void*)1;
    for (int i = job->first; i < job->n; i += job->stride) job->fn(job->ctx, i, scratch);
    free(scratch);
    return NULL;
}

static int parallel_for(int n, row_fn fn, void* ctx, int scratch_len) {
    if (n <= 0) return 0;
    int T = oracle_get_threads();
    if (T > n) T = n;
    pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)T);
    struct pf_job* jobs = (struct pf_job*)malloc(sizeof(struct pf_job) * (size_t)T);
    if (!tid || !jobs) { free(tid); free(jobs); return -1; }
    int err = 0;
    for (int t = 0; t < T; ++t) {
        jobs[t].fn = fn; jobs[t].ctx = ctx; jobs[t].n = n; jobs[t].stride = T;
        jobs[t].first = t; jobs[t].scratch_len = scratch_len;
    }
    int started = 0;   /* threads 1..started are running */
    for (int t = 1; t < T; ++t) {
        if (pthread_create(&tid[t], NULL, pf_worker, &jobs[t]) != 0) break;
        started = t;
    }
    if (pf_worker(&jobs[0]) != NULL) err = -1;
    for (int t = 1; t <= started; ++t) {
        void* r = NULL;
        pthread_join(tid[t], &r);
        if (r != NULL) err = -1;
    }
    /* stripes whose thread could not be started are finished here, serially */
    for (int t = started + 1; t < T; ++t)
        if (pf_worker(&jobs[t]) != NULL) err = -1;
    free(tid); free(jobs);
    return err;
}

/* ---- the definition ---- */
static int key_visible(int i, int j, int L, int causal) {
    return j < L && (!causal || j <= i);
}

static double dot(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int k = 0; k < d; ++k) s += a[k] * b[k];
    return s;
}

struct head {
    const double *q, *k, *v, *dO;
    int N, d, causal, L;
    double scale;
    /* outputs / intermediates */
    double *O, *lse, *D, *dQ, *dK, *dV, *P;
    const int* rows;   /* row list for the *_rows entry points, or NULL */
};

/* Row i: scores over J_i, max, sum of exponentials, lse, then O_i (and D_i if dO given). */
static void fwd_row(struct head* h, int i, double* O_out, double* lse_out, double* D_out, double* s) {
    const int N = h->N, d = h->d;
    const double* qi = h->q + (size_t)i * d;
    double m = -INFINITY;
    int count = 0;
    for (int j = 0; j < N; ++j) {
        if (!key_visible(i, j, h->L, h->causal)) continue;
        s[j] = h->scale * dot(qi, h->k + (size_t)j * d, d);
        if (s[j] > m) m = s[j];
        ++count;
    }
    for (int c = 0; c < d; ++c) O_out[c] = 0.0;
    if (count == 0) {
        *lse_out = -INFINITY;
        if (D_out) *D_out = 0.0;
        return;
    }
    double l = 0.0;
    for (int j = 0; j < N; ++j)
        if (key_visible(i, j, h->L, h->causal)) l += exp(s[j] - m);
    const double lse = m + log(l);
    for (int j = 0; j < N; ++j) {
        if (!key_visible(i, j, h->L, h->causal)) continue;
        const double p = exp(s[j] - lse);
        const double* vj = h->v + (size_t)j * d;
        for (int c = 0; c < d; ++c) O_out[c] += p * vj[c];
    }
    *lse_out = lse;
    if (D_out) *D_out = dot(h->dO + (size_t)i * d, O_out, d);
}

static void fwd_row_task(void* ctx, int i, double* scratch) {
    struct head* h = (struct head*)ctx;
    fwd_row(h, i, h->O + (size_t)i * h->d, h->lse + i, h->D ? h->D + i : NULL, scratch);
}

static void fwd_rows_task(void* ctx, int t, double* scratch) {
    struct head* h = (struct head*)ctx;
    fwd_row(h, h->rows[t], h->O + (size_t)t * h->d, h->lse + t, NULL, scratch);
}

static int check_args(const void* q, const void* k, int N, int d, int L) {
    if (!q || !k || N < 0 || d <= 0 || L < 0 || L > N) return -1;
    return 0;
}

/* O [N][d], lse [N] for one head. Returns 0 on success. */
int oracle_attention_fwd(const double* q, const double* k, const double* v, int N, int d,
                         double scale, int causal, int L, double* O, double* lse) {
    if (check_args(q, k, N, d, L) || !v || !O || !lse) return -1;
    struct head h = {0};
    h.q = q; h.k = k; h.v = v; h.N = N; h.d = d; h.scale = scale; h.causal = causal; h.L = L;
    h.O = O; h.lse = lse;
    return parallel_for(N, fwd_row_task, &h, N);
}

/* Only the listed query rows: O [nrows][d], lse [nrows]. */
int oracle_attention_fwd_rows(const double* q, const double* k, const double* v, int N, int d,
                              double scale, int causal, int L, const int* rows, int nrows,
                              double* O, double* lse) {
    if (check_args(q, k, N, d, L) || !v || !O || !lse || (nrows > 0 && !rows)) return -1;
    for (int t = 0; t < nrows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -1;
    struct head h = {0};
    h.q = q; h.k = k; h.v = v; h.N = N; h.d = d; h.scale = scale; h.causal = causal; h.L = L;
    h.O = O; h.lse = lse; h.rows = rows;
    return parallel_for(nrows, fwd_rows_task, &h, N);
}

/* The full probability matrix P [N][N] (zeros outside J_i), for tiny N only. */
static void probs_task(void* ctx, int i, double* s) {
    struct head* h = (struct head*)ctx;
    const int N = h->N;
    double* Pi = h->P + (size_t)i * N;
    double m = -INFINITY;
    int count = 0;
    for (int j = 0; j < N; ++j) {
        Pi[j] = 0.0;
        if (!key_visible(i, j, h->L, h->causal)) continue;
        s[j] = h->scale * dot(h->q + (size_t)i * h->d, h->k + (size_t)j * h->d, h->d);
        if (s[j] > m) m = s[j];
        ++count;
    }
    if (count == 0) return;
    double l = 0.0;
    for (int j = 0; j < N; ++j)
        if (key_visible(i, j, h->L, h->causal)) l += exp(s[j] - m);
    const double lse = m + log(l);
    for (int j = 0; j < N; ++j)
        if (key_visible(i, j, h->L, h->causal)) Pi[j] = exp(s[j] - lse);
}

int oracle_attention_probs(const double* q, const double* k, int N, int d, double scale,
                           int causal, int L, double* P) {
    if (check_args(q, k, N, d, L) || !P) return -1;
    struct head h = {0};
    h.q = q; h.k = k; h.N = N; h.d = d; h.scale = scale; h.causal = causal; h.L = L; h.P = P;
    return parallel_for(N, probs_task, &h, N);
}

/* dQ_i = scale * sum_j P_ij (dP_ij - D_i) k_j, recomputing P_ij from lse_i. */
static void dq_row(struct head* h, int i, double* dQ_out) {
    const int N = h->N, d = h->d;
    const double* qi = h->q + (size_t)i * d;
    const double* dOi = h->dO + (size_t)i * d;
    for (int c = 0; c < d; ++c) dQ_out[c] = 0.0;
    for (int j = 0; j < N; ++j) {
        if (!key_visible(i, j, h->L, h->causal)) continue;
        const double s = h->scale * dot(qi, h->k + (size_t)j * d, d);
        const double p = exp(s - h->lse[i]);
        const double dp = dot(dOi, h->v + (size_t)j * d, d);
        const double ds = p * (dp - h->D[i]);
        const double* kj = h->k + (size_t)j * d;
        for (int c = 0; c < d; ++c) dQ_out[c] += h->scale * ds * kj[c];
    }
}

/* dK_j = scale * sum_i dS_ij q_i and dV_j = sum_i P_ij dO_i. */
static void dkv_col(struct head* h, int j, double* dK_out, double* dV_out) {
    const int N = h->N, d = h->d;
    const double* kj = h->k + (size_t)j * d;
    const double* vj = h->v + (size_t)j * d;
    for (int c = 0; c < d; ++c) { dK_out[c] = 0.0; dV_out[c] = 0.0; }
    for (int i = 0; i < N; ++i) {
        if (!key_visible(i, j, h->L, h->causal)) continue;
        const double* qi = h->q + (size_t)i * d;
        const double* dOi = h->dO + (size_t)i * d;
        const double s = h->scale * dot(qi, kj, d);
        const double p = exp(s - h->lse[i]);
        const double dp = dot(dOi, vj, d);
        const double ds = p * (dp - h->D[i]);
        for (int c = 0; c < d; ++c) {
            dK_out[c] += h->scale * ds * qi[c];
            dV_out[c] += p * dOi[c];
        }
    }
}

static void dq_task(void* ctx, int i, double* scratch) {
    (void)scratch;
    struct head* h = (struct head*)ctx;
    dq_row(h, i, h->dQ + (size_t)i * h->d);
}

static void dkv_task(void* ctx, int j, double* scratch) {
    (void)scratch;
    struct head* h = (struct head*)ctx;
    dkv_col(h, j, h->dK + (size_t)j * h->d, h->dV + (size_t)j * h->d);
}

static void dq_rows_task(void* ctx, int t, double* scratch) {
    (void)scratch;
    struct head* h = (struct head*)ctx;
    dq_row(h, h->rows[t], h->dQ + (size_t)t * h->d);
}

struct rows_pair { struct head* h; const int* cols; };

static void dkv_rows_task(void* ctx, int t, double* scratch) {
    (void)scratch;
    struct rows_pair* rp = (struct rows_pair*)ctx;
    struct head* h = rp->h;
    dkv_col(h, rp->cols[t], h->dK + (size_t)t * h->d, h->dV + (size_t)t * h->d);
}

/*
 * Full backward for one head.  Also returns the forward O [N][d], lse [N] and D [N] it
 * computed on the way (caller-owned arrays).
 */
int oracle_attention_bwd(const double* q, const double* k, const double* v, const double* dO,
                         int N, int d, double scale, int causal, int L,
                         double* dQ, double* dK, double* dV, double* O, double* lse, double* D) {
    if (check_args(q, k, N, d, L) || !v || !dO || !dQ || !dK || !dV || !O || !lse || !D) return -1;
    struct head h = {0};
    h.q = q; h.k = k; h.v = v; h.dO = dO; h.N = N; h.d = d; h.scale = scale;
    h.causal = causal; h.L = L; h.O = O; h.lse = lse; h.D = D; h.dQ = dQ; h.dK = dK; h.dV = dV;
    if (parallel_for(N, fwd_row_task, &h, N)) return -1;
    if (parallel_for(N, dq_task, &h, 1)) return -1;
    if (parallel_for(N, dkv_task, &h, 1)) return -1;
    return 0;
}

/*
 * Backward restricted to listed outputs: dQ for the query rows `qrows` ([nq][d]) and
 * dK, dV for the key rows `krows` ([nk][d]).  lse and D are still formed for every row
 * because dK_j and dV_j sum over all i.
 */
int oracle_attention_bwd_rows(const double* q, const double* k, const double* v, const double* dO,
                              int N, int d, double scale, int causal, int L,
                              const int* qrows, int nq, const int* krows, int nk,
                              double* dQ, double* dK, double* dV) {
    if (check_args(q, k, N, d, L) || !v || !dO) return -1;
    if ((nq > 0 && (!qrows || !dQ)) || (nk > 0 && (!krows || !dK || !dV))) return -1;
    for (int t = 0; t < nq; ++t) if (qrows[t] < 0 || qrows[t] >= N) return -1;
    for (int t = 0; t < nk; ++t) if (krows[t] < 0 || krows[t] >= N) return -1;
    double* O = (double*)malloc(sizeof(double) * (size_t)N * (size_t)d);
    double* lse = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    double* D = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
    if (!O || !lse || !D) { free(O); free(lse); free(D); return -1; }
    struct head h = {0};
    h.q = q; h.k = k; h.v = v; h.dO = dO; h.N = N; h.d = d; h.scale = scale;
    h.causal = causal; h.L = L; h.O = O; h.lse = lse; h.D = D; h.dQ = dQ; h.dK = dK; h.dV = dV;
    int err = parallel_for(N, fwd_row_task, &h, N);
    if (!err) { h.rows = qrows; err = parallel_for(nq, dq_rows_task, &h, 1); }
    if (!err) {
        struct rows_pair rp = { &h, krows };
        err = parallel_for(nk, dkv_rows_task, &rp, 1);
    }
    free(O); free(lse); free(D);
    return err;
}
