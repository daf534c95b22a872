/*
 * gdn_oracle.c -- CPU oracle for the Gated DeltaNet (gated delta rule) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only the test-suite, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library; both sides only read the same seeded inputs.
 *
 * Everything is plain f64 (long double for the brute-force form), written for
 * a reader to check against the definitions by eye: no blocking, no fusion, no
 * reordering beyond what each definition states.
 *
 * Sources (the three web pages the method is taken from, plus the recurrence
 * they implement):
 *   - "ssm_gdn_tc_route.rs" (metrale_model_layers/layers/ops), module doc and
 *     GDN_TC_SPINE_ENTRY: the prefill "state spine" chunk_delta_h carries an f32
 *     state H across chunks; operands are bf16, the accumulator is the state.
 *   - "ssm_gdn_woa.rs" (metrale_model_layers/layers/ops), gdn_decode_wy4_woa /
 *     gdn_wy4_fold / gdn_wy4_flag_clear: the K=4 write-on-accept verify writes
 *     outputs but no state; the fold applies rows 0..na_tab[b] to H once.
 *   - "ssm_ba_gates_hopper.rs" (spark_model/layers/ops), module doc and
 *     ba_gates_slot: the BA projection (N = 2*nv outputs per token over a K-wide
 *     activation row) and the [gate(nv) | beta(nv)] output row.
 *   - The gated delta rule itself, per (sequence, value head):
 *       S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *       o_t = S_t q_t   (times an explicit `scale`, 1.0 in every workload).
 *
 * Tensor layouts (all dense, row-major, f64):
 *   q, k   [T][H_k][d_k]     v, o [T][H_v][d_v]     g, beta [T][H_v]
 *   h0, hT [num_seqs][H_v][d_k][d_v]  -- the state is stored as H = S^T.
 *   v-head h reads k-head h / (H_v / H_k) (contiguous grouping, as ba_gates_slot
 *   groups v-heads).
 *
 * Parity pins for every function here live in tests/test_oracle.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* A tiny thread pool over independent (sequence, v-head) units.              */
/* ------------------------------------------------------------------------- */

typedef void (*unit_fn)(void* ctx, int unit);

typedef struct {
    unit_fn fn;
    void* ctx;
    int n_units;
    int next;
    pthread_mutex_t lock;
} pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        pthread_mutex_lock(&p->lock);
        int u = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

static void run_units(unit_fn fn, void* ctx, int n_units, int nthreads) {
    if (nthreads <= 1 || n_units <= 1) {
        for (int u = 0; u < n_units; ++u) fn(ctx, u);
        return;
    }
    if (nthreads > n_units) nthreads = n_units;
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n_units = n_units;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, pool_worker, &p);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------------- */
/* Shared problem description                                                 */
/* ------------------------------------------------------------------------- */

typedef struct {
    const double *q, *k, *v, *g, *beta;
    const int* cu_seqlens;
    int num_seqs, H_k, H_v, d_k, d_v;
    double scale;
    const double* h0; /* may be NULL: zero initial state */
    double *o, *hT;   /* hT may be NULL */
    int chunk;        /* chunked form only */
} problem_t;

static const double* q_row(const problem_t* P, int t, int hk) {
    return P->q + ((size_t)t * P->H_k + hk) * P->d_k;
}
static const double* k_row(const problem_t* P, int t, int hk) {
    return P->k + ((size_t)t * P->H_k + hk) * P->d_k;
}
static const double* v_row(const problem_t* P, int t, int h) {
    return P->v + ((size_t)t * P->H_v + h) * P->d_v;
}
static double* o_row(const problem_t* P, int t, int h) {
    return P->o + ((size_t)t * P->H_v + h) * P->d_v;
}

/* Load the unit's initial state H = S_0^T ([d_k][d_v]) or zeros. */
static void load_state(const problem_t* P, int n, int h, double* H) {
    size_t sz = (size_t)P->d_k * P->d_v;
    if (P->h0)
        memcpy(H, P->h0 + ((size_t)n * P->H_v + h) * sz, sz * sizeof(double));
    else
        memset(H, 0, sz * sizeof(double));
}

static void store_state(const problem_t* P, int n, int h, const double* H) {
    if (!P->hT) return;
    size_t sz = (size_t)P->d_k * P->d_v;
    memcpy(P->hT + ((size_t)n * P->H_v + h) * sz, H, sz * sizeof(double));
}

/* ------------------------------------------------------------------------- */
/* (1) Token-by-token recurrence -- the definition.                           */
/*                                                                           */
/* For each token: S' = exp(g_t) S;  delta = beta_t (v_t - S' k_t);          */
/* S = S' + delta k_t^T;  o_t = scale * S q_t   (the output reads the state   */
/* AFTER the token's update).  Held as H = S^T, so (S k)_j = sum_i H[i][j]k_i. */
/* ------------------------------------------------------------------------- */

static void token_steps(const problem_t* P, int h, int t_begin, int t_end, double* H,
                        int write_o) {
    const int dk = P->d_k, dv = P->d_v;
    const int hk = h / (P->H_v / P->H_k);
    double* delta = (double*)malloc(sizeof(double) * (size_t)dv);
    for (int t = t_begin; t < t_end; ++t) {
        const double* kt = k_row(P, t, hk);
        const double* qt = q_row(P, t, hk);
        const double* vt = v_row(P, t, h);
        const double gamma = exp(P->g[(size_t)t * P->H_v + h]);
        const double b = P->beta[(size_t)t * P->H_v + h];
        for (int i = 0; i < dk * dv; ++i) H[i] *= gamma; /* S' = gamma S */
        for (int j = 0; j < dv; ++j) {                   /* delta = b (v - S' k) */
            double pred = 0.0;
            for (int i = 0; i < dk; ++i) pred += H[(size_t)i * dv + j] * kt[i];
            delta[j] = b * (vt[j] - pred);
        }
        for (int i = 0; i < dk; ++i) /* S = S' + delta k^T */
            for (int j = 0; j < dv; ++j) H[(size_t)i * dv + j] += kt[i] * delta[j];
        if (write_o) {
            double* ot = o_row(P, t, h);
            for (int j = 0; j < dv; ++j) { /* o = scale * S q */
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += H[(size_t)i * dv + j] * qt[i];
                ot[j] = P->scale * acc;
            }
        }
    }
    free(delta);
}

static void token_unit(void* ctx, int unit) {
    const problem_t* P = (const problem_t*)ctx;
    const int n = unit / P->H_v, h = unit % P->H_v;
    double* H = (double*)malloc(sizeof(double) * (size_t)P->d_k * P->d_v);
    load_state(P, n, h, H);
    token_steps(P, h, P->cu_seqlens[n], P->cu_seqlens[n + 1], H, 1);
    store_state(P, n, h, H);
    free(H);
}

int oracle_gdn_token(const double* q, const double* k, const double* v, const double* g,
                     const double* beta, const int* cu_seqlens, int num_seqs, int H_k, int H_v,
                     int d_k, int d_v, double scale, const double* h0, double* o, double* hT,
                     int nthreads) {
    if (H_k <= 0 || H_v % H_k != 0) return 1;
    problem_t P = {q, k, v, g, beta, cu_seqlens, num_seqs, H_k, H_v, d_k, d_v, scale, h0, o, hT, 0};
    run_units(token_unit, &P, num_seqs * H_v, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* (2) Chunked form -- the WY/UT chunk-parallel restatement, f64.             */
/*                                                                           */
/* Per chunk of L rows (local index r), with G_r = g_0 + ... + g_r:           */
/*   A[r][s] = beta_r exp(G_r - G_s) (k_r . k_s)        for s < r            */
/*   (I + A) W = diag(beta exp(G)) K,  (I + A) U = diag(beta) V   (forward    */
/*   substitution; I + A is unit lower triangular)                            */
/*   Vn = U - W H                       (the per-row update terms delta_r)    */
/*   O  = scale [diag(exp G) Q H + (Q K^T o Gamma) Vn],                       */
/*        Gamma[r][s] = exp(G_r - G_s) for s <= r, else 0                     */
/*   H <- exp(G_{L-1}) H + sum_r exp(G_{L-1} - G_r) k_r Vn_r^T                */
/* A short final chunk simply has L < chunk rows.                             */
/* ------------------------------------------------------------------------- */

static void chunk_unit(void* ctx, int unit) {
    const problem_t* P = (const problem_t*)ctx;
    const int n = unit / P->H_v, h = unit % P->H_v;
    const int dk = P->d_k, dv = P->d_v, C = P->chunk;
    const int hk = h / (P->H_v / P->H_k);
    double* H = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* G = (double*)malloc(sizeof(double) * (size_t)C);
    double* A = (double*)malloc(sizeof(double) * (size_t)C * C);
    double* W = (double*)malloc(sizeof(double) * (size_t)C * dk);
    double* U = (double*)malloc(sizeof(double) * (size_t)C * dv);
    double* Vn = (double*)malloc(sizeof(double) * (size_t)C * dv);
    double* Hn = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    load_state(P, n, h, H);
    const int t_begin = P->cu_seqlens[n], t_end = P->cu_seqlens[n + 1];
    for (int t0 = t_begin; t0 < t_end; t0 += C) {
        const int L = (t_end - t0 < C) ? (t_end - t0) : C;
        /* gate cumsum */
        double run = 0.0;
        for (int r = 0; r < L; ++r) {
            run += P->g[(size_t)(t0 + r) * P->H_v + h];
            G[r] = run;
        }
        /* strictly lower A */
        for (int r = 0; r < L; ++r) {
            const double br = P->beta[(size_t)(t0 + r) * P->H_v + h];
            for (int s = 0; s < L; ++s) {
                double a = 0.0;
                if (s < r) {
                    const double* kr = k_row(P, t0 + r, hk);
                    const double* ks = k_row(P, t0 + s, hk);
                    double dot = 0.0;
                    for (int i = 0; i < dk; ++i) dot += kr[i] * ks[i];
                    a = br * exp(G[r] - G[s]) * dot;
                }
                A[(size_t)r * C + s] = a;
            }
        }
        /* forward substitution for W and U */
        for (int r = 0; r < L; ++r) {
            const double br = P->beta[(size_t)(t0 + r) * P->H_v + h];
            const double* kr = k_row(P, t0 + r, hk);
            const double* vr = v_row(P, t0 + r, h);
            for (int i = 0; i < dk; ++i) {
                double w = br * exp(G[r]) * kr[i];
                for (int s = 0; s < r; ++s) w -= A[(size_t)r * C + s] * W[(size_t)s * dk + i];
                W[(size_t)r * dk + i] = w;
            }
            for (int j = 0; j < dv; ++j) {
                double u = br * vr[j];
                for (int s = 0; s < r; ++s) u -= A[(size_t)r * C + s] * U[(size_t)s * dv + j];
                U[(size_t)r * dv + j] = u;
            }
        }
        /* Vn = U - W H */
        for (int r = 0; r < L; ++r)
            for (int j = 0; j < dv; ++j) {
                double acc = U[(size_t)r * dv + j];
                for (int i = 0; i < dk; ++i) acc -= W[(size_t)r * dk + i] * H[(size_t)i * dv + j];
                Vn[(size_t)r * dv + j] = acc;
            }
        /* O = scale [diag(e^G) Q H + (Q K^T o Gamma) Vn] */
        for (int r = 0; r < L; ++r) {
            const double* qr = q_row(P, t0 + r, hk);
            double* orow = o_row(P, t0 + r, h);
            for (int j = 0; j < dv; ++j) {
                double inter = 0.0;
                for (int i = 0; i < dk; ++i) inter += qr[i] * H[(size_t)i * dv + j];
                double intra = 0.0;
                for (int s = 0; s <= r; ++s) {
                    const double* ks = k_row(P, t0 + s, hk);
                    double qk = 0.0;
                    for (int i = 0; i < dk; ++i) qk += qr[i] * ks[i];
                    intra += qk * exp(G[r] - G[s]) * Vn[(size_t)s * dv + j];
                }
                orow[j] = P->scale * (exp(G[r]) * inter + intra);
            }
        }
        /* H <- e^{G_last} H + sum_r e^{G_last - G_r} k_r Vn_r^T */
        const double Gl = G[L - 1];
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) {
                double acc = exp(Gl) * H[(size_t)i * dv + j];
                for (int r = 0; r < L; ++r)
                    acc += exp(Gl - G[r]) * k_row(P, t0 + r, hk)[i] * Vn[(size_t)r * dv + j];
                Hn[(size_t)i * dv + j] = acc;
            }
        memcpy(H, Hn, sizeof(double) * (size_t)dk * dv);
    }
    store_state(P, n, h, H);
    free(H); free(G); free(A); free(W); free(U); free(Vn); free(Hn);
}

int oracle_gdn_chunked(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, const int* cu_seqlens, int num_seqs, int H_k, int H_v,
                       int d_k, int d_v, double scale, const double* h0, double* o, double* hT,
                       int chunk, int nthreads) {
    if (H_k <= 0 || H_v % H_k != 0 || chunk <= 0) return 1;
    problem_t P = {q, k, v, g, beta, cu_seqlens, num_seqs, H_k, H_v, d_k, d_v, scale, h0, o, hT, chunk};
    run_units(chunk_unit, &P, num_seqs * H_v, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* (3) Brute force for short sequences (long double, dense matrices).         */
/*                                                                           */
/* With the d_k x d_k transition M_t = exp(g_t) (I - beta_t k_t k_t^T):       */
/*   S_t = S_0 M_1 ... M_t + sum_{s<=t} beta_s v_s k_s^T M_{s+1} ... M_t      */
/*   o_t = scale S_t q_t                                                      */
/* Every S_t is rebuilt from scratch by explicit matrix products; the rank-1  */
/* update form of (1) is never used.  Intended for T <= 8 and small d.        */
/* ------------------------------------------------------------------------- */

typedef long double ld;

static void mat_mul_ld(const ld* X, const ld* Y, ld* Z, int a, int b, int c) {
    /* Z[a][c] = X[a][b] Y[b][c] */
    for (int i = 0; i < a; ++i)
        for (int j = 0; j < c; ++j) {
            ld acc = 0.0L;
            for (int l = 0; l < b; ++l) acc += X[(size_t)i * b + l] * Y[(size_t)l * c + j];
            Z[(size_t)i * c + j] = acc;
        }
}

static void brute_unit(void* ctx, int unit) {
    const problem_t* P = (const problem_t*)ctx;
    const int n = unit / P->H_v, h = unit % P->H_v;
    const int dk = P->d_k, dv = P->d_v;
    const int hk = h / (P->H_v / P->H_k);
    const int t_begin = P->cu_seqlens[n], t_end = P->cu_seqlens[n + 1];
    const int T = t_end - t_begin;
    ld* M = (ld*)malloc(sizeof(ld) * (size_t)(T > 0 ? T : 1) * dk * dk); /* M_1..M_T */
    ld* S0 = (ld*)malloc(sizeof(ld) * (size_t)dv * dk);                  /* S_0 = H0^T */
    ld* S = (ld*)malloc(sizeof(ld) * (size_t)dv * dk);
    ld* X = (ld*)malloc(sizeof(ld) * (size_t)dv * dk);
    ld* Y = (ld*)malloc(sizeof(ld) * (size_t)dv * dk);
    for (int a = 0; a < dv; ++a)
        for (int b = 0; b < dk; ++b)
            S0[(size_t)a * dk + b] =
                P->h0 ? (ld)P->h0[((size_t)n * P->H_v + h) * dk * dv + (size_t)b * dv + a] : 0.0L;
    for (int t = 0; t < T; ++t) {
        const double* kt = k_row(P, t_begin + t, hk);
        const ld gamma = expl((ld)P->g[(size_t)(t_begin + t) * P->H_v + h]);
        const ld b = (ld)P->beta[(size_t)(t_begin + t) * P->H_v + h];
        ld* Mt = M + (size_t)t * dk * dk;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dk; ++j)
                Mt[(size_t)i * dk + j] = gamma * ((i == j ? 1.0L : 0.0L) - b * (ld)kt[i] * (ld)kt[j]);
    }
    for (int t = 0; t < T; ++t) { /* state after token t (0-based) */
        /* S = S_0 M_0 ... M_t */
        memcpy(X, S0, sizeof(ld) * (size_t)dv * dk);
        for (int u = 0; u <= t; ++u) {
            mat_mul_ld(X, M + (size_t)u * dk * dk, Y, dv, dk, dk);
            memcpy(X, Y, sizeof(ld) * (size_t)dv * dk);
        }
        memcpy(S, X, sizeof(ld) * (size_t)dv * dk);
        /* + sum_s beta_s v_s k_s^T M_{s+1} ... M_t */
        for (int s = 0; s <= t; ++s) {
            const double* ks = k_row(P, t_begin + s, hk);
            const double* vs = v_row(P, t_begin + s, h);
            const ld bs = (ld)P->beta[(size_t)(t_begin + s) * P->H_v + h];
            for (int a = 0; a < dv; ++a)
                for (int c = 0; c < dk; ++c) X[(size_t)a * dk + c] = bs * (ld)vs[a] * (ld)ks[c];
            for (int u = s + 1; u <= t; ++u) {
                mat_mul_ld(X, M + (size_t)u * dk * dk, Y, dv, dk, dk);
                memcpy(X, Y, sizeof(ld) * (size_t)dv * dk);
            }
            for (int i = 0; i < dv * dk; ++i) S[i] += X[i];
        }
        const double* qt = q_row(P, t_begin + t, hk);
        double* ot = o_row(P, t_begin + t, h);
        for (int a = 0; a < dv; ++a) {
            ld acc = 0.0L;
            for (int c = 0; c < dk; ++c) acc += S[(size_t)a * dk + c] * (ld)qt[c];
            ot[a] = (double)((ld)P->scale * acc);
        }
    }
    if (P->hT) {
        const ld* Sfin = (T > 0) ? S : S0;
        for (int a = 0; a < dv; ++a)
            for (int b = 0; b < dk; ++b)
                P->hT[((size_t)n * P->H_v + h) * dk * dv + (size_t)b * dv + a] =
                    (double)Sfin[(size_t)a * dk + b];
    }
    free(M); free(S0); free(S); free(X); free(Y);
}

int oracle_gdn_brute(const double* q, const double* k, const double* v, const double* g,
                     const double* beta, const int* cu_seqlens, int num_seqs, int H_k, int H_v,
                     int d_k, int d_v, double scale, const double* h0, double* o, double* hT) {
    if (H_k <= 0 || H_v % H_k != 0) return 1;
    problem_t P = {q, k, v, g, beta, cu_seqlens, num_seqs, H_k, H_v, d_k, d_v, scale, h0, o, hT, 0};
    run_units(brute_unit, &P, num_seqs * H_v, 1);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* (4) K-row speculative verify and the post-verdict fold.                    */
/*                                                                           */
/* "ssm_gdn_woa.rs", gdn_decode_wy4_woa: for each sequence b (rows b*K ..     */
/* b*K+K-1) the verify produces the K outputs of the recurrence started from  */
/* that sequence's state H0_b, and leaves every state untouched.              */
/* gdn_wy4_fold: the fold then replaces H0_b by the state after the first     */
/* na_b rows (na_b = 0: unchanged).  A sequence with present[b] == 0 is       */
/* padding: its output rows are zero and its state is not touched.            */
/* h_states is the per-sequence state gathered densely [batch][H_v][d_k][d_v]; */
/* h_out receives the folded states in the same layout.                       */
/* ------------------------------------------------------------------------- */

typedef struct {
    problem_t P;
    const int* na;
    const int* present;
    int K;
    double* h_out;
} verify_t;

static void verify_unit(void* ctx, int unit) {
    const verify_t* V = (const verify_t*)ctx;
    const problem_t* P = &V->P;
    const int b = unit / P->H_v, h = unit % P->H_v;
    const size_t sz = (size_t)P->d_k * P->d_v;
    const double* H0 = P->h0 + ((size_t)b * P->H_v + h) * sz;
    double* Hout = V->h_out + ((size_t)b * P->H_v + h) * sz;
    if (!V->present[b]) {
        for (int r = 0; r < V->K; ++r) memset(o_row(P, b * V->K + r, h), 0, sizeof(double) * P->d_v);
        memcpy(Hout, H0, sz * sizeof(double));
        return;
    }
    double* H = (double*)malloc(sizeof(double) * sz);
    /* verify: K outputs from H0; the working copy is discarded */
    memcpy(H, H0, sz * sizeof(double));
    token_steps(P, h, b * V->K, b * V->K + V->K, H, 1);
    /* fold: the state after the first na rows */
    memcpy(H, H0, sz * sizeof(double));
    int na = V->na[b];
    if (na > 0 && na <= V->K) {
        /* token_steps with write_o = 0 so the verify outputs stay as they are */
        token_steps(P, h, b * V->K, b * V->K + na, H, 0);
    }
    memcpy(Hout, H, sz * sizeof(double));
    free(H);
}

int oracle_gdn_verify_fold(const double* h_states, const double* q, const double* k,
                           const double* v, const double* g, const double* beta, const int* na,
                           const int* present, int batch, int K, int H_k, int H_v, int d_k,
                           int d_v, double scale, double* o, double* h_out, int nthreads) {
    if (H_k <= 0 || H_v % H_k != 0 || K <= 0) return 1;
    verify_t V;
    problem_t P = {q, k, v, g, beta, NULL, batch, H_k, H_v, d_k, d_v, scale, h_states, o, NULL, 0};
    V.P = P;
    V.na = na;
    V.present = present;
    V.K = K;
    V.h_out = h_out;
    run_units(verify_unit, &V, batch * H_v, nthreads);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* (5) BA gates ("ssm_ba_gates_hopper.rs", module doc and ba_gates_slot).     */
/*                                                                           */
/* ba[m][n] = sum_k x[m][k] w[n][k]  (N = 2*nv outputs per token)             */
/* Output n of group grp = n / (2 vpg), within = n % (2 vpg):                 */
/*   within <  vpg : beta[grp*vpg + within]       = sigmoid(ba)               */
/*   within >= vpg : gate[grp*vpg + within - vpg] =                           */
/*                   -exp(A_log[vh]) * softplus(ba + dt_bias[vh])             */
/* and the token's output row is [gate(0..nv) | beta(0..nv)].                 */
/* softplus(x) = max(x, 0) + log1p(exp(-|x|)),  sigmoid(x) = 1/(1 + e^-x).    */
/* ------------------------------------------------------------------------- */

typedef struct {
    const double *x, *w, *a_log, *dt_bias;
    double* out;
    int M, N, K, nv, vpg;
} ba_t;

static void ba_unit(void* ctx, int m) {
    const ba_t* B = (const ba_t*)ctx;
    const double* xm = B->x + (size_t)m * B->K;
    double* row = B->out + (size_t)m * 2 * B->nv;
    for (int n = 0; n < B->N; ++n) {
        const double* wn = B->w + (size_t)n * B->K;
        double ba = 0.0;
        for (int kk = 0; kk < B->K; ++kk) ba += xm[kk] * wn[kk];
        const int within = n % (2 * B->vpg), grp = n / (2 * B->vpg);
        if (within < B->vpg) {
            const int vh = grp * B->vpg + within;
            row[B->nv + vh] = 1.0 / (1.0 + exp(-ba));
        } else {
            const int vh = grp * B->vpg + (within - B->vpg);
            const double z = ba + B->dt_bias[vh];
            const double softplus = (z > 0.0 ? z : 0.0) + log1p(exp(-fabs(z)));
            row[vh] = -exp(B->a_log[vh]) * softplus;
        }
    }
}

int oracle_ba_gates(const double* x, const double* w, const double* a_log, const double* dt_bias,
                    double* out, int M, int N, int K, int nv, int vpg, int nthreads) {
    if (N != 2 * nv || vpg <= 0 || nv % vpg != 0) return 1;
    ba_t B = {x, w, a_log, dt_bias, out, M, N, K, nv, vpg};
    run_units(ba_unit, &B, M, nthreads);
    return 0;
}
