/*
 * CPU fp64 oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, the package smoke check and the CPU-baseline leg of bench.py
 * may load this library. The CUDA product path never calls it and shares no
 * code, header or helper with it.
 *
 * Source of the arithmetic ("Gated Delta Networks: Improving Mamba2 with
 * Delta Rule", as described on the pages collected for this project):
 *   - recurrence   S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T
 *                  (phantomic12 "gated-deltanet" page, mechanism paragraph;
 *                   dmarx anthology LIT-137, "Standing in the anthology")
 *   - readout      o_t = S_t q_t, read from the state AFTER the gated write
 *                  (portpowered "Gated DeltaNet" page, "How It Works" and
 *                   "Math Or Compute Schema")
 *   - state shape  fixed per head (head_k_dim x head_v_dim), constant in T
 *                  (phantomic12 page, mechanism paragraph)
 *
 * S is d_v x d_k in the formula (S k is a d_v vector). Expanding the product
 * gives S_t = alpha S_{t-1} + beta (v - alpha S_{t-1} k) k^T, which is what the
 * loop below evaluates (one matrix-vector product, one rank-1 update). Every
 * value is fp64; inputs are upcast exactly by the caller; nothing is rounded
 * on the way out.
 *
 * Memory layouts (row-major, same as the library's C ABI):
 *   q, k [B, T, H, d_k]; v, o [B, T, H, d_v]; g, beta [B, T, H];
 *   states [N, H, d_k, d_v] with state[n][h][j][i] = S_{i j}.
 * g is log(alpha); alpha = exp(g). With cu_seqlens (B == 1) sequence n covers
 * tokens [cu[n], cu[n+1]) and starts from its own initial state.
 *
 * Channel-wise gate (the Kimi Delta Attention variant, named as this
 * recurrence's successor on the dmarx anthology LIT-137 page, "Standing in the
 * anthology", and on SOTA-135, "Sequence": the scalar decay becomes one decay
 * per d_k channel). alpha_t is then a d_k vector and diag(alpha_t) stands
 * where the scalar stood:
 *     S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 * so, with R = S_{t-1} diag(alpha_t) (column j of S scaled by alpha_tj),
 * S_t = R + beta_t (v_t - R k_t) k_t^T and o_t = S_t q_t. The gate input is
 * g = log(alpha) of shape [B, T, H, d_k] (gdn_oracle_kda_*).
 *
 * Gradients (gdn_oracle_chunk_bwd). The pages call the chunkwise algorithm a
 * training algorithm (phantomic12 page, mechanism paragraph) but give no
 * gradients. For a loss with dL/do_t = do_t and dL/dS_final = dS_N they
 * follow by reverse-mode differentiation of the scalar-gate recurrence above.
 * With G = dL/dS_t (all later tokens' contributions already in),
 * x = S_{t-1} k, u = beta (v - alpha x), going backwards over t:
 *     G += do_t q_t^T                         (o_t = S_t q_t)
 *     dq_t = S_t^T do_t
 *     Gk = G k;   dv_t = beta Gk;   dbeta_t = Gk . (v - alpha x)
 *     dalpha_t = <G, S_{t-1}> - beta (Gk . x);   dg_t = alpha dalpha_t
 *     dk_t = G^T u - alpha beta S_{t-1}^T Gk
 *     G <- alpha (G - beta Gk k^T)            (= dL/dS_{t-1})
 * and dS_0 = G at the sequence start. S_{t-1} is recomputed forward from
 * states kept every 64 tokens.
 *
 * Parity: pinned by tests/test_oracle_pins.py, tests/test_oracle_kda_pins.py
 * and tests/test_oracle_bwd_pins.py
 * (closed forms, special cases, exact rational arithmetic, hand-worked
 * tokens, the dense chunked WY/UT forms).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *s0;
    const int32_t *cu;
    double *o, *s_out;
    int B, T, H, dk, dv, N;
    int channel_gate;      /* 0: g [B,T,H] scalar gate; 1: g [B,T,H,d_k] per channel */
    /* backward only (o, s_out unused): upstream gradients and the outputs */
    const double *d_o, *d_sN;
    double *dq, *dk_, *dv_, *dg, *dbeta, *ds0;
    int next;              /* next (seq, head) unit to hand out */
    pthread_mutex_t lock;
} job_t;

/* Tokens [t0, t1) of row block b (b = batch index, or 0 for packed sequences)
 * that sequence n covers. */
static void seq_span(const job_t *J, int n, int *b, int *t0, int *t1)
{
    if (J->cu) { *b = 0; *t0 = J->cu[n]; *t1 = J->cu[n + 1]; }
    else       { *b = n; *t0 = 0;        *t1 = J->T; }
}

/* S (formula orientation, S[i*dk + j] = S_ij) from the S^T memory layout. */
static void load_state(const job_t *J, int n, int h, double *S)
{
    const int dk = J->dk, dv = J->dv;
    if (J->s0) {
        const double *st = J->s0 + ((size_t)n * J->H + h) * dk * dv;
        for (int j = 0; j < dk; ++j)
            for (int i = 0; i < dv; ++i) S[(size_t)i * dk + j] = st[(size_t)j * dv + i];
    }
}

static void store_state(const job_t *J, int n, int h, const double *S)
{
    const int dk = J->dk, dv = J->dv;
    if (J->s_out) {
        double *st = J->s_out + ((size_t)n * J->H + h) * dk * dv;
        for (int j = 0; j < dk; ++j)
            for (int i = 0; i < dv; ++i) st[(size_t)j * dv + i] = S[(size_t)i * dk + j];
    }
}

/* One (sequence, head) recurrence with the scalar gate. */
static void run_unit(job_t *J, int n, int h)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    int b, t0, t1;
    seq_span(J, n, &b, &t0, &t1);

    double *S = (double *)calloc((size_t)dv * dk, sizeof(double)); /* S[i*dk + j] */
    double *x = (double *)malloc(sizeof(double) * dv);
    load_state(J, n, h, S);
    for (int t = t0; t < t1; ++t) {
        const size_t row = ((size_t)b * J->T + t) * H + h;
        const double *kt = J->k + row * dk, *qt = J->q + row * dk, *vt = J->v + row * dv;
        const double alpha = exp(J->g[row]);
        const double beta = J->beta[row];
        /* x = S_{t-1} k_t */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
            x[i] = acc;
        }
        /* S_t = alpha S_{t-1} + beta (v_t - alpha x) k_t^T */
        for (int i = 0; i < dv; ++i) {
            const double u = beta * (vt[i] - alpha * x[i]);
            for (int j = 0; j < dk; ++j)
                S[(size_t)i * dk + j] = alpha * S[(size_t)i * dk + j] + u * kt[j];
        }
        /* o_t = S_t q_t (after the write) */
        double *ot = J->o + row * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
            ot[i] = acc;
        }
    }
    store_state(J, n, h, S);
    free(S);
    free(x);
}

/* One (sequence, head) recurrence with the channel-wise gate (see the header):
 * R = S_{t-1} diag(alpha_t); S_t = R + beta_t (v_t - R k_t) k_t^T; o_t = S_t q_t. */
static void run_unit_kda(job_t *J, int n, int h)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    int b, t0, t1;
    seq_span(J, n, &b, &t0, &t1);

    double *S = (double *)calloc((size_t)dv * dk, sizeof(double)); /* S[i*dk + j] */
    double *x = (double *)malloc(sizeof(double) * dv);
    double *a = (double *)malloc(sizeof(double) * dk);
    load_state(J, n, h, S);
    for (int t = t0; t < t1; ++t) {
        const size_t row = ((size_t)b * J->T + t) * H + h;
        const double *kt = J->k + row * dk, *qt = J->q + row * dk, *vt = J->v + row * dv;
        const double *gt = J->g + row * dk;
        const double beta = J->beta[row];
        for (int j = 0; j < dk; ++j) a[j] = exp(gt[j]);
        /* x = R k_t = S_{t-1} diag(alpha_t) k_t */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * a[j] * kt[j];
            x[i] = acc;
        }
        /* S_t = R + beta (v_t - x) k_t^T */
        for (int i = 0; i < dv; ++i) {
            const double ui = beta * (vt[i] - x[i]);
            for (int j = 0; j < dk; ++j)
                S[(size_t)i * dk + j] = a[j] * S[(size_t)i * dk + j] + ui * kt[j];
        }
        /* o_t = S_t q_t (after the write) */
        double *ot = J->o + row * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
            ot[i] = acc;
        }
    }
    store_state(J, n, h, S);
    free(S);
    free(x);
    free(a);
}

/* One scalar-gate step in place: S <- alpha S + beta (v - alpha S k) k^T;
 * x (d_v) receives S_{t-1} k. */
static void step_forward(int dk, int dv, double *S, double *x, const double *kt,
                         const double *vt, double alpha, double beta)
{
    for (int i = 0; i < dv; ++i) {
        double acc = 0.0;
        for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
        x[i] = acc;
    }
    for (int i = 0; i < dv; ++i) {
        const double ui = beta * (vt[i] - alpha * x[i]);
        for (int j = 0; j < dk; ++j)
            S[(size_t)i * dk + j] = alpha * S[(size_t)i * dk + j] + ui * kt[j];
    }
}

#define BWD_CKPT 64   /* tokens between kept states in the backward pass */

/* Gradients of one (sequence, head) recurrence (see the header). */
static void run_unit_bwd(job_t *J, int n, int h)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const size_t SS = (size_t)dv * dk;
    int b, t0, t1;
    seq_span(J, n, &b, &t0, &t1);
    const int L = t1 - t0;
    const int nck = (L + BWD_CKPT - 1) / BWD_CKPT;

    /* states at the start of every BWD_CKPT-token block */
    double *ck = (double *)calloc((size_t)(nck > 0 ? nck : 1) * SS, sizeof(double));
    double *S = (double *)calloc(SS, sizeof(double));
    double *blk = (double *)malloc(sizeof(double) * BWD_CKPT * SS);  /* S_{t-1} of one block */
    double *G = (double *)calloc(SS, sizeof(double));
    double *x = (double *)malloc(sizeof(double) * dv);
    double *u = (double *)malloc(sizeof(double) * dv);
    double *Gk = (double *)malloc(sizeof(double) * dv);
    load_state(J, n, h, S);
    for (int c = 0; c < nck; ++c) {
        memcpy(ck + (size_t)c * SS, S, sizeof(double) * SS);
        const int ta = t0 + c * BWD_CKPT, tb = ta + BWD_CKPT < t1 ? ta + BWD_CKPT : t1;
        for (int t = ta; t < tb; ++t) {
            const size_t row = ((size_t)b * J->T + t) * H + h;
            step_forward(dk, dv, S, x, J->k + row * dk, J->v + row * dv, exp(J->g[row]),
                         J->beta[row]);
        }
    }
    /* G = dL/dS_final, formula orientation */
    if (J->d_sN) {
        const double *st = J->d_sN + ((size_t)n * H + h) * SS;
        for (int j = 0; j < dk; ++j)
            for (int i = 0; i < dv; ++i) G[(size_t)i * dk + j] = st[(size_t)j * dv + i];
    }
    for (int c = nck - 1; c >= 0; --c) {
        const int ta = t0 + c * BWD_CKPT, tb = ta + BWD_CKPT < t1 ? ta + BWD_CKPT : t1;
        /* recompute S_{t-1} for every token of the block */
        memcpy(S, ck + (size_t)c * SS, sizeof(double) * SS);
        for (int t = ta; t < tb; ++t) {
            const size_t row = ((size_t)b * J->T + t) * H + h;
            memcpy(blk + (size_t)(t - ta) * SS, S, sizeof(double) * SS);
            step_forward(dk, dv, S, x, J->k + row * dk, J->v + row * dv, exp(J->g[row]),
                         J->beta[row]);
        }
        for (int t = tb - 1; t >= ta; --t) {
            const size_t row = ((size_t)b * J->T + t) * H + h;
            const double *kt = J->k + row * dk, *qt = J->q + row * dk, *vt = J->v + row * dv;
            const double *dot = J->d_o + row * dv;
            const double alpha = exp(J->g[row]), beta = J->beta[row];
            const double *Sp = blk + (size_t)(t - ta) * SS;      /* S_{t-1} */
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += Sp[(size_t)i * dk + j] * kt[j];
                x[i] = acc;
                u[i] = beta * (vt[i] - alpha * acc);
            }
            /* G += do_t q_t^T */
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j) G[(size_t)i * dk + j] += dot[i] * qt[j];
            /* dq_t = S_t^T do_t with S_t = alpha S_{t-1} + u k^T */
            for (int j = 0; j < dk; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dv; ++i)
                    acc += (alpha * Sp[(size_t)i * dk + j] + u[i] * kt[j]) * dot[i];
                J->dq[row * dk + j] = acc;
            }
            double gx = 0.0, db = 0.0, gs = 0.0;
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += G[(size_t)i * dk + j] * kt[j];
                Gk[i] = acc;
                J->dv_[row * dv + i] = beta * acc;
                db += acc * (vt[i] - alpha * x[i]);
                gx += acc * x[i];
            }
            for (size_t e = 0; e < SS; ++e) gs += G[e] * Sp[e];
            J->dbeta[row] = db;
            J->dg[row] = alpha * (gs - beta * gx);
            for (int j = 0; j < dk; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dv; ++i)
                    acc += G[(size_t)i * dk + j] * u[i] - alpha * beta * Sp[(size_t)i * dk + j] * Gk[i];
                J->dk_[row * dk + j] = acc;
            }
            /* G <- dL/dS_{t-1} */
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    G[(size_t)i * dk + j] = alpha * (G[(size_t)i * dk + j] - beta * Gk[i] * kt[j]);
        }
    }
    {
        double *st = J->ds0 + ((size_t)n * H + h) * SS;
        for (int j = 0; j < dk; ++j)
            for (int i = 0; i < dv; ++i) st[(size_t)j * dv + i] = G[(size_t)i * dk + j];
    }
    free(ck); free(S); free(blk); free(G); free(x); free(u); free(Gk);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (u >= J->N * J->H) break;
        if (J->d_o)               run_unit_bwd(J, u / J->H, u % J->H);
        else if (J->channel_gate) run_unit_kda(J, u / J->H, u % J->H);
        else                      run_unit(J, u / J->H, u % J->H);
    }
    return NULL;
}

static int run_jobs(job_t *J, int nthreads)
{
    pthread_mutex_init(&J->lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J->N * J->H) nthreads = J->N * J->H;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return 0;
}

static int run_all(const double *q, const double *k, const double *v,
                   const double *g, const double *beta,
                   const double *initial_state, const int32_t *cu_seqlens,
                   int B, int T, int H, int d_k, int d_v, int num_seqs,
                   double *o, double *final_state, int nthreads, int channel_gate)
{
    if (!q || !k || !v || !g || !beta || !o) return -1;
    if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1) return -1;
    int N = B;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -1;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
        N = num_seqs;
    }
    job_t J = {q, k, v, g, beta, initial_state, cu_seqlens, o, final_state,
               B, T, H, d_k, d_v, N, channel_gate, NULL, NULL,
               NULL, NULL, NULL, NULL, NULL, NULL, 0};
    return run_jobs(&J, nthreads);
}

/* Gradients of gdn_oracle_chunk_fwd (scalar gate) for the loss
 * L = sum(d_o * o) + sum(d_final_state * final_state). d_o [B,T,H,d_v];
 * d_final_state [N,H,d_k,d_v] or NULL (zero). Outputs: dq, dk [B,T,H,d_k],
 * dv [B,T,H,d_v], dg, dbeta [B,T,H], d_initial_state [N,H,d_k,d_v] (all
 * required). Returns 0, or -1 on bad arguments. */
int gdn_oracle_chunk_bwd(const double *q, const double *k, const double *v,
                         const double *g, const double *beta,
                         const double *initial_state, const int32_t *cu_seqlens,
                         int B, int T, int H, int d_k, int d_v, int num_seqs,
                         const double *d_o, const double *d_final_state,
                         double *dq, double *dk, double *dv, double *dg, double *dbeta,
                         double *d_initial_state, int nthreads)
{
    if (!q || !k || !v || !g || !beta || !d_o) return -1;
    if (!dq || !dk || !dv || !dg || !dbeta || !d_initial_state) return -1;
    if (B < 1 || T < 0 || H < 1 || d_k < 1 || d_v < 1) return -1;
    int N = B;
    if (cu_seqlens) {
        if (B != 1 || num_seqs < 1 || cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -1;
        for (int n = 0; n < num_seqs; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
        N = num_seqs;
    }
    job_t J = {q, k, v, g, beta, initial_state, cu_seqlens, NULL, NULL,
               B, T, H, d_k, d_v, N, 0, d_o, d_final_state,
               dq, dk, dv, dg, dbeta, d_initial_state, 0};
    return run_jobs(&J, nthreads);
}

/* Returns 0 on success, -1 on bad arguments. `o` must hold B*T*H*d_v values;
 * `final_state` (nullable) N*H*d_k*d_v; `initial_state` nullable (zeros). */
int gdn_oracle_chunk_fwd(const double *q, const double *k, const double *v,
                         const double *g, const double *beta,
                         const double *initial_state, const int32_t *cu_seqlens,
                         int B, int T, int H, int d_k, int d_v, int num_seqs,
                         double *o, double *final_state, int nthreads)
{
    return run_all(q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k, d_v,
                   num_seqs, o, final_state, nthreads, 0);
}

/* Channel-wise gate: same contract, g = log(alpha) is [B, T, H, d_k]. */
int gdn_oracle_kda_chunk_fwd(const double *q, const double *k, const double *v,
                             const double *g, const double *beta,
                             const double *initial_state, const int32_t *cu_seqlens,
                             int B, int T, int H, int d_k, int d_v, int num_seqs,
                             double *o, double *final_state, int nthreads)
{
    return run_all(q, k, v, g, beta, initial_state, cu_seqlens, B, T, H, d_k, d_v,
                   num_seqs, o, final_state, nthreads, 1);
}

static int decode_all(const double *q, const double *k, const double *v,
                      const double *g, const double *beta, double *state,
                      double *o, int N, int H, int d_k, int d_v, int nthreads,
                      int channel_gate)
{
    if (!q || !k || !v || !g || !beta || !state || !o) return -1;
    if (N < 1 || H < 1 || d_k < 1 || d_v < 1) return -1;
    /* A decode step is a length-1 sequence per (n, h) with its own state. */
    int32_t *cu = (int32_t *)malloc(sizeof(int32_t) * (N + 1));
    for (int n = 0; n <= N; ++n) cu[n] = n;
    double *s_out = (double *)malloc(sizeof(double) * (size_t)N * H * d_k * d_v);
    /* Tokens laid out as [1, N, H, d]: token index = n. */
    int rc = run_all(q, k, v, g, beta, state, cu, 1, N, H, d_k, d_v, N,
                     o, s_out, nthreads, channel_gate);
    if (rc == 0) memcpy(state, s_out, sizeof(double) * (size_t)N * H * d_k * d_v);
    free(s_out);
    free(cu);
    return rc;
}

/* One recurrent step for N*H independent states, in place:
 * state [N,H,d_k,d_v] (S^T storage), q/k [N,H,d_k], v/o [N,H,d_v], g/beta [N,H].
 * Same arithmetic as one iteration of the scalar-gate loop. */
int gdn_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *g, const double *beta, double *state,
                           double *o, int N, int H, int d_k, int d_v, int nthreads)
{
    return decode_all(q, k, v, g, beta, state, o, N, H, d_k, d_v, nthreads, 0);
}

/* Channel-wise gate: g is [N, H, d_k]. */
int gdn_oracle_kda_decode_step(const double *q, const double *k, const double *v,
                               const double *g, const double *beta, double *state,
                               double *o, int N, int H, int d_k, int d_v, int nthreads)
{
    return decode_all(q, k, v, g, beta, state, o, N, H, d_k, d_v, nthreads, 1);
}
