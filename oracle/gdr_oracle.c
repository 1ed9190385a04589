/*
 * gdr_oracle.c -- fp64 sequential reference of the gated delta rule forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library and its
 * Python binding) may link, import or call this file; only the test-suite, the
 * smoke check and the benchmark's CPU-baseline leg do.  It shares no code, header
 * or constant with the CUDA implementation.
 *
 * What it computes (the definition, read in the order the source states it):
 *   "GatedDeltaRule.ixx File Reference" (Mila), Detailed Description:
 *     per value head a state S[dk][dv];  each step
 *        S <- S * exp(g_t)
 *        delta <- (v_t - k_t^T S) * beta_t
 *        S <- S + k_t (outer) delta
 *        o_t <- q_t^T S                     (the state after the update)
 *     q and k L2-normalised over dk, q additionally scaled by 1/sqrt(dk);
 *     beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias).
 *   tessera PR #77 "Track L -- genuine gated delta rule + Mamba2 SSM", summary
 *     "The core finding (L0)": the erase term (I - beta k k^T) is what separates
 *     the rule from gated linear attention; erase = 0 below gives the latter
 *     (S <- alpha S + beta k v^T).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - L2 norm epsilon: x / sqrt(sum x^2 + 1e-6).
 *   - Grouped heads: value head h reads key/query head h / (Hv / Hk).
 *   - Varlen: every sequence starts from its own initial state (zeros if none).
 *
 * Everything is double precision; inputs arrive as float (bf16 and fp32 inputs
 * widen to float and then to double exactly).  Work is split over (sequence,
 * value head) units with plain pthreads; each unit is an independent loop over
 * time.  There is no chunking, blocking or algebraic regrouping here.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_NORM_EPS 1e-6

/* softplus(x) = log(1 + exp(x)), written in the overflow-free form. */
static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Gating of one token of one value head ("GatedDeltaRule.ixx", Detailed Description:
 * beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias)). */
void oracle_gating(double a, double b, double A_log, double dt_bias, double* g, double* beta) {
#ifdef ORACLE_MUTATE_GATE_SIGN
    *g = exp(A_log) * softplus(a + dt_bias);
#else
    *g = -exp(A_log) * softplus(a + dt_bias);
#endif
    *beta = sigmoid(b);
}

/* L2 normalisation over n elements, times `scale` ("GatedDeltaRule.ixx": q and k are
 * brought to unit L2 norm, and q is then multiplied by dk^-1/2). */
static void l2_normalise(const float* x, int n, double scale, double* out) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += (double)x[i] * (double)x[i];
    double r = scale / sqrt(ss + ORACLE_NORM_EPS);
    for (int i = 0; i < n; ++i) out[i] = (double)x[i] * r;
}

/* One step of the rule on one head's state S[dk][dv] (row-major, dv fastest), from
 * prepared q_hat, k_hat, gamma = exp(g) and beta.  Writes o[dv]. */
static void step(double* S, const double* qh, const double* kh, const float* v, double gamma,
                 double beta, int erase, int dk, int dv, double* delta, double* o) {
    /* S <- S * exp(g) */
    for (int i = 0; i < dk * dv; ++i) S[i] *= gamma;
    /* delta <- (v - k^T S) * beta  (without the erase term: delta <- v * beta) */
    for (int j = 0; j < dv; ++j) {
        double ks = 0.0;
        if (erase)
            for (int i = 0; i < dk; ++i) ks += kh[i] * S[i * dv + j];
#ifdef ORACLE_MUTATE_ERASE_SIGN
        delta[j] = ((double)v[j] + ks) * beta;
#else
        delta[j] = ((double)v[j] - ks) * beta;
#endif
    }
#ifdef ORACLE_MUTATE_OUTPUT_BEFORE_UPDATE
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += qh[i] * S[i * dv + j];
        o[j] = acc;
    }
#endif
    /* S <- S + k (outer) delta */
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] += kh[i] * delta[j];
#ifndef ORACLE_MUTATE_OUTPUT_BEFORE_UPDATE
    /* o <- q^T S, from the updated state */
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += qh[i] * S[i * dv + j];
        o[j] = acc;
    }
#endif
}

typedef struct {
    /* raw inputs (float; exact copies of bf16 / fp32 values) */
    const float *q, *k, *v, *a, *b;
    const float *A_log, *dt_bias;
    /* prepared inputs (double), used instead of the raw ones when qh != NULL */
    const double *qh, *kh, *g, *beta;
    const double* init_state;
    double *out, *final_state;
    const int64_t* cu_seqlens;
    int nseq, Hk, Hv, dk, dv, erase;
    int next_unit; /* shared work counter */
    pthread_mutex_t lock;
} job_t;

static void run_unit(job_t* J, int unit) {
    const int s = unit / J->Hv, h = unit % J->Hv;
    const int dk = J->dk, dv = J->dv, Hk = J->Hk, Hv = J->Hv;
    const int kh_idx = h / (Hv / Hk);
    const int64_t t0 = J->cu_seqlens[s], t1 = J->cu_seqlens[s + 1];
    double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
    double* qh = (double*)malloc(sizeof(double) * (size_t)dk);
    double* kv = (double*)malloc(sizeof(double) * (size_t)dk);
    double* delta = (double*)malloc(sizeof(double) * (size_t)dv);
    if (J->init_state)
        memcpy(S, J->init_state + ((size_t)s * Hv + h) * dk * dv, sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);
#ifdef ORACLE_MUTATE_DROP_QSCALE
    const double qscale = 1.0;
#else
    const double qscale = 1.0 / sqrt((double)dk);
#endif
    for (int64_t t = t0; t < t1; ++t) {
        const size_t qk_off = ((size_t)t * Hk + kh_idx) * dk;
        const size_t th = (size_t)t * Hv + h;
        double g, beta;
        if (J->qh) {
            memcpy(qh, J->qh + qk_off, sizeof(double) * dk);
            memcpy(kv, J->kh + qk_off, sizeof(double) * dk);
            g = J->g[th];
            beta = J->beta[th];
        } else {
            l2_normalise(J->q + qk_off, dk, qscale, qh);
            l2_normalise(J->k + qk_off, dk, 1.0, kv);
            oracle_gating(J->a[th], J->b[th], J->A_log[h], J->dt_bias[h], &g, &beta);
        }
        step(S, qh, kv, J->v + th * dv, exp(g), beta, J->erase, dk, dv, delta,
             J->out + th * dv);
    }
    if (J->final_state)
        memcpy(J->final_state + ((size_t)s * Hv + h) * dk * dv, S, sizeof(double) * dk * dv);
    free(S);
    free(qh);
    free(kv);
    free(delta);
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    const int total = J->nseq * J->Hv;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= total) break;
        run_unit(J, u);
    }
    return NULL;
}

static int run_job(job_t* J, int nthreads) {
    if (J->Hk <= 0 || J->Hv <= 0 || J->Hv % J->Hk != 0 || J->dk <= 0 || J->dv <= 0 || J->nseq <= 0)
        return -1;
    if (nthreads < 1) nthreads = 1;
    J->next_unit = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, worker, J) == 0) ++started;
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return 0;
}

/*
 * Full forward pass from raw inputs.
 *   q, k        [N, Hk, dk]   (N = total tokens over all sequences)
 *   v           [N, Hv, dv]
 *   a, b        [N, Hv]
 *   A_log, dt_bias [Hv]
 *   init_state  [nseq, Hv, dk, dv] or NULL (zeros)
 *   out         [N, Hv, dv];  final_state [nseq, Hv, dk, dv] or NULL
 *   cu_seqlens  [nseq + 1], cu_seqlens[0] = 0, cu_seqlens[nseq] = N
 *   erase       1 = gated delta rule, 0 = gated linear attention
 * Returns 0, or -1 on inconsistent sizes.
 */
int oracle_gdr_forward(const float* q, const float* k, const float* v, const float* a,
                       const float* b, const float* A_log, const float* dt_bias,
                       const double* init_state, double* out, double* final_state,
                       const int64_t* cu_seqlens, int nseq, int Hk, int Hv, int dk, int dv,
                       int erase, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.a = a; J.b = b; J.A_log = A_log; J.dt_bias = dt_bias;
    J.init_state = init_state; J.out = out; J.final_state = final_state;
    J.cu_seqlens = cu_seqlens; J.nseq = nseq; J.Hk = Hk; J.Hv = Hv; J.dk = dk; J.dv = dv;
    J.erase = erase;
    return run_job(&J, nthreads);
}

/*
 * The recurrence alone, from prepared inputs: q_hat, k_hat [N, Hk, dk] (already
 * normalised and scaled), g, beta [N, Hv] (log-decay and write strength), v as above.
 */
int oracle_gdr_core(const double* qh, const double* kh, const float* v, const double* g,
                    const double* beta, const double* init_state, double* out,
                    double* final_state, const int64_t* cu_seqlens, int nseq, int Hk, int Hv,
                    int dk, int dv, int erase, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof(J));
    J.qh = qh; J.kh = kh; J.v = v; J.g = g; J.beta = beta;
    J.init_state = init_state; J.out = out; J.final_state = final_state;
    J.cu_seqlens = cu_seqlens; J.nseq = nseq; J.Hk = Hk; J.Hv = Hv; J.dk = dk; J.dv = dv;
    J.erase = erase;
    return run_job(&J, nthreads);
}

/*
 * The preparation step alone: q_hat, k_hat [N, Hk, dk] and g, beta [N, Hv] from the raw
 * inputs, exactly as oracle_gdr_forward forms them before each step.
 */
void oracle_prepare(const float* q, const float* k, const float* a, const float* b,
                    const float* A_log, const float* dt_bias, double* qh, double* kh, double* g,
                    double* beta, int64_t N, int Hk, int Hv, int dk) {
#ifdef ORACLE_MUTATE_DROP_QSCALE
    const double qscale = 1.0;
#else
    const double qscale = 1.0 / sqrt((double)dk);
#endif
    for (int64_t t = 0; t < N; ++t) {
        for (int h = 0; h < Hk; ++h) {
            const size_t off = ((size_t)t * Hk + h) * dk;
            l2_normalise(q + off, dk, qscale, qh + off);
            l2_normalise(k + off, dk, 1.0, kh + off);
        }
        for (int h = 0; h < Hv; ++h) {
            const size_t th = (size_t)t * Hv + h;
            oracle_gating(a[th], b[th], A_log[h], dt_bias[h], &g[th], &beta[th]);
        }
    }
}

/* Gating over an array of n tokens of one head (for pins on the gate formula). */
void oracle_gating_array(int n, const double* a, const double* b, double A_log, double dt_bias,
                         double* g, double* beta) {
    for (int i = 0; i < n; ++i) oracle_gating(a[i], b[i], A_log, dt_bias, &g[i], &beta[i]);
}
