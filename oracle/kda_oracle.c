/*
 * kda_oracle.c -- plain, slow fp64 CPU oracle for the KDA (gated delta rule with
 * per-channel decay) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library path links, loads or calls this
 * file: only the tests, the package smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes.  The pages ("Trillion-Scale MoE Multimodal Models: Practical
 * Techniques ..." section 3.2, and "Breaking Through Trillion-Parameter Multimodal
 * MoE ..." section 2.1) fix the lower-bounded log-decay
 *
 *     g_t = g_min * sigmoid(a_t),  g_min = -5             (bounded gate)
 *
 * and name the unbounded alternative log(sigmoid(x)) with range (-inf, 0).  They call
 * the attention "incremental" with a constant-size state updated token by token
 * ("Trillion-Parameter MoE Multimodal Models: Engineering ..." section 3.2) and say it
 * is a Delta-Net-style linear attention with a per-chunk cumulative decay Gamma
 * ("Breaking Through ..." section 2.1).  The recurrence itself is not printed on the
 * pages; the plainest reading consistent with all of the above, used here, is
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t                      (output reads the state after token t)
 *
 * with S a dk x dv matrix, natural-log decay, decay applied before the erase/write.
 *
 * Every computation is fp64.  Inputs are float32 arrays (bf16 inputs are exactly
 * representable in float32, so the caller passes the quantised values unchanged).
 *
 * Layouts (row-major, innermost last):
 *   q, k, a : [B, T, H, dk]    v, o : [B, T, H, dv]    beta : [B, T, H]
 *   S0, ST  : [B, H, dk, dv]
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_GATE_BOUNDED 0    /* g = g_min * sigmoid(a)                      */
#define ORACLE_GATE_LOGSIGMOID 1 /* g = log(sigmoid(a)), unbounded (ablation)   */

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* ------------------------------------------------------------------------------ */
/* Gate.  "Trillion-Scale ..." section 3.2 (g = g_min * Sigmoid(...), g_min = -5) and
 * "Breaking Through ..." section 2.1 (g_t = g_min * sigma(w x_t + b); the unbounded form
 * is log(sigma(x))).  The pre-activation a is the argument of the sigmoid.              */
static double gate_f64(double a, double g_min, int kind)
{
    if (kind == ORACLE_GATE_BOUNDED)
        return g_min / (1.0 + exp(-a)); /* g_min * sigmoid(a) */
    /* log(sigmoid(a)) = -log(1 + exp(-a)), written so neither branch overflows. */
    if (a >= 0.0)
        return -log1p(exp(-a));
    return a - log1p(exp(a));
}

void oracle_gate_f64(const float *a, int64_t n, double g_min, int kind, double *g)
{
    for (int64_t i = 0; i < n; ++i)
        g[i] = gate_f64((double)a[i], g_min, kind);
}

/* g rounded once (round-to-nearest-even) from the fp64 value to float32. */
void oracle_gate_f32(const float *a, int64_t n, double g_min, int kind, float *g)
{
    for (int64_t i = 0; i < n; ++i)
        g[i] = (float)gate_f64((double)a[i], g_min, kind);
}

/* Gate with a per-head scale on the pre-activation.  "Trillion-Scale ..." section 3.2
 * writes the bounded gate as g = g_min * Sigmoid(e^A * h * z): the argument of the sigmoid
 * is the projection h * z (the caller's `a`) scaled by e^A, one A per head.  a is
 * [n_tok, H, dk] flattened, A_log is [H]; evaluated in fp64 and rounded once.            */
void oracle_gate_heads_f32(const float *a, int64_t n_tok, int H, int dk, double g_min, const float *A_log,
                           float *g)
{
    for (int64_t t = 0; t < n_tok; ++t)
        for (int h = 0; h < H; ++h) {
            const double scale = exp((double)A_log[h]);
            for (int c = 0; c < dk; ++c) {
                const int64_t i = (t * H + h) * dk + c;
                g[i] = (float)gate_f64((double)a[i] * scale, g_min, ORACLE_GATE_BOUNDED);
            }
        }
}

/* ------------------------------------------------------------------------------ */
/* Work distribution over independent (b, h) sequences.                           */
typedef struct {
    int B, T, H, dk, dv, C;
    const float *q, *k, *v, *a, *beta;
    double g_min;
    int kind;
    const double *S0;
    double *o, *ST;
    int nthreads, tid;
    int status;
    /* backward only: upstream gradients in (dO, dST), input gradients out (g*) */
    const float *dO;
    const double *dST;
    double *gq, *gk, *gv, *ga, *gbeta, *gS0;
} job_t;

static int resolve_threads(int nthreads, int units)
{
    if (nthreads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = n > 0 ? (int)n : 1;
    }
    if (nthreads > units)
        nthreads = units;
    return nthreads < 1 ? 1 : nthreads;
}

static int run_jobs(job_t *proto, void *(*fn)(void *))
{
    int units = proto->B * proto->H;
    int nt = resolve_threads(proto->nthreads, units);
    job_t *jobs = (job_t *)calloc((size_t)nt, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return ORACLE_ERR_NOMEM;
    }
    for (int i = 0; i < nt; ++i) {
        jobs[i] = *proto;
        jobs[i].nthreads = nt;
        jobs[i].tid = i;
        jobs[i].status = ORACLE_OK;
    }
    for (int i = 1; i < nt; ++i)
        pthread_create(&th[i], NULL, fn, &jobs[i]);
    fn(&jobs[0]);
    int st = jobs[0].status;
    for (int i = 1; i < nt; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].status != ORACLE_OK)
            st = jobs[i].status;
    }
    free(jobs);
    free(th);
    return st;
}

#define IDX_TOK(b, t, h, c, T, H, D) (((((int64_t)(b) * (T) + (t)) * (H) + (h)) * (D)) + (c))
#define IDX_BETA(b, t, h, T, H) ((((int64_t)(b) * (T) + (t)) * (H)) + (h))
#define IDX_S(b, h, H, dk, dv) ((((int64_t)(b) * (H)) + (h)) * (int64_t)(dk) * (dv))

/* ------------------------------------------------------------------------------ */
/* Token-by-token recurrence (the definition).                                     */
static void *recurrence_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *kS = (double *)malloc(sizeof(double) * (size_t)dv);
    double *decay = (double *)malloc(sizeof(double) * (size_t)dk);
    if (!S || !kS || !decay) {
        J->status = ORACLE_ERR_NOMEM;
        free(S);
        free(kS);
        free(decay);
        return NULL;
    }
    for (int unit = J->tid; unit < J->B * H; unit += J->nthreads) {
        const int b = unit / H, h = unit % H;
        const int64_t s_off = IDX_S(b, h, H, dk, dv);
        if (J->S0)
            memcpy(S, J->S0 + s_off, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t = 0; t < T; ++t) {
            const float *q = J->q + IDX_TOK(b, t, h, 0, T, H, dk);
            const float *k = J->k + IDX_TOK(b, t, h, 0, T, H, dk);
            const float *a = J->a + IDX_TOK(b, t, h, 0, T, H, dk);
            const float *v = J->v + IDX_TOK(b, t, h, 0, T, H, dv);
            const double beta = (double)J->beta[IDX_BETA(b, t, h, T, H)];
            double *o = J->o + IDX_TOK(b, t, h, 0, T, H, dv);
            /* Diag(exp g_t) S_{t-1}: decay every row i (key channel) of the state. */
            for (int i = 0; i < dk; ++i)
                decay[i] = exp(gate_f64((double)a[i], J->g_min, J->kind));
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(int64_t)i * dv + j] *= decay[i];
            /* k^T (decayed S): the part of the state the erase term removes. */
            for (int j = 0; j < dv; ++j)
                kS[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    kS[j] += (double)k[i] * S[(int64_t)i * dv + j];
            /* S_t = (I - beta k k^T) S_dec + beta k v^T, term by term. */
            for (int i = 0; i < dk; ++i) {
                const double ki = (double)k[i];
                for (int j = 0; j < dv; ++j)
                    S[(int64_t)i * dv + j] += -beta * ki * kS[j] + beta * ki * (double)v[j];
            }
            /* o_t = S_t^T q_t */
            for (int j = 0; j < dv; ++j)
                o[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double qi = (double)q[i];
                for (int j = 0; j < dv; ++j)
                    o[j] += S[(int64_t)i * dv + j] * qi;
            }
        }
        if (J->ST)
            memcpy(J->ST + s_off, S, sizeof(double) * (size_t)dk * dv);
    }
    free(S);
    free(kS);
    free(decay);
    return NULL;
}

static int check_common(int B, int T, int H, int dk, int dv, const void *q, const void *k,
                        const void *v, const void *a, const void *beta)
{
    if (B < 0 || T < 0 || H < 0 || dk < 1 || dv < 1)
        return ORACLE_ERR_ARG;
    if ((int64_t)B * T * H > 0 && (!q || !k || !v || !a || !beta))
        return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

/* S0 may be NULL (zero state) and may alias ST (each unit copies S0 before it writes
 * ST); o may be NULL only when T == 0.                                              */
int oracle_recurrence(int B, int T, int H, int dk, int dv, const float *q, const float *k,
                      const float *v, const float *a, const float *beta, double g_min, int kind,
                      const double *S0, double *o, double *ST, int nthreads)
{
    int st = check_common(B, T, H, dk, dv, q, k, v, a, beta);
    if (st != ORACLE_OK)
        return st;
    if (B * H == 0)
        return ORACLE_OK;
    if (T > 0 && !o)
        return ORACLE_ERR_ARG;
    job_t J = {B, T, H, dk, dv, 0, q, k, v, a, beta, g_min, kind, S0, o, ST, nthreads, 0, 0};
    return run_jobs(&J, recurrence_worker);
}

/* ------------------------------------------------------------------------------ */
/* Chunked form, derived from the recurrence (the pages' "chunked computation with a
 * cumulative decay Gamma and its inverse", "Trillion-Scale ..." section 3.1).  Inside a
 * chunk with entering state S, G_r = sum_{s<=r} g_s and, with u_r the per-token delta
 * corrections,
 *   (I + A) U = diag(beta) (V - Kbar S),  A_rj = beta_r sum_c k_rc k_jc e^{G_rc - G_jc} (j<r)
 *   O = Qbar S + lower_incl(P) U,         P_rj = sum_c q_rc k_jc e^{G_rc - G_jc}     (j<=r)
 *   S_next = Diag(e^{G_last}) S + sum_j (k_j * e^{G_last - G_j}) u_j^T
 * with Kbar = k * e^{G}, Qbar = q * e^{G}.  Every exponential here is of a pairwise
 * difference, so nothing overflows at any chunk size; U is found by forward
 * substitution.                                                                     */
static void *chunked_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv, C = J->C;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *G = (double *)malloc(sizeof(double) * (size_t)C * dk);
    double *U = (double *)malloc(sizeof(double) * (size_t)C * dv);
    double *Snew = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    if (!S || !G || !U || !Snew) {
        J->status = ORACLE_ERR_NOMEM;
        free(S);
        free(G);
        free(U);
        free(Snew);
        return NULL;
    }
    for (int unit = J->tid; unit < J->B * H; unit += J->nthreads) {
        const int b = unit / H, h = unit % H;
        const int64_t s_off = IDX_S(b, h, H, dk, dv);
        if (J->S0)
            memcpy(S, J->S0 + s_off, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t0 = 0; t0 < T; t0 += C) {
            const int n = (T - t0) < C ? (T - t0) : C;
            /* cumulative log-decay inside the chunk */
            for (int r = 0; r < n; ++r) {
                const float *a = J->a + IDX_TOK(b, t0 + r, h, 0, T, H, dk);
                for (int c = 0; c < dk; ++c) {
                    const double gv = gate_f64((double)a[c], J->g_min, J->kind);
                    G[(int64_t)r * dk + c] = (r ? G[(int64_t)(r - 1) * dk + c] : 0.0) + gv;
                }
            }
            /* delta corrections U by forward substitution on (I + A) U = rhs */
            for (int r = 0; r < n; ++r) {
                const float *kr = J->k + IDX_TOK(b, t0 + r, h, 0, T, H, dk);
                const float *vr = J->v + IDX_TOK(b, t0 + r, h, 0, T, H, dv);
                const double br = (double)J->beta[IDX_BETA(b, t0 + r, h, T, H)];
                double *ur = U + (int64_t)r * dv;
                /* rhs_r = beta_r (v_r - (k_r * e^{G_r})^T S) */
                for (int j = 0; j < dv; ++j)
                    ur[j] = (double)vr[j];
                for (int c = 0; c < dk; ++c) {
                    const double kb = (double)kr[c] * exp(G[(int64_t)r * dk + c]);
                    for (int j = 0; j < dv; ++j)
                        ur[j] -= kb * S[(int64_t)c * dv + j];
                }
                for (int j = 0; j < dv; ++j)
                    ur[j] *= br;
                /* - sum_{s<r} A_rs u_s */
                for (int s = 0; s < r; ++s) {
                    const float *ks = J->k + IDX_TOK(b, t0 + s, h, 0, T, H, dk);
                    double A_rs = 0.0;
                    for (int c = 0; c < dk; ++c)
                        A_rs += (double)kr[c] * (double)ks[c] *
                                exp(G[(int64_t)r * dk + c] - G[(int64_t)s * dk + c]);
                    A_rs *= br;
                    for (int j = 0; j < dv; ++j)
                        ur[j] -= A_rs * U[(int64_t)s * dv + j];
                }
            }
            /* outputs O = Qbar S + lower_incl(P) U */
            for (int r = 0; r < n; ++r) {
                const float *qr = J->q + IDX_TOK(b, t0 + r, h, 0, T, H, dk);
                double *o = J->o + IDX_TOK(b, t0 + r, h, 0, T, H, dv);
                for (int j = 0; j < dv; ++j)
                    o[j] = 0.0;
                for (int c = 0; c < dk; ++c) {
                    const double qb = (double)qr[c] * exp(G[(int64_t)r * dk + c]);
                    for (int j = 0; j < dv; ++j)
                        o[j] += qb * S[(int64_t)c * dv + j];
                }
                for (int s = 0; s <= r; ++s) {
                    const float *ks = J->k + IDX_TOK(b, t0 + s, h, 0, T, H, dk);
                    double P_rs = 0.0;
                    for (int c = 0; c < dk; ++c)
                        P_rs += (double)qr[c] * (double)ks[c] *
                                exp(G[(int64_t)r * dk + c] - G[(int64_t)s * dk + c]);
                    for (int j = 0; j < dv; ++j)
                        o[j] += P_rs * U[(int64_t)s * dv + j];
                }
            }
            /* state carried to the next chunk */
            const double *Gl = G + (int64_t)(n - 1) * dk;
            for (int c = 0; c < dk; ++c) {
                const double dc = exp(Gl[c]);
                for (int j = 0; j < dv; ++j)
                    Snew[(int64_t)c * dv + j] = dc * S[(int64_t)c * dv + j];
            }
            for (int s = 0; s < n; ++s) {
                const float *ks = J->k + IDX_TOK(b, t0 + s, h, 0, T, H, dk);
                for (int c = 0; c < dk; ++c) {
                    const double kh = (double)ks[c] * exp(Gl[c] - G[(int64_t)s * dk + c]);
                    for (int j = 0; j < dv; ++j)
                        Snew[(int64_t)c * dv + j] += kh * U[(int64_t)s * dv + j];
                }
            }
            memcpy(S, Snew, sizeof(double) * (size_t)dk * dv);
        }
        if (J->ST)
            memcpy(J->ST + s_off, S, sizeof(double) * (size_t)dk * dv);
    }
    free(S);
    free(G);
    free(U);
    free(Snew);
    return NULL;
}

int oracle_chunked(int C, int B, int T, int H, int dk, int dv, const float *q, const float *k,
                   const float *v, const float *a, const float *beta, double g_min, int kind,
                   const double *S0, double *o, double *ST, int nthreads)
{
    int st = check_common(B, T, H, dk, dv, q, k, v, a, beta);
    if (st != ORACLE_OK || C < 1)
        return st != ORACLE_OK ? st : ORACLE_ERR_ARG;
    if (B * H == 0)
        return ORACLE_OK;
    if (T > 0 && !o)
        return ORACLE_ERR_ARG;
    job_t J = {B, T, H, dk, dv, C, q, k, v, a, beta, g_min, kind, S0, o, ST, nthreads, 0, 0};
    return run_jobs(&J, chunked_worker);
}

/* ------------------------------------------------------------------------------ */
/* Backward of the recurrence (reverse-mode derivative, written out by hand).
 *
 * "Trillion-Parameter MoE Multimodal Models: Engineering ..." section 3.2 says long
 * sequences are trained by recursing in chunks; training needs the gradients of a scalar
 * loss L with respect to every input, given dL/do_t for every token and dL/dS_T.  The
 * pages print no backward, so this is the derivative of the recurrence above and nothing
 * else.  Per token, with S_prev = S_{t-1}:
 *
 *   Sd  = Diag(e^{g_t}) S_prev          (decayed state)
 *   r   = v_t - Sd^T k_t,  u = beta_t r (delta correction)
 *   S_t = Sd + k_t u^T,    o_t = S_t^T q_t
 *
 * and, walking t from T down to 1 with dS = dL/dS_t (dL/dS_T first):
 *
 *   dS      += q_t do_t^T               dq_t = S_t do_t
 *   du       = dS^T k_t                 dk_t = dS u + Sd (-beta_t du)
 *   dbeta_t  = du . r                   dv_t = beta_t du
 *   dSd      = dS + k_t (-beta_t du)^T
 *   dg_t[i]  = sum_j dSd[i,j] Sd[i,j]   da_t = dg_t * dg/da
 *   dS_prev  = Diag(e^{g_t}) dSd
 *
 * dL/dS0 is the last dS_prev.  The states S_{t-1} are recomputed from checkpoints kept
 * every BWD_SEG tokens, so memory stays O((T / BWD_SEG + BWD_SEG) dk dv) per sequence.  */
#define BWD_SEG 64

/* dg/da for the two gates: g_min * s (1 - s) (bounded) or 1 - s (log-sigmoid), with
 * s = sigmoid(a).                                                                      */
static double gate_grad_f64(double a, double g_min, int kind)
{
    const double s = 1.0 / (1.0 + exp(-a));
    if (kind == ORACLE_GATE_BOUNDED)
        return g_min * s * (1.0 - s);
    return 1.0 - s;
}

/* One forward token: S_prev -> S (both dk x dv); decay and r are scratch.           */
static void bwd_forward_token(const job_t *J, int b, int t, int h, const double *S_prev, double *S,
                              double *decay, double *r)
{
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    const float *k = J->k + IDX_TOK(b, t, h, 0, T, H, dk);
    const float *a = J->a + IDX_TOK(b, t, h, 0, T, H, dk);
    const float *v = J->v + IDX_TOK(b, t, h, 0, T, H, dv);
    const double beta = (double)J->beta[IDX_BETA(b, t, h, T, H)];
    for (int i = 0; i < dk; ++i) {
        decay[i] = exp(gate_f64((double)a[i], J->g_min, J->kind));
        for (int j = 0; j < dv; ++j)
            S[(int64_t)i * dv + j] = decay[i] * S_prev[(int64_t)i * dv + j];
    }
    for (int j = 0; j < dv; ++j) {
        double kS = 0.0;
        for (int i = 0; i < dk; ++i)
            kS += (double)k[i] * S[(int64_t)i * dv + j];
        r[j] = (double)v[j] - kS;
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(int64_t)i * dv + j] += (double)k[i] * beta * r[j];
}

static void *backward_worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    const size_t SZ = (size_t)dk * dv;
    const int nseg = (T + BWD_SEG - 1) / BWD_SEG;
    double *ckpt = (double *)malloc(sizeof(double) * SZ * (size_t)(nseg > 0 ? nseg : 1));
    double *seg = (double *)malloc(sizeof(double) * SZ * (BWD_SEG + 1));
    double *Sd = (double *)malloc(sizeof(double) * SZ);
    double *dS = (double *)malloc(sizeof(double) * SZ);
    double *decay = (double *)malloc(sizeof(double) * (size_t)dk);
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    double *du = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!ckpt || !seg || !Sd || !dS || !decay || !r || !du) {
        J->status = ORACLE_ERR_NOMEM;
        goto done;
    }
    for (int unit = J->tid; unit < J->B * H; unit += J->nthreads) {
        const int b = unit / H, h = unit % H;
        const int64_t s_off = IDX_S(b, h, H, dk, dv);
        /* forward, keeping the state that enters every segment */
        double *S = seg, *S_next = seg + SZ;
        if (J->S0)
            memcpy(S, J->S0 + s_off, sizeof(double) * SZ);
        else
            memset(S, 0, sizeof(double) * SZ);
        for (int t = 0; t < T; ++t) {
            if (t % BWD_SEG == 0)
                memcpy(ckpt + (size_t)(t / BWD_SEG) * SZ, S, sizeof(double) * SZ);
            bwd_forward_token(J, b, t, h, S, S_next, decay, r);
            memcpy(S, S_next, sizeof(double) * SZ);
        }
        /* reverse sweep */
        if (J->dST)
            memcpy(dS, J->dST + s_off, sizeof(double) * SZ);
        else
            memset(dS, 0, sizeof(double) * SZ);
        for (int sg = nseg - 1; sg >= 0; --sg) {
            const int t0 = sg * BWD_SEG, t1 = (t0 + BWD_SEG < T) ? t0 + BWD_SEG : T;
            /* seg[j] = S_{t0 + j - 1}: the state entering token t0 + j, j = 0 .. t1 - t0 */
            memcpy(seg, ckpt + (size_t)sg * SZ, sizeof(double) * SZ);
            for (int t = t0; t < t1; ++t)
                bwd_forward_token(J, b, t, h, seg + (size_t)(t - t0) * SZ, seg + (size_t)(t - t0 + 1) * SZ,
                                  decay, r);
            for (int t = t1 - 1; t >= t0; --t) {
                const double *S_prev = seg + (size_t)(t - t0) * SZ;
                const double *S_t = seg + (size_t)(t - t0 + 1) * SZ;
                const float *q = J->q + IDX_TOK(b, t, h, 0, T, H, dk);
                const float *k = J->k + IDX_TOK(b, t, h, 0, T, H, dk);
                const float *a = J->a + IDX_TOK(b, t, h, 0, T, H, dk);
                const float *dO = J->dO + IDX_TOK(b, t, h, 0, T, H, dv);
                const double beta = (double)J->beta[IDX_BETA(b, t, h, T, H)];
                double *dq = J->gq + IDX_TOK(b, t, h, 0, T, H, dk);
                double *dkk = J->gk + IDX_TOK(b, t, h, 0, T, H, dk);
                double *dvv = J->gv + IDX_TOK(b, t, h, 0, T, H, dv);
                double *da = J->ga + IDX_TOK(b, t, h, 0, T, H, dk);
                /* this token's decayed state Sd and r = v - Sd^T k, again */
                for (int i = 0; i < dk; ++i) {
                    decay[i] = exp(gate_f64((double)a[i], J->g_min, J->kind));
                    for (int j = 0; j < dv; ++j)
                        Sd[(int64_t)i * dv + j] = decay[i] * S_prev[(int64_t)i * dv + j];
                }
                for (int j = 0; j < dv; ++j) {
                    double kS = 0.0;
                    for (int i = 0; i < dk; ++i)
                        kS += (double)k[i] * Sd[(int64_t)i * dv + j];
                    r[j] = (double)J->v[IDX_TOK(b, t, h, j, T, H, dv)] - kS;
                }
                /* o_t = S_t^T q_t */
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j)
                        dS[(int64_t)i * dv + j] += (double)q[i] * (double)dO[j];
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j)
                        acc += S_t[(int64_t)i * dv + j] * (double)dO[j];
                    dq[i] = acc;
                }
                /* S_t = Sd + k u^T, u = beta r */
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i)
                        acc += (double)k[i] * dS[(int64_t)i * dv + j];
                    du[j] = acc;
                }
                double db = 0.0;
                for (int j = 0; j < dv; ++j) {
                    db += du[j] * r[j];
                    dvv[j] = beta * du[j];
                }
                J->gbeta[IDX_BETA(b, t, h, T, H)] = db;
                for (int i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j)
                        acc += dS[(int64_t)i * dv + j] * beta * r[j]          /* from k u^T        */
                               - Sd[(int64_t)i * dv + j] * beta * du[j];      /* from r = v - Sd^T k */
                    dkk[i] = acc;
                }
                /* dSd = dS - beta k du^T; dg; dS_prev */
                for (int i = 0; i < dk; ++i) {
                    double dg = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        const double d = dS[(int64_t)i * dv + j] - beta * (double)k[i] * du[j];
                        dg += d * Sd[(int64_t)i * dv + j];
                        dS[(int64_t)i * dv + j] = decay[i] * d;
                    }
                    da[i] = dg * gate_grad_f64((double)a[i], J->g_min, J->kind);
                }
            }
        }
        if (J->gS0)
            memcpy(J->gS0 + s_off, dS, sizeof(double) * SZ);
    }
done:
    free(ckpt);
    free(seg);
    free(Sd);
    free(dS);
    free(decay);
    free(r);
    free(du);
    return NULL;
}

/* Gradients of L given dO = dL/do [B,T,H,dv] and dST = dL/dS_T [B,H,dk,dv] (NULL: zero).
 * Outputs dq, dk, da [B,T,H,dk], dv [B,T,H,dv], dbeta [B,T,H], dS0 [B,H,dk,dv] (NULL:
 * not stored), all fp64.  S0 NULL means a zero initial state.                          */
int oracle_backward(int B, int T, int H, int dk, int dv, const float *q, const float *k,
                    const float *v, const float *a, const float *beta, double g_min, int kind,
                    const double *S0, const float *dO, const double *dST, double *dq, double *dk_,
                    double *dv_, double *da, double *dbeta, double *dS0, int nthreads)
{
    int st = check_common(B, T, H, dk, dv, q, k, v, a, beta);
    if (st != ORACLE_OK)
        return st;
    if (B * H == 0)
        return ORACLE_OK;
    if (T > 0 && (!dO || !dq || !dk_ || !dv_ || !da || !dbeta))
        return ORACLE_ERR_ARG;
    job_t J = {B, T, H, dk, dv, 0, q, k, v, a, beta, g_min, kind, S0, NULL, NULL, nthreads, 0, 0,
               dO, dST, dq, dk_, dv_, da, dbeta, dS0};
    return run_jobs(&J, backward_worker);
}

/* ------------------------------------------------------------------------------ */
/* One decode step: the recurrence for a single token of N independent sequences.
 * Inputs [N, H, d], beta [N, H], state S [N, H, dk, dv] updated in place.          */
int oracle_decode(int N, int H, int dk, int dv, const float *q, const float *k, const float *v,
                  const float *a, const float *beta, double g_min, int kind, double *S,
                  double *o, int nthreads)
{
    if (!S)
        return ORACLE_ERR_ARG;
    return oracle_recurrence(N, 1, H, dk, dv, q, k, v, a, beta, g_min, kind, S, o, S, nthreads);
}

/* ------------------------------------------------------------------------------ */
/* The numerical claim of "Trillion-Scale ..." section 3.2 / "Breaking Through ..."
 * section 2.1, made concrete: inside one tile of n tokens, factor the pairwise decay
 * e^{G_r - G_j} as a row factor e^{G_r - G_ref} times a column factor e^{G_ref - G_j},
 * both in float32, and multiply the factored operands densely (every (r, j) pair,
 * upper triangle included, as a dense GEMM would).  Reports how many factors or
 * products are not finite and how many nonzero factors are subnormal.
 * g: [n, dk] log-decay of the tile (float32), k: [n, dk], ref: index of the reference
 * token inside the tile (G_ref = sum of g over tokens 0..ref).  counts[0..2] receive
 * (non-finite factors, subnormal factors, non-finite dense products); prod (nullable,
 * [n, n]) receives the dense products row_r . col_j.                                */
int oracle_tile_factors_f32(const float *g, const float *k, int n, int dk, int ref, int64_t *counts,
                            float *prod)
{
    if (!g || !k || !counts || n < 1 || dk < 1 || ref < 0 || ref >= n)
        return ORACLE_ERR_ARG;
    float *G = (float *)malloc(sizeof(float) * (size_t)n * dk);
    float *row = (float *)malloc(sizeof(float) * (size_t)n * dk);
    float *col = (float *)malloc(sizeof(float) * (size_t)n * dk);
    if (!G || !row || !col) {
        free(G);
        free(row);
        free(col);
        return ORACLE_ERR_NOMEM;
    }
    for (int c = 0; c < dk; ++c) {
        float acc = 0.0f;
        for (int r = 0; r < n; ++r) {
            acc += g[(int64_t)r * dk + c];
            G[(int64_t)r * dk + c] = acc;
        }
    }
    counts[0] = counts[1] = counts[2] = 0;
    for (int r = 0; r < n; ++r)
        for (int c = 0; c < dk; ++c) {
            const float Gr = G[(int64_t)r * dk + c], Gf = G[(int64_t)ref * dk + c];
            const float fr = k[(int64_t)r * dk + c] * expf(Gr - Gf);
            const float fc = k[(int64_t)r * dk + c] * expf(Gf - Gr);
            row[(int64_t)r * dk + c] = fr;
            col[(int64_t)r * dk + c] = fc;
            counts[0] += !isfinite(fr) + !isfinite(fc);
            counts[1] += (fpclassify(fr) == FP_SUBNORMAL) + (fpclassify(fc) == FP_SUBNORMAL);
        }
    for (int r = 0; r < n; ++r)
        for (int j = 0; j < n; ++j) {
            float acc = 0.0f;
            for (int c = 0; c < dk; ++c)
                acc += row[(int64_t)r * dk + c] * col[(int64_t)j * dk + c];
            counts[2] += !isfinite(acc);
            if (prod)
                prod[(int64_t)r * n + j] = acc;
        }
    free(G);
    free(row);
    free(col);
    return ORACLE_OK;
}
