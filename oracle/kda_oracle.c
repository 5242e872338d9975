/*
 * fp64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg load this file; the CUDA library never does, and this file
 * includes nothing from it.
 *
 * What it computes (the plain definition, token by token, in fp64):
 *
 *   S~_t = Diag(alpha_t) S_{t-1}                 "forget": every row c of the
 *                                                d_k x d_v state is scaled by
 *                                                alpha_t[c]   (Ten questions, Q8)
 *   u_t  = beta_t (v_t - S~_t^T k_t)             "look up, take the error"
 *                                                (Ten questions, Q6; 22,580 §5.2)
 *   S_t  = S~_t + k_t u_t^T                      "write the correction"
 *                                                (Ten questions, Q3 + Q6)
 *   o_t  = S_t^T (s q_t),  s = d_k^{-1/2}         "read"  (Ten questions, Q4;
 *                                                the query scale is the one of the
 *                                                KDA bra-ket blog's preamble)
 *
 * which is S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 * o_t = S_t^T (s q_t) -- the equation of "Ten questions", intro and 终局, with
 * the scale of the bra-ket blog.  alpha_t = exp(log_alpha_t) per channel;
 * log_alpha = -inf gives alpha = 0 exactly.
 *
 * Citations name the pages by title:
 *   "Ten questions"  = 会加减乘除就够:十个问题,手算读懂 Kimi K3 心脏里的全部数学
 *                      (jokeuncle.github.io)
 *   "22,580"         = 22,580：从 GPT-2 到 Kimi K3 —— 大模型架构七年进化全解
 *                      (yichencityu.github.io)
 *   "KDA bra-ket blog" = the translated blog on the DeltaNet family (mynewscn.com)
 *
 * Layout (all row-major): tokens are packed along one axis.
 *   q, k, log_alpha [T_total, H, dk];  v [T_total, H, dv];  beta [T_total, H]
 *   S0 [N, H, dk, dv] (NULL = zero state);  cu_seqlens [N + 1] (int64 offsets)
 * Each input has its own element type code (KO_F64, KO_F32, KO_BF16 = raw
 * uint16 bf16 bits); every value is widened exactly to fp64 before use.
 *
 * A task is one (sequence n, head h) pair.  Outputs are compact, in task order:
 *   out      : for task j, T_n x dv values (T_n = length of sequence n)
 *   S_final  : for task j, dk x dv values
 * Tasks run in parallel on plain pthreads; each task is independent.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { KO_F64 = 0, KO_F32 = 1, KO_BF16 = 2 };

static double widen(const void *p, int dt, int64_t i) {
    switch (dt) {
    case KO_F64:
        return ((const double *)p)[i];
    case KO_F32:
        return (double)((const float *)p)[i];
    case KO_BF16: {
        uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    default:
        return NAN;
    }
}

typedef struct {
    const void *q, *k, *v, *la, *beta, *S0;
    int q_dt, k_dt, v_dt, la_dt, b_dt, s0_dt;
    const int64_t *cu;
    int64_t H, dk, dv;
    double scale;
    const int64_t *tasks;
    const int64_t *out_off;
    int64_t ntasks;
    double *out, *S_final;
    int64_t next;            /* shared task counter */
    pthread_mutex_t lock;
} job_t;

static void run_task(job_t *J, int64_t j) {
    const int64_t n = J->tasks[2 * j], h = J->tasks[2 * j + 1];
    const int64_t H = J->H, dk = J->dk, dv = J->dv;
    double *S = J->S_final + j * dk * dv;        /* the state lives in the output slot */
    double *kv = malloc(sizeof(double) * (size_t)(2 * dk + dv + 2 * dv));
    double *kt = kv, *qt = kv + dk, *vt = kv + 2 * dk, *r = vt + dv, *u = r + dv;
    double *o = J->out + J->out_off[j];

    for (int64_t c = 0; c < dk; ++c)
        for (int64_t x = 0; x < dv; ++x)
            S[c * dv + x] = J->S0 ? widen(J->S0, J->s0_dt, ((n * H + h) * dk + c) * dv + x) : 0.0;

    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const int64_t base_k = (t * H + h) * dk, base_v = (t * H + h) * dv;
        for (int64_t c = 0; c < dk; ++c) {
            kt[c] = widen(J->k, J->k_dt, base_k + c);
            qt[c] = J->scale * widen(J->q, J->q_dt, base_k + c);
        }
        for (int64_t x = 0; x < dv; ++x) vt[x] = widen(J->v, J->v_dt, base_v + x);
        const double b = widen(J->beta, J->b_dt, t * H + h);

        /* forget: S~ = Diag(alpha) S */
        for (int64_t c = 0; c < dk; ++c) {
            const double a = exp(widen(J->la, J->la_dt, base_k + c));
            for (int64_t x = 0; x < dv; ++x) S[c * dv + x] *= a;
        }
        /* look up: r = S~^T k */
        for (int64_t x = 0; x < dv; ++x) r[x] = 0.0;
        for (int64_t c = 0; c < dk; ++c)
            for (int64_t x = 0; x < dv; ++x) r[x] += S[c * dv + x] * kt[c];
        /* error times strength: u = beta (v - r) */
        for (int64_t x = 0; x < dv; ++x) u[x] = b * (vt[x] - r[x]);
        /* write: S = S~ + k u^T */
        for (int64_t c = 0; c < dk; ++c)
            for (int64_t x = 0; x < dv; ++x) S[c * dv + x] += kt[c] * u[x];
        /* read: o = S^T (s q) */
        double *ot = o + (t - J->cu[n]) * dv;
        for (int64_t x = 0; x < dv; ++x) ot[x] = 0.0;
        for (int64_t c = 0; c < dk; ++c)
            for (int64_t x = 0; x < dv; ++x) ot[x] += S[c * dv + x] * qt[c];
    }
    free(kv);
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t j = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (j >= J->ntasks) break;
        run_task(J, j);
    }
    return NULL;
}

/* Returns 0 on success, -1 on a bad argument. */
int kda_oracle_recurrent(const void *q, int q_dt, const void *k, int k_dt, const void *v, int v_dt,
                         const void *log_alpha, int la_dt, const void *beta, int b_dt,
                         const void *S0, int s0_dt, const int64_t *cu_seqlens, int64_t N,
                         int64_t H, int64_t dk, int64_t dv, double scale, const int64_t *tasks,
                         int64_t ntasks, double *out, double *S_final, int nthreads) {
    if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !tasks || !out || !S_final)
        return -1;
    if (N <= 0 || H <= 0 || dk <= 0 || dv <= 0 || ntasks < 0) return -1;
    int64_t *out_off = malloc(sizeof(int64_t) * (size_t)(ntasks + 1));
    out_off[0] = 0;
    for (int64_t j = 0; j < ntasks; ++j) {
        const int64_t n = tasks[2 * j], h = tasks[2 * j + 1];
        if (n < 0 || n >= N || h < 0 || h >= H || cu_seqlens[n + 1] < cu_seqlens[n]) {
            free(out_off);
            return -1;
        }
        out_off[j + 1] = out_off[j] + (cu_seqlens[n + 1] - cu_seqlens[n]) * dv;
    }
    job_t J = {q, k, v, log_alpha, beta, S0, q_dt, k_dt, v_dt, la_dt, b_dt, s0_dt,
               cu_seqlens, H, dk, dv, scale, tasks, out_off, ntasks, out, S_final, 0,
               PTHREAD_MUTEX_INITIALIZER};
    if (nthreads < 1) nthreads = 1;
    if (nthreads > ntasks) nthreads = ntasks > 0 ? (int)ntasks : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
    worker(&J);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    free(out_off);
    return 0;
}
