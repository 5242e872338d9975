/*
 * fp64 CPU oracle for the gradients of the KDA recurrence (reverse mode, token by token).
 *
 * TEST INFRASTRUCTURE ONLY, like kda_oracle.c: only the tests and the bench's CPU-baseline
 * leg load it; the CUDA library never does, and this file includes nothing from it.
 *
 * The pages discuss training ("22,580" §6.1: prefill is what training runs) but print no
 * backward pass; this is the derivative of the forward oracle's definition, step by step in
 * reverse.  For one (sequence, head), the forward step t is
 *
 *   S~_t = Diag(alpha_t) S_{t-1},  u_t = beta_t (v_t - S~_t^T k_t),
 *   S_t  = S~_t + k_t u_t^T,       o_t = S_t^T (s q_t),  alpha_t = exp(log_alpha_t).
 *
 * Given dO_t = dL/do_t for every token and dS_T = dL/dS_final (zero when absent), with G the
 * gradient with respect to S_t, the reverse step t is
 *
 *   G     += s q_t dO_t^T                       dq_t = s S_t dO_t
 *   du     = G^T k_t                            dk_t = G u_t
 *   r      = v_t - S~_t^T k_t  (so u_t = beta_t r)
 *   dv_t   = beta_t du                          dbeta_t = du . r
 *   G~     = G - beta_t k_t du^T                dk_t -= beta_t S~_t du
 *   dlog_alpha_t[c] = sum_j G~[c][j] S~_t[c][j]   (d alpha = G~ S_{t-1} per row; times alpha)
 *   G      = Diag(alpha_t) G~                   -> the gradient with respect to S_{t-1}
 *
 * and dS0 = G after the first token.  The states S_t are recomputed from checkpoints kept
 * every kSeg tokens of the forward pass, so memory stays at kSeg states per task.
 *
 * Layout as kda_oracle.c (packed tokens; q, k, log_alpha [T_total, H, dk]; v [T_total, H, dv];
 * beta [T_total, H]; S0 [N, H, dk, dv] or NULL), plus dO [T_total, H, dv] and dS_final
 * [N, H, dk, dv] or NULL.  Every input has its own element type code (fp64 / fp32 / bf16
 * bits), widened exactly.  Outputs are fp64 in full layout: dq, dk, dlog_alpha [T_total, H, dk],
 * dv [T_total, H, dv], dbeta [T_total, H], dS0 [N, H, dk, dv]; only the tasks' rows are written.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { KB_F64 = 0, KB_F32 = 1, KB_BF16 = 2 };
enum { kSeg = 64 };

static double wid(const void *p, int dt, int64_t i) {
    switch (dt) {
    case KB_F64:
        return ((const double *)p)[i];
    case KB_F32:
        return (double)((const float *)p)[i];
    case KB_BF16: {
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
    const void *q, *k, *v, *la, *beta, *S0, *dO, *dSf;
    int q_dt, k_dt, v_dt, la_dt, b_dt, s0_dt, do_dt, dsf_dt;
    const int64_t *cu;
    int64_t H, dk, dv;
    double scale;
    const int64_t *tasks;
    int64_t ntasks;
    double *dq, *dk_out, *dv_out, *dla, *dbeta, *dS0;
    int64_t next;
    pthread_mutex_t lock;
} bjob_t;

/* One forward token on S (in place): decay, look up, write.  Returns u in u_out (dv). */
static void fwd_token(const bjob_t *J, int64_t t, int64_t h, double *S, double *u_out) {
    const int64_t H = J->H, dk = J->dk, dv = J->dv;
    const int64_t bk = (t * H + h) * dk, bv = (t * H + h) * dv;
    for (int64_t c = 0; c < dk; ++c) {
        const double a = exp(wid(J->la, J->la_dt, bk + c));
        for (int64_t x = 0; x < dv; ++x) S[c * dv + x] *= a;
    }
    const double b = wid(J->beta, J->b_dt, t * H + h);
    for (int64_t x = 0; x < dv; ++x) {
        double r = wid(J->v, J->v_dt, bv + x);
        for (int64_t c = 0; c < dk; ++c) r -= S[c * dv + x] * wid(J->k, J->k_dt, bk + c);
        u_out[x] = b * r;
    }
    for (int64_t c = 0; c < dk; ++c) {
        const double kc = wid(J->k, J->k_dt, bk + c);
        for (int64_t x = 0; x < dv; ++x) S[c * dv + x] += kc * u_out[x];
    }
}

static void run_btask(bjob_t *J, int64_t j) {
    const int64_t n = J->tasks[2 * j], h = J->tasks[2 * j + 1];
    const int64_t H = J->H, dk = J->dk, dv = J->dv, DD = dk * dv;
    const int64_t t0 = J->cu[n], t1 = J->cu[n + 1], T = t1 - t0;
    const int64_t nseg = (T + kSeg - 1) / kSeg;
    double *ck = malloc(sizeof(double) * (size_t)((nseg > 0 ? nseg : 1) * DD));   /* S before each segment */
    double *St = malloc(sizeof(double) * (size_t)((kSeg + 1) * DD));             /* S_{t-1}, S_t in a segment */
    double *G = malloc(sizeof(double) * (size_t)DD);
    double *Gt = malloc(sizeof(double) * (size_t)DD);
    double *tmp = malloc(sizeof(double) * (size_t)(4 * (dk + dv)));
    double *u = tmp, *du = tmp + dv, *r = tmp + 2 * dv, *kt = tmp + 3 * dv, *qt = kt + dk;
    double *S = St;

    for (int64_t c = 0; c < DD; ++c)
        S[c] = J->S0 ? wid(J->S0, J->s0_dt, (n * H + h) * DD + c) : 0.0;
    for (int64_t sg = 0; sg < nseg; ++sg) {            /* forward: checkpoints */
        memcpy(ck + sg * DD, S, sizeof(double) * (size_t)DD);
        for (int64_t t = t0 + sg * kSeg; t < t1 && t < t0 + (sg + 1) * kSeg; ++t) fwd_token(J, t, h, S, u);
    }
    for (int64_t c = 0; c < DD; ++c)
        G[c] = J->dSf ? wid(J->dSf, J->dsf_dt, (n * H + h) * DD + c) : 0.0;

    for (int64_t sg = nseg - 1; sg >= 0; --sg) {
        const int64_t a0 = t0 + sg * kSeg, a1 = (a0 + kSeg < t1) ? a0 + kSeg : t1;
        memcpy(St, ck + sg * DD, sizeof(double) * (size_t)DD);          /* St[0] = S_{a0-1} */
        for (int64_t t = a0; t < a1; ++t) {
            memcpy(St + (t - a0 + 1) * DD, St + (t - a0) * DD, sizeof(double) * (size_t)DD);
            fwd_token(J, t, h, St + (t - a0 + 1) * DD, u);
        }
        for (int64_t t = a1 - 1; t >= a0; --t) {
            const double *Sp = St + (t - a0) * DD, *Sc = St + (t - a0 + 1) * DD;   /* S_{t-1}, S_t */
            const int64_t bk = (t * H + h) * dk, bv = (t * H + h) * dv;
            for (int64_t c = 0; c < dk; ++c) {
                kt[c] = wid(J->k, J->k_dt, bk + c);
                qt[c] = J->scale * wid(J->q, J->q_dt, bk + c);
            }
            const double b = wid(J->beta, J->b_dt, t * H + h);
            /* read-out: G += s q dO^T, dq = s S_t dO */
            for (int64_t c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int64_t x = 0; x < dv; ++x) {
                    const double g = wid(J->dO, J->do_dt, bv + x);
                    G[c * dv + x] += qt[c] * g;
                    acc += Sc[c * dv + x] * g;
                }
                J->dq[bk + c] = J->scale * acc;
            }
            /* S~ = Diag(alpha) S_{t-1}; r = v - S~^T k; u = beta r */
            for (int64_t c = 0; c < dk; ++c) {
                const double a = exp(wid(J->la, J->la_dt, bk + c));
                for (int64_t x = 0; x < dv; ++x) Gt[c * dv + x] = a * Sp[c * dv + x];    /* Gt holds S~ for now */
            }
            for (int64_t x = 0; x < dv; ++x) {
                double rr = wid(J->v, J->v_dt, bv + x);
                for (int64_t c = 0; c < dk; ++c) rr -= Gt[c * dv + x] * kt[c];
                r[x] = rr;
                u[x] = b * rr;
            }
            /* du = G^T k; dk = G u - beta S~ du; dv = beta du; dbeta = du . r */
            for (int64_t x = 0; x < dv; ++x) {
                double acc = 0.0;
                for (int64_t c = 0; c < dk; ++c) acc += G[c * dv + x] * kt[c];
                du[x] = acc;
            }
            double db = 0.0;
            for (int64_t x = 0; x < dv; ++x) {
                J->dv_out[bv + x] = b * du[x];
                db += du[x] * r[x];
            }
            J->dbeta[t * H + h] = db;
            for (int64_t c = 0; c < dk; ++c) {
                double acc = 0.0;
                for (int64_t x = 0; x < dv; ++x) acc += G[c * dv + x] * u[x] - b * Gt[c * dv + x] * du[x];
                J->dk_out[bk + c] = acc;
            }
            /* G~ = G - beta k du^T; dlog_alpha = rowsum(G~ * S~); G <- Diag(alpha) G~ */
            for (int64_t c = 0; c < dk; ++c) {
                const double a = exp(wid(J->la, J->la_dt, bk + c));
                double acc = 0.0;
                for (int64_t x = 0; x < dv; ++x) {
                    const double gt = G[c * dv + x] - b * kt[c] * du[x];
                    acc += gt * Gt[c * dv + x];
                    G[c * dv + x] = a * gt;
                }
                J->dla[bk + c] = acc;
            }
        }
    }
    for (int64_t c = 0; c < DD; ++c) J->dS0[(n * H + h) * DD + c] = G[c];
    free(ck);
    free(St);
    free(G);
    free(Gt);
    free(tmp);
}

static void *bworker(void *arg) {
    bjob_t *J = (bjob_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t j = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (j >= J->ntasks) break;
        run_btask(J, j);
    }
    return NULL;
}

/* Returns 0 on success, -1 on a bad argument. */
int kda_oracle_backward(const void *q, int q_dt, const void *k, int k_dt, const void *v, int v_dt,
                        const void *log_alpha, int la_dt, const void *beta, int b_dt, const void *S0,
                        int s0_dt, const void *dO, int do_dt, const void *dS_final, int dsf_dt,
                        const int64_t *cu_seqlens, int64_t N, int64_t H, int64_t dk, int64_t dv,
                        double scale, const int64_t *tasks, int64_t ntasks, double *dq, double *dk_out,
                        double *dv_out, double *dlog_alpha, double *dbeta, double *dS0, int nthreads) {
    if (!q || !k || !v || !log_alpha || !beta || !dO || !cu_seqlens || !tasks || !dq || !dk_out ||
        !dv_out || !dlog_alpha || !dbeta || !dS0)
        return -1;
    if (N <= 0 || H <= 0 || dk <= 0 || dv <= 0 || ntasks < 0) return -1;
    for (int64_t j = 0; j < ntasks; ++j) {
        const int64_t n = tasks[2 * j], h = tasks[2 * j + 1];
        if (n < 0 || n >= N || h < 0 || h >= H || cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    }
    bjob_t J = {q, k, v, log_alpha, beta, S0, dO, dS_final, q_dt, k_dt, v_dt, la_dt, b_dt, s0_dt,
                do_dt, dsf_dt, cu_seqlens, H, dk, dv, scale, tasks, ntasks, dq, dk_out, dv_out,
                dlog_alpha, dbeta, dS0, 0, PTHREAD_MUTEX_INITIALIZER};
    if (nthreads < 1) nthreads = 1;
    if (nthreads > ntasks) nthreads = ntasks > 0 ? (int)ntasks : 1;
    pthread_t *th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, bworker, &J);
    bworker(&J);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    return 0;
}
