/*
 * KDA oracle, backward: plain, slow, fp64, token-by-token reverse pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests do.  It shares no code, header, table or
 * helper with the CUDA library, nor with the forward oracle's file.
 *
 * Forward (per head; S_0 = h0, or zero when h0 is NULL), for t = 1..T:
 *   S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T,
 *   o_t = S_t^T q_t,
 * the gated delta rule of Kimi Delta Attention ("T11E1: K3 tech report"
 * transcript, the KDA turn; "Kimi K3 goes trillion-scale with sparse MoE
 * efficiency" subtitles, cue 14).  The pages give no backward pass; this
 * file is the reverse-mode derivative of that recurrence, taken step by step
 * through its rank-1 form
 *   Sd = Diag(a) S_{t-1}, a = exp(g_t)     (forget)
 *   p  = Sd^T k_t                          (recall)
 *   u  = beta_t (v_t - p)                  (delta-rule correction)
 *   S_t = Sd + k_t u^T                     (write)
 *   o_t = S_t^T q_t                        (read)
 * For a scalar loss with dL/do_t = dO_t and dL/dS_T = dhT, walking t from T
 * down to 1 with dS = dL/dS_t (dS = dhT before the first step back):
 *   dq_t  = S_t dO_t                  dS  += q_t dO_t^T
 *   dk_t  = dS u                      du   = dS^T k_t
 *   dbeta_t = du . (v_t - p)          dv_t = beta_t du
 *   dp    = -beta_t du                dSd  = dS + k_t dp^T
 *   dk_t += Sd dp                     dg_t[i] = sum_j dSd[i][j] Sd[i][j]
 *   dS    = Diag(a) dSd               (this is dL/dS_{t-1})
 * and dh0 = dS after the last step back.  (dg uses Sd = a * S_{t-1}: the
 * derivative of exp(g) is exp(g).)
 *
 * States are needed in reverse order.  They are kept at every CKPT-th token
 * in the forward sweep and recomputed one segment at a time going back, so
 * the memory per head is (T/CKPT + CKPT) states.
 *
 * Parity pins (tests, not this file): central finite differences of the
 * forward oracle, reverse-mode autograd of an independently written forward
 * loop, the single-token closed form, the beta = 0 closed form, the exact
 * transpose identity in (v, h0), and the split/resume identity of the
 * backward chain.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#include <unistd.h>

#define CKPT 64

/* One forward step in place: S <- S_t from S_{t-1}.  When Sd, p, u are not
 * NULL they receive the decayed state, the recall and the correction. */
static void step_fwd(int dk, int dv, const double* qt, const double* kt,
                     const double* vt, const double* gt, double bt,
                     double* S, double* Sd, double* p, double* u)
{
    (void)qt;
    for (int i = 0; i < dk; ++i) {
        const double a = exp(gt[i]);
        double* row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    if (Sd) memcpy(Sd, S, sizeof(double) * (size_t)dk * dv);
    for (int j = 0; j < dv; ++j) p[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double* row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) p[j] += row[j] * kt[i];
    }
    for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - p[j]);
    for (int i = 0; i < dk; ++i) {
        double* row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] += kt[i] * u[j];
    }
}

/* One head.  Layout (all contiguous, row-major):
 *   q, k, g        : [T][dk]     v : [T][dv]     beta : [T]
 *   h0             : [dk][dv] or NULL (zero state)
 *   dO             : [T][dv] or NULL (no loss on the outputs)
 *   dhT            : [dk][dv] or NULL (no loss on the final state)
 *   dq, dk_, dg    : [T][dk]     dv_ : [T][dv]   dbeta : [T]
 *   dh0            : [dk][dv]
 * Returns 0, or -1 when scratch memory cannot be obtained. */
int kda_oracle_head_bwd(int64_t T, int dk, int dv,
                        const double* q, const double* k, const double* v,
                        const double* g, const double* beta, const double* h0,
                        const double* dO, const double* dhT,
                        double* dq, double* dk_, double* dv_, double* dg,
                        double* dbeta, double* dh0)
{
    const size_t st = (size_t)dk * dv;
    const int64_t n_ck = (T + CKPT - 1) / CKPT;
    double* ck = (double*)malloc(sizeof(double) * st * (size_t)(n_ck > 0 ? n_ck : 1));
    double* seg = (double*)malloc(sizeof(double) * st * CKPT);   /* S_{t-1} per token */
    double* work = (double*)malloc(sizeof(double) * (3 * st + 4 * (size_t)dv));
    if (!ck || !seg || !work) {
        free(ck); free(seg); free(work);
        return -1;
    }
    double* S = work;          /* running state */
    double* Sd = S + st;       /* decayed state of the current step */
    double* dS = Sd + st;      /* dL/dS_t */
    double* p = dS + st;
    double* u = p + dv;
    double* du = u + dv;
    double* dp = du + dv;

    /* forward sweep: keep the state before every CKPT-th token */
    if (h0) memcpy(S, h0, sizeof(double) * st);
    else memset(S, 0, sizeof(double) * st);
    for (int64_t t = 0; t < T; ++t) {
        if (t % CKPT == 0) memcpy(ck + (size_t)(t / CKPT) * st, S, sizeof(double) * st);
        step_fwd(dk, dv, q + t * dk, k + t * dk, v + t * dv, g + t * dk, beta[t],
                 S, NULL, p, u);
    }

    /* reverse sweep, one checkpoint segment at a time */
    if (dhT) memcpy(dS, dhT, sizeof(double) * st);
    else memset(dS, 0, sizeof(double) * st);
    for (int64_t c = n_ck - 1; c >= 0; --c) {
        const int64_t t0 = c * CKPT;
        const int64_t t1 = (t0 + CKPT < T) ? t0 + CKPT : T;
        memcpy(S, ck + (size_t)c * st, sizeof(double) * st);
        for (int64_t t = t0; t < t1; ++t) {
            memcpy(seg + (size_t)(t - t0) * st, S, sizeof(double) * st);
            step_fwd(dk, dv, q + t * dk, k + t * dk, v + t * dv, g + t * dk, beta[t],
                     S, NULL, p, u);
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const double* qt = q + t * dk;
            const double* kt = k + t * dk;
            const double* vt = v + t * dv;
            const double* gt = g + t * dk;
            const double bt = beta[t];
            /* rebuild S_{t-1} -> (Sd, p, u, S_t) */
            memcpy(S, seg + (size_t)(t - t0) * st, sizeof(double) * st);
            step_fwd(dk, dv, qt, kt, vt, gt, bt, S, Sd, p, u);
            double* dqt = dq + t * dk;
            double* dkt = dk_ + t * dk;
            double* dvt = dv_ + t * dv;
            double* dgt = dg + t * dk;
            /* read: o_t = S_t^T q_t */
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                if (dO) {
                    const double* row = S + (size_t)i * dv;
                    for (int j = 0; j < dv; ++j) acc += row[j] * dO[t * dv + j];
                }
                dqt[i] = acc;
            }
            if (dO) {
                for (int i = 0; i < dk; ++i) {
                    double* row = dS + (size_t)i * dv;
                    for (int j = 0; j < dv; ++j) row[j] += qt[i] * dO[t * dv + j];
                }
            }
            /* write: S_t = Sd + k u^T */
            for (int i = 0; i < dk; ++i) {
                const double* row = dS + (size_t)i * dv;
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += row[j] * u[j];
                dkt[i] = acc;
            }
            for (int j = 0; j < dv; ++j) du[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double* row = dS + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) du[j] += row[j] * kt[i];
            }
            /* correction: u = beta (v - p) */
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {
                db += du[j] * (vt[j] - p[j]);
                dvt[j] = bt * du[j];
                dp[j] = -bt * du[j];
            }
            dbeta[t] = db;
            /* recall: p = Sd^T k  (dSd = dS + k dp^T, held in dS) */
            for (int i = 0; i < dk; ++i) {
                const double* row = Sd + (size_t)i * dv;
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += row[j] * dp[j];
                dkt[i] += acc;
            }
            for (int i = 0; i < dk; ++i) {
                double* row = dS + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) row[j] += kt[i] * dp[j];
            }
            /* forget: Sd = Diag(exp g) S_{t-1} */
            for (int i = 0; i < dk; ++i) {
                const double* srow = Sd + (size_t)i * dv;
                double* row = dS + (size_t)i * dv;
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += row[j] * srow[j];
                dgt[i] = acc;
                const double a = exp(gt[i]);
                for (int j = 0; j < dv; ++j) row[j] *= a;
            }
        }
    }
    memcpy(dh0, dS, sizeof(double) * st);
    free(ck); free(seg); free(work);
    return 0;
}

/* ---- many heads on host threads: one head is one unit of work ---------- */

typedef struct {
    int64_t n, T;
    int dk, dv;
    const double *q, *k, *v, *g, *beta, *h0, *dO, *dhT;
    double *dq, *dk_, *dv_, *dg, *dbeta, *dh0;
    int64_t next;
    pthread_mutex_t lock;
    int status;
} bwd_job;

static void* bwd_worker(void* arg)
{
    bwd_job* J = (bwd_job*)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t h = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (h >= J->n) break;
        const int64_t T = J->T;
        const int dk = J->dk, dv = J->dv;
        const int64_t sz = (int64_t)dk * dv;
        const int rc = kda_oracle_head_bwd(
            T, dk, dv,
            J->q + h * T * dk, J->k + h * T * dk, J->v + h * T * dv,
            J->g + h * T * dk, J->beta + h * T,
            J->h0 ? J->h0 + h * sz : NULL,
            J->dO ? J->dO + h * T * dv : NULL,
            J->dhT ? J->dhT + h * sz : NULL,
            J->dq + h * T * dk, J->dk_ + h * T * dk, J->dv_ + h * T * dv,
            J->dg + h * T * dk, J->dbeta + h * T, J->dh0 + h * sz);
        if (rc) {
            pthread_mutex_lock(&J->lock);
            J->status = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/* n independent heads stacked on a leading axis, each laid out as in
 * kda_oracle_head_bwd.  n_threads <= 0 uses every online core.
 * Returns 0 or a negative code. */
int kda_oracle_heads_bwd(int64_t n, int64_t T, int dk, int dv,
                         const double* q, const double* k, const double* v,
                         const double* g, const double* beta, const double* h0,
                         const double* dO, const double* dhT,
                         double* dq, double* dk_, double* dv_, double* dg,
                         double* dbeta, double* dh0, int n_threads)
{
    if (n < 0 || T < 0 || dk <= 0 || dv <= 0 || !dh0) return -2;
    if (T > 0 && (!q || !k || !v || !g || !beta || !dq || !dk_ || !dv_ || !dg || !dbeta))
        return -2;
    if (n_threads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = c > 0 ? (int)c : 1;
    }
    if (n_threads > n) n_threads = n > 0 ? (int)n : 1;
    bwd_job J = {n, T, dk, dv, q, k, v, g, beta, h0, dO, dhT,
                 dq, dk_, dv_, dg, dbeta, dh0, 0, PTHREAD_MUTEX_INITIALIZER, 0};
    if (n_threads == 1) {
        bwd_worker(&J);
        return J.status;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, bwd_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) bwd_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J.status;
}
