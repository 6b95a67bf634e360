/*
 * KDA oracle: plain, slow, fp64, token-by-token CPU recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library and includes none of its files.
 *
 * What it computes (per head, S starts at h0, or at zero when h0 is NULL):
 *   S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *   o_t = S_t^T q_t
 * with S a d_k x d_v matrix.  Sources:
 *   - "T11E1: K3 tech report" podcast transcript (williamliu.ai), the turn on
 *     Kimi Delta Attention: a recurrent state updated with a learned write
 *     strength (beta) and channel-wise forgetting (g, one log-decay per key
 *     channel), and the next turn: log-decay bounded below by -5.
 *   - "Kimi K3 goes trillion-scale with sparse MoE efficiency" subtitles
 *     (podcast.do-not-panic.com), cue 14: a delta-rule recurrence with a
 *     channel-wise forget gate and one fixed-size recurrent state.
 *   - "177: Kimi K3 in Detail" episode notes (zjai.club), Deep dive section
 *     15: delta rule, channel-wise forget gates, lower bound on retention.
 * The product form above is evaluated in its rank-1 order, which is the
 * same expression multiplied out:
 *   S <- Diag(exp g_t) S                 (channel-wise forgetting, rows of S)
 *   p  = S^T k_t                          (what the decayed state recalls at k_t)
 *   u  = beta_t (v_t - p)                 (delta-rule correction)
 *   S <- S + k_t u^T                      (write)
 *   o_t = S^T q_t                         (read the updated state)
 * There is no output scale (no 1/sqrt(d_k)) and no normalisation here: q and
 * k arrive normalised as a precondition.
 *
 * Parity pins (tests, not this file): the single-token closed form, beta = 0
 * (pure decay) closed form, g = 0 (plain delta rule), the dense d_k x d_k
 * product form for short sequences, an independent chunked (WY) formulation,
 * associative-memory recall with orthonormal keys, linearity and the
 * split/resume identity, and a hand-derived worked example.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* One head.  Layout (all contiguous, row-major):
 *   q, k, g : [T][dk]     v : [T][dv]     beta : [T]
 *   h0      : [dk][dv] or NULL (zero state)
 *   o       : [T][dv]     (may be NULL: outputs not wanted)
 *   hT      : [dk][dv]    (must not be NULL; receives the final state)
 * Returns 0, or -1 when scratch memory cannot be obtained. */
int kda_oracle_head(int64_t T, int dk, int dv,
                    const double* q, const double* k, const double* v,
                    const double* g, const double* beta, const double* h0,
                    double* o, double* hT)
{
    double* S = hT;
    double* p = (double*)malloc(sizeof(double) * (size_t)dv * 2);
    if (!p) return -1;
    double* u = p + dv;
    if (h0) {
        if (h0 != S) memcpy(S, h0, sizeof(double) * (size_t)dk * dv);
    } else {
        memset(S, 0, sizeof(double) * (size_t)dk * dv);
    }
    for (int64_t t = 0; t < T; ++t) {
        const double* qt = q + t * dk;
        const double* kt = k + t * dk;
        const double* vt = v + t * dv;
        const double* gt = g + t * dk;
        const double bt = beta[t];
        /* forget: row i of S scaled by exp(g_t[i]) */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(gt[i]);
            double* row = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
        /* recall p = S^T k */
        for (int j = 0; j < dv; ++j) p[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double ki = kt[i];
            const double* row = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) p[j] += row[j] * ki;
        }
        /* delta-rule correction and write */
        for (int j = 0; j < dv; ++j) u[j] = bt * (vt[j] - p[j]);
        for (int i = 0; i < dk; ++i) {
            const double ki = kt[i];
            double* row = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) row[j] += ki * u[j];
        }
        /* read the updated state */
        if (o) {
            double* ot = o + t * dv;
            for (int j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                const double qi = qt[i];
                const double* row = S + (size_t)i * dv;
                for (int j = 0; j < dv; ++j) ot[j] += row[j] * qi;
            }
        }
    }
    free(p);
    return 0;
}

/* ---- many heads on host threads: one head is one unit of work ---------- */

typedef struct {
    int64_t n, T;
    int dk, dv;
    const double *q, *k, *v, *g, *beta, *h0;
    double *o, *hT;
    int64_t next;          /* shared work counter */
    pthread_mutex_t lock;
    int status;
} oracle_job;

static void* oracle_worker(void* arg)
{
    oracle_job* J = (oracle_job*)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t h = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (h >= J->n) break;
        const int64_t T = J->T;
        const int dk = J->dk, dv = J->dv;
        const int rc = kda_oracle_head(
            T, dk, dv,
            J->q + h * T * dk, J->k + h * T * dk, J->v + h * T * dv,
            J->g + h * T * dk, J->beta + h * T,
            J->h0 ? J->h0 + h * (int64_t)dk * dv : NULL,
            J->o ? J->o + h * T * dv : NULL,
            J->hT + h * (int64_t)dk * dv);
        if (rc) {
            pthread_mutex_lock(&J->lock);
            J->status = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/* n independent heads, each laid out as in kda_oracle_head and stacked on a
 * leading axis: q [n][T][dk], ..., beta [n][T], h0/hT [n][dk][dv], o [n][T][dv].
 * n_threads <= 0 uses every online core.  Returns 0 or a negative code. */
int kda_oracle_heads(int64_t n, int64_t T, int dk, int dv,
                     const double* q, const double* k, const double* v,
                     const double* g, const double* beta, const double* h0,
                     double* o, double* hT, int n_threads)
{
    if (n < 0 || T < 0 || dk <= 0 || dv <= 0 || !hT) return -2;
    if (T > 0 && (!q || !k || !v || !g || !beta)) return -2;
    if (n_threads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        n_threads = c > 0 ? (int)c : 1;
    }
    if (n_threads > n) n_threads = n > 0 ? (int)n : 1;
    oracle_job J = {n, T, dk, dv, q, k, v, g, beta, h0, o, hT, 0,
                    PTHREAD_MUTEX_INITIALIZER, 0};
    if (n_threads == 1) {
        oracle_worker(&J);
        return J.status;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) return -1;
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, oracle_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) oracle_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J.status;
}

/* Number of online host cores, as the thread pool above sees them. */
int kda_oracle_num_cores(void)
{
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}
