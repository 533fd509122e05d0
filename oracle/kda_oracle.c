/*
 * KDA oracle: plain, slow, fp64 CPU reference for the Kimi Delta Attention
 * recurrence.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this; the product path never does.
 * It shares no code, header or table with the CUDA path.
 *
 * What it computes (one (sequence n, head h) unit at a time, tokens in order):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * This is the delta rule with per-channel retention that the pages describe
 * in words: a fixed-size per-head state that "forgets" (per-channel decay,
 * then the delta-rule erase along k_t) and "writes" (beta_t k_t v_t^T), with
 * the per-step log-decay bounded below at -5.  Sources:
 *   - neurohive.io, "Kimi K3 ... overview", section "Sequence length: hybrid
 *     KDA and Gated MLA attention" (delta rule = forget old + write new;
 *     linear attention with a fixed-size recurrent state; log-decay bounded
 *     from below at -5).
 *   - best.xiaohu.ai, "Kimi K3 tech report", section "Sequence length:
 *     replacing most attention layers with fixed-size memory" (older context
 *     decays gradually across channels; constant memory footprint).
 *
 * The step is evaluated in the algebraically expanded form
 *     A = Diag(a) S_{t-1},  a_c = exp(max(g_t[c], -5))
 *     S_t = A + beta_t k_t (v_t - A^T k_t)^T
 * which equals the product form above exactly in real arithmetic:
 *     (I - b k k^T) A + b k v^T = A + b k (v - A^T k)^T.
 * The clamp max(g, -5) is the library's reading of the bound (a no-op on
 * every input that already satisfies g >= -5); g > 0 is left as given.
 *
 * Layout: rows are tokens of the packed sequence dimension.
 *   q, k, g : [rows, H, dk]    v : [rows, H, dv]    beta : [rows, H]
 *   o       : [rows, H, dv]
 *   state_in / state_out : [N, H, dk, dv] (row c = key channel, col j = value channel)
 *   sequence n owns rows cu_seqlens[n] .. cu_seqlens[n+1]-1.
 * state_in may be NULL (zero initial state); state_out may be NULL.
 * Work is split over (n, h) units with POSIX threads; each unit is
 * independent, so the thread count changes nothing in the result.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *state_in;
    const int64_t *cu_seqlens;
    int N, H, dk, dv;
    double *o, *state_out;
    int next_unit;          /* shared work counter (protected by lock) */
    pthread_mutex_t lock;
    int status;
} oracle_job;

/* One (n, h) unit: the token recurrence, fp64 throughout. */
static int run_unit(const oracle_job *J, int n, int h, double *S, double *A_kT)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int64_t t0 = J->cu_seqlens[n], t1 = J->cu_seqlens[n + 1];
    const size_t sdim = (size_t)dk * (size_t)dv;

    if (J->state_in)
        memcpy(S, J->state_in + ((size_t)n * H + h) * sdim, sdim * sizeof(double));
    else
        memset(S, 0, sdim * sizeof(double));

    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = J->q + ((size_t)t * H + h) * dk;
        const double *kt = J->k + ((size_t)t * H + h) * dk;
        const double *gt = J->g + ((size_t)t * H + h) * dk;
        const double *vt = J->v + ((size_t)t * H + h) * dv;
        const double bt = J->beta[(size_t)t * H + h];
        double *ot = J->o + ((size_t)t * H + h) * dv;

        /* decay: S <- Diag(a) S, a_c = exp(max(g_c, -5)) */
        for (int c = 0; c < dk; ++c) {
            const double gc = gt[c] < -5.0 ? -5.0 : gt[c];
            const double a = exp(gc);
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] *= a;
        }
        /* prediction p = S^T k (S already decayed) */
        for (int j = 0; j < dv; ++j) A_kT[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double kc = kt[c];
            const double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) A_kT[j] += row[j] * kc;
        }
        /* delta-rule write: S <- S + beta k (v - p)^T */
        for (int j = 0; j < dv; ++j) A_kT[j] = bt * (vt[j] - A_kT[j]);
        for (int c = 0; c < dk; ++c) {
            const double kc = kt[c];
            double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) row[j] += kc * A_kT[j];
        }
        /* readout o_t = S_t^T q_t (post-update state) */
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double qc = qt[c];
            const double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) ot[j] += row[j] * qc;
        }
    }
    if (J->state_out)
        memcpy(J->state_out + ((size_t)n * H + h) * sdim, S, sdim * sizeof(double));
    return 0;
}

static void *worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *S = (double *)malloc((size_t)J->dk * J->dv * sizeof(double));
    double *tmp = (double *)malloc((size_t)J->dv * sizeof(double));
    if (!S || !tmp) {
        pthread_mutex_lock(&J->lock);
        J->status = -2;
        pthread_mutex_unlock(&J->lock);
        free(S);
        free(tmp);
        return NULL;
    }
    const int units = J->N * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= units) break;
        run_unit(J, u / J->H, u % J->H, S, tmp);
    }
    free(S);
    free(tmp);
    return NULL;
}

/*
 * Entry point.  Returns 0 on success, -1 on bad arguments, -2 on allocation
 * failure.  n_threads <= 0 means one thread.
 */
int kda_oracle_recurrence(const double *q, const double *k, const double *v,
                          const double *g, const double *beta,
                          const double *state_in, const int64_t *cu_seqlens,
                          int N, int H, int dk, int dv,
                          double *o, double *state_out, int n_threads)
{
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !o) return -1;
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int n = 0; n < N; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;

    oracle_job J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.state_in = state_in;
    J.cu_seqlens = cu_seqlens;
    J.N = N; J.H = H; J.dk = dk; J.dv = dv;
    J.o = o; J.state_out = state_out;
    J.next_unit = 0;
    J.status = 0;
    pthread_mutex_init(&J.lock, NULL);

    if (n_threads <= 1) {
        worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
        if (!th) { pthread_mutex_destroy(&J.lock); return -2; }
        int started = 0;
        for (int i = 0; i < n_threads; ++i)
            if (pthread_create(&th[i], NULL, worker, &J) == 0) ++started;
        if (started == 0) worker(&J);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return J.status;
}
