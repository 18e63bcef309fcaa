/*
 * KDA forward oracle: plain, slow, fp64, host-only.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may build, load or call this file.  It shares
 * no code, header, table or constant with the CUDA library; the product path
 * never reaches it.
 *
 * What it computes, and where that is defined:
 *
 *   Kimi K3 technical-report digest (discuss.pytorch.kr, "Kimi K3 model
 *   weights and technical report"), section "Kimi Delta Attention: delta rule
 *   with a per-channel forget gate", state-update equation:
 *
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *       o_t = S_t^T q_t
 *
 *   with q_t, k_t in R^dk, v_t in R^dv, S_t in R^{dk x dv}, alpha_t in
 *   (0,1)^dk acting per key channel (rows of S), beta_t in (0,1) a scalar.
 *   The same digest, section "Bounded decay", gives alpha_t = exp(g_t) with
 *   the log-decay g_t the input here ("log_alpha").  The architecture page
 *   (digitalbourgeois.tistory.com, "Kimi K3 architecture") reads the update as
 *   forget (decay), erase (remove what overlaps the new key), write.
 *
 * The step below is that equation written out in those three moves:
 *       S' = Diag(exp g_t) S                 (forget)
 *       u  = S'^T k_t                         (what the key currently reads)
 *       S  = S' + beta_t k_t (v_t - u)^T      (erase + write; equals
 *                                              (I - b k k^T) S' + b k v^T)
 *       o_t = S^T q_t                         (read with the UPDATED state)
 * No 1/sqrt(dk) scale is applied to q: the equation shows none.
 *
 * Layouts: token-major [T_total][H][d] for q, k, v, g and out; beta is
 * [T_total][H]; states are [N][H][dk][dv] (key index major).  Sequences are
 * given by int64 offsets[N+1] into the token axis.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* One recurrence step on a single head.  S is [dk][dv], row-major. */
static void kda_step(double *S, int dk, int dv, const double *q, const double *k,
                     const double *v, const double *g, double beta, double *o,
                     double *u)
{
    /* forget: Diag(alpha_t) scales row i (key channel i) by exp(g_i) */
    for (int i = 0; i < dk; ++i) {
        const double a = exp(g[i]);
        double *row = S + (int64_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    /* u = S'^T k */
    for (int j = 0; j < dv; ++j) u[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        const double *row = S + (int64_t)i * dv;
        for (int j = 0; j < dv; ++j) u[j] += row[j] * ki;
    }
    /* erase + write: S += beta k (v - u)^T */
    for (int j = 0; j < dv; ++j) u[j] = beta * (v[j] - u[j]);
    for (int i = 0; i < dk; ++i) {
        const double ki = k[i];
        double *row = S + (int64_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] += ki * u[j];
    }
    /* read: o = S^T q with the updated S */
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double qi = q[i];
            const double *row = S + (int64_t)i * dv;
            for (int j = 0; j < dv; ++j) o[j] += row[j] * qi;
        }
    }
}

/*
 * One (sequence, head) chain.  Row t of q/k lives at q + t*qk_stride, and so
 * on for the other operands.  s0 may be NULL (zero initial state); out and
 * s_final may be NULL.
 */
void kda_oracle_chain(int64_t T, int dk, int dv,
                      const double *q, const double *k, int64_t qk_stride,
                      const double *v, int64_t v_stride,
                      const double *g, int64_t g_stride,
                      const double *beta, int64_t beta_stride,
                      const double *s0, double *out, int64_t out_stride,
                      double *s_final)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    if (s0) memcpy(S, s0, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);
    for (int64_t t = 0; t < T; ++t) {
        kda_step(S, dk, dv, q + t * qk_stride, k + t * qk_stride, v + t * v_stride,
                 g + t * g_stride, beta[t * beta_stride],
                 out ? out + t * out_stride : NULL, u);
    }
    if (s_final) memcpy(s_final, S, sizeof(double) * (size_t)dk * dv);
    free(S);
    free(u);
}

typedef struct {
    const double *q, *k, *v, *g, *beta, *init;
    double *out, *fin;
    const int64_t *offsets;
    int N, H, dk, dv;
    int64_t next;      /* shared work counter (chain index), guarded by mu */
    pthread_mutex_t mu;
} fwd_job;

static void *fwd_worker(void *arg)
{
    fwd_job *J = (fwd_job *)arg;
    const int64_t total = (int64_t)J->N * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const int64_t w = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (w >= total) break;
        const int n = (int)(w / J->H), h = (int)(w % J->H);
        const int64_t t0 = J->offsets[n], T = J->offsets[n + 1] - t0;
        const int64_t H = J->H, dk = J->dk, dv = J->dv;
        const int64_t sz = dk * dv;
        kda_oracle_chain(T, J->dk, J->dv,
                         J->q + (t0 * H + h) * dk, J->k + (t0 * H + h) * dk, H * dk,
                         J->v + (t0 * H + h) * dv, H * dv,
                         J->g + (t0 * H + h) * dk, H * dk,
                         J->beta + t0 * H + h, H,
                         J->init ? J->init + ((int64_t)n * H + h) * sz : NULL,
                         J->out ? J->out + (t0 * H + h) * dv : NULL, H * dv,
                         J->fin ? J->fin + ((int64_t)n * H + h) * sz : NULL);
    }
    return NULL;
}

/*
 * Whole forward over N packed sequences and H heads, threaded over
 * (sequence, head) chains.  Returns the number of threads used.
 */
int kda_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *g, const double *beta, const double *init_state,
                   double *out, double *final_state, int N, const int64_t *offsets,
                   int H, int dk, int dv, int nthreads)
{
    fwd_job J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.init = init_state;
    J.out = out; J.fin = final_state; J.offsets = offsets;
    J.N = N; J.H = H; J.dk = dk; J.dv = dv; J.next = 0;
    pthread_mutex_init(&J.mu, NULL);
    const int64_t chains = (int64_t)N * H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > chains) nthreads = chains > 0 ? (int)chains : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, fwd_worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return nthreads;
}

/*
 * One decode step for B independent sequences and H heads: the same step,
 * applied once to a resident state [B][H][dk][dv] that is updated in place.
 * q,k,g: [B][H][dk]; v,out: [B][H][dv]; beta: [B][H].
 */
void kda_oracle_decode_step(const double *q, const double *k, const double *v,
                            const double *g, const double *beta, double *state,
                            double *out, int B, int H, int dk, int dv)
{
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        kda_step(state + bh * dk * dv, dk, dv, q + bh * dk, k + bh * dk, v + bh * dv,
                 g + bh * dk, beta[bh], out + bh * dv, u);
    }
    free(u);
}
