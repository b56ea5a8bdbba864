/*
 * Gated delta-rule oracle: a plain sequential fp64 loop over tokens.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes (the page "How the New Flash Models Work: Inside
 * GLM-5.3-Flash and Qwen3.8-Flash-Next", section "Linear attention: a
 * fixed-size memory in place of the cache", the Gated DeltaNet equation and
 * the Kimi Delta Attention equation):
 *
 *     S_t = S_{t-1} D_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t,
 *
 * with S_t a d_v x d_k matrix per (sequence, head), and D_t = alpha_t I
 * (scalar gate, Gated DeltaNet) or D_t = Diag(alpha_t) (one gate per key
 * channel, Kimi Delta Attention).  The gate arrives as its logarithm
 * g_t = log(alpha_t) <= 0, so alpha_t = exp(g_t); g = -inf is a hard reset.
 *
 * Each token is applied in the order the equation is written: the decay
 * multiplies S_{t-1} first, the erase term (I - beta k k^T) then acts on the
 * decayed state, the write beta v k^T is added, and the output reads the
 * post-update state S_t.  Expanding the product,
 *
 *     s   = S_{t-1} D_t                     (column j scaled by alpha_t[j])
 *     u   = beta_t (v_t - s k_t)
 *     S_t = s + u k_t^T
 *     o_t = S_t q_t
 *
 * which is the same matrix as the equation because
 * s (I - beta k k^T) + beta v k^T = s + beta (v - s k) k^T.
 *
 * No scale is applied to q (the pages give none).  Every sequence starts from
 * its own initial state (or zero) and the final state after its last token is
 * returned; an empty sequence returns its initial state unchanged.
 *
 * Layouts (all row-major, fp64): q, k [total_T][H_qk][d_k]; v, o
 * [total_T][H][d_v]; g [total_T][H] (scalar mode) or [total_T][H][d_k]
 * (channel mode); beta [total_T][H]; h0, final [num_seqs][H][d_v][d_k];
 * cu_seqlens [num_seqs + 1] int64, 0 = cu[0] <= ... <= cu[num_seqs] = total_T.
 *
 * Head mapping: H value heads each own a state; the query/key heads may be
 * fewer (H_qk dividing H), each shared by H / H_qk consecutive value heads,
 * value head h reading query/key head h / (H / H_qk).  This is the grouping
 * of the Qwen Gated DeltaNet layer (16 query-key heads, 48 value heads;
 * page "Qwen3.8-Flash-Next and GLM-5.3-Flash ...", section "Gated DeltaNet
 * carries most of the sequence").  H_qk = H is the plain one-to-one case.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *h0;
    const int64_t *cu;
    int64_t num_seqs, H, H_qk, dk, dv;
    int channel_gate;
    double *o, *final_state;
    int64_t next;                 /* next (sequence, head) pair to take */
    pthread_mutex_t lock;
} oracle_job;

/* One (sequence n, head h) pair: the token loop written out. */
static void run_pair(const oracle_job *J, int64_t n, int64_t h, double *S, double *u,
                     double *a)
{
    const int64_t H = J->H, dk = J->dk, dv = J->dv;
    const int64_t hq = h / (H / J->H_qk);           /* query/key head of value head h */
    const int64_t SS = dv * dk;
    double *Sfin = J->final_state ? J->final_state + (n * H + h) * SS : NULL;

    if (J->h0)
        memcpy(S, J->h0 + (n * H + h) * SS, sizeof(double) * (size_t)SS);
    else
        memset(S, 0, sizeof(double) * (size_t)SS);

    for (int64_t t = J->cu[n]; t < J->cu[n + 1]; ++t) {
        const double *qt = J->q + (t * J->H_qk + hq) * dk;
        const double *kt = J->k + (t * J->H_qk + hq) * dk;
        const double *vt = J->v + (t * H + h) * dv;
        const double bt = J->beta[t * H + h];
        double *ot = J->o + (t * H + h) * dv;

        /* s = S_{t-1} D_t */
        if (J->channel_gate) {
            const double *gt = J->g + (t * H + h) * dk;
            for (int64_t j = 0; j < dk; ++j)
                a[j] = exp(gt[j]);
        } else {
            const double alpha = exp(J->g[t * H + h]);
            for (int64_t j = 0; j < dk; ++j)
                a[j] = alpha;
        }
        for (int64_t r = 0; r < dv; ++r)
            for (int64_t j = 0; j < dk; ++j)
                S[r * dk + j] *= a[j];
        /* u = beta (v - s k) */
        for (int64_t r = 0; r < dv; ++r) {
            double x = 0.0;
            for (int64_t j = 0; j < dk; ++j)
                x += S[r * dk + j] * kt[j];
            u[r] = bt * (vt[r] - x);
        }
        /* S_t = s + u k^T */
        for (int64_t r = 0; r < dv; ++r)
            for (int64_t j = 0; j < dk; ++j)
                S[r * dk + j] += u[r] * kt[j];
        /* o_t = S_t q_t */
        for (int64_t r = 0; r < dv; ++r) {
            double y = 0.0;
            for (int64_t j = 0; j < dk; ++j)
                y += S[r * dk + j] * qt[j];
            ot[r] = y;
        }
    }
    if (Sfin)
        memcpy(Sfin, S, sizeof(double) * (size_t)SS);
}

static void *worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)(J->dv * J->dk));
    double *u = (double *)malloc(sizeof(double) * (size_t)J->dv);
    double *a = (double *)malloc(sizeof(double) * (size_t)J->dk);
    if (!S || !u || !a) {
        free(S);
        free(u);
        free(a);
        return (void *)1;
    }
    const int64_t pairs = J->num_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t p = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (p >= pairs)
            break;
        run_pair(J, p / J->H, p % J->H, S, u, a);
    }
    free(S);
    free(u);
    free(a);
    return NULL;
}

/*
 * Runs the recurrence for every (sequence, head) pair with `nthreads` POSIX
 * threads (pairs are independent).  h0 and final_state may be NULL.
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
int gdr_oracle_run(const double *q, const double *k, const double *v,
                   const double *g, const double *beta, const double *h0,
                   const int64_t *cu_seqlens, int64_t num_seqs, int64_t H,
                   int64_t H_qk, int64_t d_k, int64_t d_v, int channel_gate, double *o,
                   double *final_state, int nthreads)
{
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !o || num_seqs < 0 ||
        H < 0 || H_qk < 1 || d_k < 1 || d_v < 1 || (H > 0 && H % H_qk != 0))
        return -1;
    for (int64_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n] || cu_seqlens[n] < 0)
            return -1;
    if (nthreads < 1)
        nthreads = 1;

    oracle_job J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.h0 = h0;
    J.cu = cu_seqlens; J.num_seqs = num_seqs; J.H = H; J.H_qk = H_qk; J.dk = d_k; J.dv = d_v;
    J.channel_gate = channel_gate ? 1 : 0;
    J.o = o; J.final_state = final_state; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);

    int rc = 0;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!tid) {
        pthread_mutex_destroy(&J.lock);
        return -2;
    }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&tid[i], NULL, worker, &J) != 0)
            break;
        ++started;
    }
    if (started == 0) {
        if (worker(&J) != NULL)
            rc = -2;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(tid[i], &ret);
        if (ret != NULL)
            rc = -2;
    }
    free(tid);
    pthread_mutex_destroy(&J.lock);
    return rc;
}
