/*
 * KDA oracle: plain fp64 CPU recurrence of Kimi Delta Attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the bench's CPU
 * baseline do. It shares no code, header or constant with the CUDA library.
 *
 * What it computes (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3,
 * eq. (1); the same update is restated as a constrained DPLR transition in
 * section 4):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with S_t in R^{dk x dv}, alpha_t = exp(log_alpha_t) in [0,1]^{dk} (one
 * forget rate per key channel, section 3), beta_t in [0,1] a per-token
 * scalar. The output is read from the state AFTER the token's update
 * (o_t = S_t^T q_t). There is no query scaling.
 *
 * Each step is written exactly as the formula reads, in this order:
 *   1. S <- Diag(alpha_t) S           (decay each key row i by alpha_t[i])
 *   2. u  = S^T k_t                   (what the decayed state recalls for k_t)
 *   3. S <- S + k_t (beta_t (v_t - u))^T
 *          which equals (I - beta k k^T) S + beta k v^T
 *   4. o_t = S^T q_t
 *
 * Sequences are packed token-major: token rows cu_seqlens[s] ..
 * cu_seqlens[s+1]-1 belong to sequence s. Heads are independent. Columns of
 * S (the dv index) are independent too, so the oracle can be run on a subset
 * of value columns by slicing v and S0; that is how large cases are sampled.
 *
 * Layouts (all row-major, all fp64):
 *   q, k, log_alpha  [n_tok][H][dk]
 *   v, o             [n_tok][H][dv]
 *   beta             [n_tok][H]
 *   S0, S_T          [n_seqs][H][dk][dv]   (S0 == NULL means zeros)
 *
 * Work is split over (sequence, head, block of 32 value columns) items on
 * n_threads POSIX threads (n_threads <= 0 means one per online core). A
 * column block runs the same four steps on its own columns of S only; the
 * columns never mix, so the split changes no arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define KDA_ORACLE_COL_BLOCK 32

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    double *o, *S_T;
    const int64_t *cu;
    int n_seqs, H, dk, dv, n_cb;
    long n_items;
    long next; /* atomic work counter */
    int status;
} kda_oracle_job;

static int run_item(kda_oracle_job *J, long item, double *S, double *a, double *u)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int cb = (int)(item % J->n_cb);
    const int h = (int)((item / J->n_cb) % H);
    const int s = (int)(item / ((long)J->n_cb * H));
    const int j0 = cb * KDA_ORACLE_COL_BLOCK;
    const int j1 = j0 + KDA_ORACLE_COL_BLOCK < dv ? j0 + KDA_ORACLE_COL_BLOCK : dv;
    const int nc = j1 - j0; /* S below holds columns j0..j1-1 only: S[i*nc + (j-j0)] */
    const int64_t t0 = J->cu[s], t1 = J->cu[s + 1];
    const size_t soff = ((size_t)s * H + h) * (size_t)dk * dv;

    for (int i = 0; i < dk; ++i)
        for (int j = j0; j < j1; ++j)
            S[(size_t)i * nc + (j - j0)] = J->S0 ? J->S0[soff + (size_t)i * dv + j] : 0.0;

    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = J->q + ((size_t)t * H + h) * dk;
        const double *kt = J->k + ((size_t)t * H + h) * dk;
        const double *lat = J->log_alpha + ((size_t)t * H + h) * dk;
        const double *vt = J->v + ((size_t)t * H + h) * dv + j0;
        const double bt = J->beta[(size_t)t * H + h];
        double *ot = J->o + ((size_t)t * H + h) * dv + j0;

        /* 1. decay: S <- Diag(alpha_t) S */
        for (int i = 0; i < dk; ++i) {
            a[i] = exp(lat[i]);
            double *row = S + (size_t)i * nc;
            for (int j = 0; j < nc; ++j) row[j] *= a[i];
        }
        /* 2. u = S^T k_t */
        for (int j = 0; j < nc; ++j) u[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double ki = kt[i];
            const double *row = S + (size_t)i * nc;
            for (int j = 0; j < nc; ++j) u[j] += ki * row[j];
        }
        /* 3. S <- S + k_t (beta_t (v_t - u))^T */
        for (int j = 0; j < nc; ++j) u[j] = bt * (vt[j] - u[j]);
        for (int i = 0; i < dk; ++i) {
            const double ki = kt[i];
            double *row = S + (size_t)i * nc;
            for (int j = 0; j < nc; ++j) row[j] += ki * u[j];
        }
        /* 4. o_t = S_t^T q_t */
        for (int j = 0; j < nc; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i) {
            const double qi = qt[i];
            const double *row = S + (size_t)i * nc;
            for (int j = 0; j < nc; ++j) ot[j] += qi * row[j];
        }
    }
    if (J->S_T)
        for (int i = 0; i < dk; ++i)
            for (int j = j0; j < j1; ++j)
                J->S_T[soff + (size_t)i * dv + j] = S[(size_t)i * nc + (j - j0)];
    return 0;
}

static void *worker(void *arg)
{
    kda_oracle_job *J = (kda_oracle_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * KDA_ORACLE_COL_BLOCK);
    double *a = (double *)malloc(sizeof(double) * (size_t)J->dk);
    double *u = (double *)malloc(sizeof(double) * KDA_ORACLE_COL_BLOCK);
    if (!S || !a || !u) {
        __atomic_store_n(&J->status, -2, __ATOMIC_RELAXED);
    } else {
        for (;;) {
            long item = __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED);
            if (item >= J->n_items) break;
            run_item(J, item, S, a, u);
        }
    }
    free(S);
    free(a);
    free(u);
    return NULL;
}

/* Number of threads the oracle uses for n_threads <= 0. */
int kda_oracle_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/*
 * Returns 0 on success, -1 on invalid arguments, -2 on allocation failure.
 */
int kda_oracle_fwd(const double *q, const double *k, const double *v,
                   const double *log_alpha, const double *beta, const double *S0,
                   double *o, double *S_T, const int64_t *cu_seqlens, int n_seqs,
                   int H, int dk, int dv, int n_threads)
{
    if (!q || !k || !v || !log_alpha || !beta || !o || !cu_seqlens) return -1;
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0) return -1;
    for (int s = 0; s < n_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    kda_oracle_job J;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;
    J.o = o; J.S_T = S_T; J.cu = cu_seqlens;
    J.n_seqs = n_seqs; J.H = H; J.dk = dk; J.dv = dv;
    J.n_cb = (dv + KDA_ORACLE_COL_BLOCK - 1) / KDA_ORACLE_COL_BLOCK;
    J.n_items = (long)n_seqs * H * J.n_cb;
    J.next = 0;
    J.status = 0;
    if (J.n_items == 0) return 0;

    int nt = n_threads > 0 ? n_threads : kda_oracle_default_threads();
    if (nt > J.n_items) nt = (int)J.n_items;
    if (nt <= 1) {
        worker(&J);
        return J.status;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nt);
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < nt; ++i) {
        if (pthread_create(&th[i], NULL, worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J.status;
}
