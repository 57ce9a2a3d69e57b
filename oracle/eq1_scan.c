/*
 * Oracle (test infrastructure only): sequential fp64 Gated DeltaNet recurrence.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline leg load this
 * file's library.  It shares no code with the CUDA path.
 *
 * What it computes -- Tail-Replay (arXiv 2608.30310) reading notes, section 2.3,
 * Eq. (1):
 *
 *     S_i = T_i S_{i-1} + beta_i v_i k_i^T,     T_i = alpha_i (I - beta_i k_i k_i^T)
 *
 * The pages leave the axis layout of the state open (same section, the remark
 * after Eq. (1)).  Reading used here: the state is stored as M = S^T, a
 * d_k x d_v matrix (row-major [d_k][d_v]); in that layout the key-space operator
 * T_i (d_k x d_k, symmetric) multiplies from the left exactly as printed:
 *
 *     M_i = T_i M_{i-1} + beta_i k_i v_i^T
 *         = alpha_i (M_{i-1} - beta_i k_i (k_i^T M_{i-1})) + beta_i k_i v_i^T
 *
 * The readout is not defined on the pages.  Reading used here: o_i = scale *
 * M_i^T q_i, taken after the update of token i (scale = 1 in every workload).
 *
 * One call covers a packed batch of sequences (cu_seqlens, N+1 offsets) and
 * heads.  Every (sequence, head) pair starts from S0 (or from zero when S0 is
 * NULL: the zero start of the tail replay, reading notes section 2.2 step 2)
 * and is stepped token by token in order.  Independent (sequence, head) pairs
 * run on separate threads; nothing inside a pair is reordered.
 *
 * Layouts (all float64, row-major):
 *   q, k        [T, H, d_k]
 *   v           [T, H, d_v]
 *   log_alpha   [T, H]      (alpha = exp(log_alpha))
 *   beta        [T, H]
 *   S0, S_final [N, H, d_k, d_v]   (M = S^T layout)
 *   o           [T, H, d_v]        (may be NULL)
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t n_seqs, n_heads, d_k, d_v;
    const int64_t *cu_seqlens;
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    double scale;
    double *o, *S_final;
    int64_t next_unit;      /* shared work counter */
    pthread_mutex_t lock;
} scan_job;

static void scan_one(const scan_job *J, int64_t seq, int64_t head, double *w) {
    const int64_t H = J->n_heads, dk = J->d_k, dv = J->d_v;
    double *M = J->S_final + (seq * H + head) * dk * dv;
    if (J->S0)
        memcpy(M, J->S0 + (seq * H + head) * dk * dv, sizeof(double) * dk * dv);
    else
        memset(M, 0, sizeof(double) * dk * dv);

    for (int64_t t = J->cu_seqlens[seq]; t < J->cu_seqlens[seq + 1]; ++t) {
        const double *kt = J->k + (t * H + head) * dk;
        const double *vt = J->v + (t * H + head) * dv;
        const double alpha = exp(J->log_alpha[t * H + head]);
        const double beta = J->beta[t * H + head];

        /* w = k_t^T M_{t-1}  (a row over the d_v columns) */
        for (int64_t j = 0; j < dv; ++j) w[j] = 0.0;
        for (int64_t d = 0; d < dk; ++d) {
            const double kd = kt[d];
            const double *Md = M + d * dv;
            for (int64_t j = 0; j < dv; ++j) w[j] += kd * Md[j];
        }
        /* M_t = alpha (M_{t-1} - beta k (k^T M_{t-1})) + beta k v^T */
        for (int64_t d = 0; d < dk; ++d) {
            const double kd = kt[d];
            double *Md = M + d * dv;
            for (int64_t j = 0; j < dv; ++j)
                Md[j] = alpha * (Md[j] - beta * kd * w[j]) + beta * kd * vt[j];
        }
        /* o_t = scale * M_t^T q_t */
        if (J->o) {
            const double *qt = J->q + (t * H + head) * dk;
            double *ot = J->o + (t * H + head) * dv;
            for (int64_t j = 0; j < dv; ++j) ot[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d) {
                const double qd = qt[d];
                const double *Md = M + d * dv;
                for (int64_t j = 0; j < dv; ++j) ot[j] += qd * Md[j];
            }
            for (int64_t j = 0; j < dv; ++j) ot[j] *= J->scale;
        }
    }
}

static void *scan_worker(void *arg) {
    scan_job *J = (scan_job *)arg;
    double *w = (double *)malloc(sizeof(double) * (size_t)J->d_v);
    const int64_t n_units = J->n_seqs * J->n_heads;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= n_units) break;
        scan_one(J, u / J->n_heads, u % J->n_heads, w);
    }
    free(w);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments. */
int oracle_gdn_scan_f64(int64_t n_seqs, int64_t n_heads, int64_t d_k, int64_t d_v,
                        const int64_t *cu_seqlens,
                        const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta,
                        const double *S0, double scale,
                        double *o, double *S_final, int n_threads) {
    if (n_seqs < 0 || n_heads <= 0 || d_k <= 0 || d_v <= 0 || !cu_seqlens || !k || !v ||
        !log_alpha || !beta || !S_final || (o && !q))
        return -1;
    scan_job J;
    J.n_seqs = n_seqs; J.n_heads = n_heads; J.d_k = d_k; J.d_v = d_v;
    J.cu_seqlens = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;
    J.scale = scale; J.o = o; J.S_final = S_final;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < n_threads; ++i)
        if (pthread_create(&th[started], NULL, scan_worker, &J) == 0) ++started;
    scan_worker(&J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
