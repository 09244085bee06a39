/*
 * KDA gated delta-rule recurrence: fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the CUDA path is
 * checked against.  Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load it.  The library path never links, loads or calls it, and it shares no
 * code, header, table or constant with the CUDA kernels.
 *
 * It is the plain definition, token by token, in double precision, with no chunking, blocking
 * or reordering.  Per (sequence, head) unit, with state S in R^{d_k x d_v} (row = key channel,
 * column = value channel):
 *
 *   g_t   = g_min * sigmoid(exp(A_h) * a_t),  g_min = -5        per key channel
 *           ("Kimi K3 · Lesson 3 of 14", passage "The mapping that changed, from §2.1.1 eq. 5":
 *            a scaled sigmoid with a fixed floor of -5 and a learnable per-head log-scale A_h)
 *   S     = Diag(exp(g_t)) S                                    fade
 *   r     = S^T k_t                                             what k_t retrieves now
 *   S     = S + beta_t k_t (v_t - r)^T                          erase + write
 *           ("Review A · Sequence and depth", Free recall, first question: fade, erase, write;
 *            "K3 Architecture Illustrated", §"Combining KDA and MLA", FIG 21: retention first,
 *            then the delta update at the current key, then the query read)
 *   o_t   = S^T (scale * q_t)                                   read, after the update
 *   out_t = sigmoid(gate_t) (.) o_t                             full-rank output gate
 *           ("Kimi K3 · Lesson 3 of 14", passage on the output gate after the recurrent read)
 *
 * Readings where the pages are silent: the read comes after the token's own update; erase acts on
 * the faded state; the gate logits are an input (their projection is not part of the recurrence);
 * a missing gate means out = o; a missing initial state means zeros.
 *
 * Parity status: every function here is pinned by CPU tests against closed forms and an
 * independent O(T^2) parallel form (see tests/test_oracle_pins.py).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KDA_ORACLE_GMIN (-5.0)

static double sigmoid_d(double x) { return 1.0 / (1.0 + exp(-x)); }

/* g = g_min * sigmoid(exp(A_log) * a) for n channels. */
void kda_oracle_gate(int64_t n, const double *a, double A_log, double *g) {
    const double scale = exp(A_log);
    for (int64_t i = 0; i < n; ++i) g[i] = KDA_ORACLE_GMIN * sigmoid_d(scale * a[i]);
}

/*
 * One (sequence, head) unit given the per-token log-decay g directly.
 * Row t of every per-token operand starts at base + t * ld_*; channels are contiguous.
 *   q, k, g : [T, d_k]     v, gate : [T, d_v]     beta : [T] (stride ld_beta)
 *   S0      : [d_k, d_v] row-major, or NULL for zeros
 *   out     : [T, d_v] (stride ld_out)            S_final : [d_k, d_v] or NULL
 * gate may be NULL (no output gate).  S is a caller-provided [d_k, d_v] scratch buffer.
 */
void kda_oracle_unit_g(int64_t T, int d_k, int d_v, const double *q, int64_t ld_q, const double *k,
                       int64_t ld_k, const double *v, int64_t ld_v, const double *g, int64_t ld_g,
                       const double *beta, int64_t ld_beta, const double *gate, int64_t ld_gate,
                       double scale, const double *S0, double *out, int64_t ld_out, double *S_final,
                       double *S /* scratch [d_k*d_v] */, double *r /* scratch [d_v] */) {
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)d_k * d_v);
    else memset(S, 0, sizeof(double) * (size_t)d_k * d_v);

    for (int64_t t = 0; t < T; ++t) {
        const double *qt = q + t * ld_q, *kt = k + t * ld_k, *vt = v + t * ld_v;
        const double *gt = g + t * ld_g;
        const double bt = beta[t * ld_beta];

        /* fade: every key channel (row of S) by its own retention factor exp(g) */
        for (int i = 0; i < d_k; ++i) {
            const double alpha = exp(gt[i]);
            double *row = S + (size_t)i * d_v;
            for (int j = 0; j < d_v; ++j) row[j] *= alpha;
        }
        /* r = S^T k : the value the faded memory currently returns for k */
        for (int j = 0; j < d_v; ++j) r[j] = 0.0;
        for (int i = 0; i < d_k; ++i) {
            const double ki = kt[i];
            const double *row = S + (size_t)i * d_v;
            for (int j = 0; j < d_v; ++j) r[j] += ki * row[j];
        }
        /* erase + write: S += beta k (v - r)^T */
        for (int i = 0; i < d_k; ++i) {
            const double c = bt * kt[i];
            double *row = S + (size_t)i * d_v;
            for (int j = 0; j < d_v; ++j) row[j] += c * (vt[j] - r[j]);
        }
        /* read o = S^T (scale q), then the sigmoid output gate */
        double *ot = out + t * ld_out;
        for (int j = 0; j < d_v; ++j) ot[j] = 0.0;
        for (int i = 0; i < d_k; ++i) {
            const double qi = scale * qt[i];
            const double *row = S + (size_t)i * d_v;
            for (int j = 0; j < d_v; ++j) ot[j] += qi * row[j];
        }
        if (gate) {
            const double *gg = gate + t * ld_gate;
            for (int j = 0; j < d_v; ++j) ot[j] *= sigmoid_d(gg[j]);
        }
    }
    if (S_final) memcpy(S_final, S, sizeof(double) * (size_t)d_k * d_v);
}

/* ---- packed multi-unit driver ---------------------------------------------------------------
 * Token-major packed layout, as a user would hold it:
 *   q, k, a : [T_total, H, d_k]    v, gate : [T_total, H, d_v]    beta : [T_total, H]
 *   A_log   : [H]                  cu_seqlens : [num_seqs + 1], sequence n = tokens
 *                                  [cu_seqlens[n], cu_seqlens[n+1])
 *   S0, S_final : [num_seqs, H, d_k, d_v] or NULL;  out : [T_total, H, d_v]
 * Units (n, h) are independent; they are split across n_threads POSIX threads.
 */
typedef struct {
    int64_t T_total;
    int H, d_k, d_v, num_seqs;
    const int64_t *cu;
    const double *q, *k, *v, *a, *beta, *gate, *A_log, *S0;
    double scale;
    double *out, *S_final;
    int n_threads, tid;
    int status;
} kda_oracle_job;

static void *kda_oracle_worker(void *arg) {
    kda_oracle_job *J = (kda_oracle_job *)arg;
    const int H = J->H, dk = J->d_k, dv = J->d_v;
    int64_t max_len = 0;
    for (int n = 0; n < J->num_seqs; ++n) {
        int64_t L = J->cu[n + 1] - J->cu[n];
        if (L > max_len) max_len = L;
    }
    double *g = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * dk);
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!g || !S || !r) {
        J->status = 1;
        free(g); free(S); free(r);
        return NULL;
    }
    const int64_t units = (int64_t)J->num_seqs * H;
    for (int64_t u = J->tid; u < units; u += J->n_threads) {
        const int n = (int)(u / H), h = (int)(u % H);
        const int64_t t0 = J->cu[n], L = J->cu[n + 1] - J->cu[n];
        for (int64_t t = 0; t < L; ++t)
            kda_oracle_gate(dk, J->a + ((t0 + t) * H + h) * dk, J->A_log[h], g + t * dk);
        const size_t st = (size_t)dk * dv;
        kda_oracle_unit_g(L, dk, dv,
                          J->q + (t0 * H + h) * dk, (int64_t)H * dk,
                          J->k + (t0 * H + h) * dk, (int64_t)H * dk,
                          J->v + (t0 * H + h) * dv, (int64_t)H * dv,
                          g, dk,
                          J->beta + t0 * H + h, H,
                          J->gate ? J->gate + (t0 * H + h) * dv : NULL, (int64_t)H * dv,
                          J->scale,
                          J->S0 ? J->S0 + ((size_t)n * H + h) * st : NULL,
                          J->out + (t0 * H + h) * dv, (int64_t)H * dv,
                          J->S_final ? J->S_final + ((size_t)n * H + h) * st : NULL, S, r);
    }
    free(g); free(S); free(r);
    return NULL;
}

/* Returns 0 on success, 1 on allocation failure, 2 on bad arguments. */
int kda_oracle_fwd(int64_t T_total, int H, int d_k, int d_v, int num_seqs, const int64_t *cu_seqlens,
                   const double *q, const double *k, const double *v, const double *a,
                   const double *beta, const double *gate, const double *A_log, double scale,
                   const double *S0, double *out, double *S_final, int n_threads) {
    if (H <= 0 || d_k <= 0 || d_v <= 0 || num_seqs < 0 || !cu_seqlens) return 2;
    if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T_total) return 2;
    for (int n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return 2;
    if (n_threads < 1) n_threads = 1;
    kda_oracle_job *jobs = (kda_oracle_job *)calloc((size_t)n_threads, sizeof(kda_oracle_job));
    pthread_t *th = (pthread_t *)calloc((size_t)n_threads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return 1; }
    for (int i = 0; i < n_threads; ++i) {
        kda_oracle_job j = {T_total, H, d_k, d_v, num_seqs, cu_seqlens, q, k, v, a, beta, gate,
                            A_log, S0, scale, out, S_final, n_threads, i, 0};
        jobs[i] = j;
    }
    for (int i = 1; i < n_threads; ++i) pthread_create(&th[i], NULL, kda_oracle_worker, &jobs[i]);
    kda_oracle_worker(&jobs[0]);
    int status = jobs[0].status;
    for (int i = 1; i < n_threads; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].status) status = jobs[i].status;
    }
    free(jobs); free(th);
    return status;
}
