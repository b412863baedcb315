/*
 * kda_oracle.c -- FP64 token-by-token Kimi Delta Attention recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the CPU oracle that the CUDA
 * library is checked against.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load it.  It shares no code, header or
 * constant with the CUDA library, and the library never calls it.
 *
 * What it computes (one independent sequence per (b, h), processed in token
 * order, everything in double precision):
 *
 *   optional per-head L2 norm of q_t and k_t:  x <- x / sqrt(sum x^2 + eps)
 *       page "Kimi K3 の KDA(1)", section 1.2.1 (use_qk_l2norm_in_kernel)
 *   alpha_t = exp(g_t) per key channel (unsigned KDA), or alpha_t = g_t
 *       itself, signed, in Complex-KDA mode
 *       page "GDN, KDA の整理", section "Kimi Delta Attention";
 *       page "Complex KDA: 理解并增强 Kimi Delta Attention 的表达能力" (gate in [-1,1])
 *   decay:  St = Diag(alpha_t) S_{t-1}          (rows are key channels)
 *   erase + write:  S_t = St + beta_t k_t (v_t - St^T k_t)^T
 *       page "Kimi K3 の KDA(1)", section 1.2.1 (decay -> erase -> write);
 *       page "GDN, KDA の整理", section "Online learning" (gradient step
 *       evaluated at the decayed state)
 *   read-out after the write:  o_t = scale * S_t^T q_t
 *       page "Kimi K3 の KDA(1)", section 1.2.1 (reads S_t, not S_{t-1})
 *
 * Layouts (all contiguous, row-major):
 *   q, k, g : [B, T, H, dk]      v, out : [B, T, H, dv]
 *   beta    : [B, T, H]          S0, S_T : [B, H, dk, dv]  (S0 may be NULL = 0)
 *
 * The function is deliberately plain: no blocking, no reordering of the sums
 * beyond the definition above.  Threads (POSIX) only split the independent
 * (b, h) sequences.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *S0;
    double *out, *S_T;
    long B, T, H, dk, dv;
    int l2norm, complex_gate;
    double scale, eps;
    long next_unit; /* guarded by mu */
    pthread_mutex_t mu;
} job_t;

static void run_sequence(job_t *J, long b, long h) {
    const long B = J->B, T = J->T, H = J->H, dk = J->dk, dv = J->dv;
    (void)B;
    double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
    double *qn = (double *)malloc(sizeof(double) * (size_t)dk);
    double *kn = (double *)malloc(sizeof(double) * (size_t)dk);
    double *r = (double *)malloc(sizeof(double) * (size_t)dv);
    const long sbase = (b * H + h) * dk * dv;
    if (J->S0) memcpy(S, J->S0 + sbase, sizeof(double) * (size_t)(dk * dv));
    else memset(S, 0, sizeof(double) * (size_t)(dk * dv));

    for (long t = 0; t < T; ++t) {
        const long row = (b * T + t) * H + h;
        const double *qt = J->q + row * dk;
        const double *kt = J->k + row * dk;
        const double *gt = J->g + row * dk;
        const double *vt = J->v + row * dv;
        const double bt = J->beta[row];
        double *ot = J->out + row * dv;

        /* per-head L2 normalisation of q and k */
        double sq = 0.0, sk = 0.0;
        for (long i = 0; i < dk; ++i) { sq += qt[i] * qt[i]; sk += kt[i] * kt[i]; }
        const double fq = J->l2norm ? 1.0 / sqrt(sq + J->eps) : 1.0;
        const double fk = J->l2norm ? 1.0 / sqrt(sk + J->eps) : 1.0;
        for (long i = 0; i < dk; ++i) { qn[i] = qt[i] * fq; kn[i] = kt[i] * fk; }

        /* decay: row i of S (key channel i) scaled by alpha_i */
        for (long i = 0; i < dk; ++i) {
            const double a = J->complex_gate ? gt[i] : exp(gt[i]);
            for (long j = 0; j < dv; ++j) S[i * dv + j] *= a;
        }
        /* residual r = v - St^T k */
        for (long j = 0; j < dv; ++j) {
            double p = 0.0;
            for (long i = 0; i < dk; ++i) p += S[i * dv + j] * kn[i];
            r[j] = vt[j] - p;
        }
        /* erase + write: S += beta k r^T */
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j) S[i * dv + j] += bt * kn[i] * r[j];
        /* read-out of the post-write state */
        for (long j = 0; j < dv; ++j) {
            double o = 0.0;
            for (long i = 0; i < dk; ++i) o += S[i * dv + j] * qn[i];
            ot[j] = J->scale * o;
        }
    }
    if (J->S_T) memcpy(J->S_T + sbase, S, sizeof(double) * (size_t)(dk * dv));
    free(S); free(qn); free(kn); free(r);
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const long u = J->next_unit++;
        pthread_mutex_unlock(&J->mu);
        if (u >= J->B * J->H) break;
        run_sequence(J, u / J->H, u % J->H);
    }
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments. nthreads <= 0 means 1. */
int kda_oracle_recurrence(const double *q, const double *k, const double *v,
                          const double *g, const double *beta, const double *S0,
                          double *out, double *S_T, long B, long T, long H,
                          long dk, long dv, int l2norm, int complex_gate,
                          double scale, double eps, int nthreads) {
    if (!q || !k || !v || !g || !beta || !out) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    job_t J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.S0 = S0;
    J.out = out; J.S_T = S_T;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv;
    J.l2norm = l2norm; J.complex_gate = complex_gate;
    J.scale = scale; J.eps = eps;
    J.next_unit = 0;
    pthread_mutex_init(&J.mu, NULL);
    long units = B * H;
    int nt = nthreads <= 0 ? 1 : nthreads;
    if (nt > units) nt = (int)(units > 0 ? units : 1);
    if (nt == 1) {
        worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
        for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, worker, &J);
        for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.mu);
    return 0;
}
