/*
 * Oracle for the Gated Delta Rule-2 token mixer: the plain recurrence, token by
 * token, in double precision on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg load this library.  It shares no code with
 * the CUDA path, and nothing on the product path calls it.
 *
 * What it computes, per (batch b, head h), starting from S = S0 (zeros if S0 is
 * NULL), for t = 0 .. T-1 (Gated DeltaNet-2 article on snilld.dk, "Hvad Gated
 * DeltaNet-2 aendrer", the compact update):
 *
 *     S_t = (I - k_t (b_t * k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t * v_t)^T
 *     o_t = S_t^T q_t
 *
 * with S of shape d_k x d_v, alpha_t = exp(log_alpha_t) the channel-wise decay
 * applied before the edit, b_t the erase gate on the key axis and w_t the write
 * gate on the value axis.  The readout uses the updated state (Gated DeltaNet-2
 * guide, "End-to-End PyTorch Implementation", the loop reads y_t after the
 * update).  The steps below are that formula expanded, in its own order:
 *
 *     1. decay:  S[i][:] *= alpha_i
 *     2. erase:  e = S^T (b * k);  S -= k e^T
 *     3. write:  S += k (w * v)^T
 *     4. read:   o = S^T q
 *
 * Layouts: q, k, log_alpha, b are [B, T, H, d_k]; v, w and o are [B, T, H, d_v];
 * S0 and S_T are [B, H, d_k, d_v]; all row-major doubles.  S_T may alias S0.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *log_alpha, *b, *w, *S0;
    double *o, *S_T;
    long B, T, H, dk, dv;
    long unit_begin, unit_end;   /* units are b * H + h */
    int status;
} job_t;

static void run_unit(job_t *J, long unit, double *S, double *e, double *wv)
{
    const long bb = unit / J->H, h = unit % J->H;
    const long dk = J->dk, dv = J->dv;

    if (J->S0)
        memcpy(S, J->S0 + unit * dk * dv, sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * dk * dv);

    for (long t = 0; t < J->T; ++t) {
        const long tok = (bb * J->T + t) * J->H + h;
        const double *qt = J->q + tok * dk, *kt = J->k + tok * dk;
        const double *lat = J->log_alpha + tok * dk, *bt = J->b + tok * dk;
        const double *vt = J->v + tok * dv, *wt = J->w + tok * dv;

        /* 1. decay, Diag(alpha_t) S */
        for (long i = 0; i < dk; ++i) {
            const double a = exp(lat[i]);
            for (long j = 0; j < dv; ++j) S[i * dv + j] *= a;
        }
        /* 2. erase along k read through b*k: e = S^T (b*k), S -= k e^T */
        for (long j = 0; j < dv; ++j) e[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double x = bt[i] * kt[i];
            for (long j = 0; j < dv; ++j) e[j] += x * S[i * dv + j];
        }
        /* 3. write k (w*v)^T; steps 2 and 3 touch the same rows, so fuse them */
        for (long j = 0; j < dv; ++j) wv[j] = wt[j] * vt[j];
        for (long i = 0; i < dk; ++i)
            for (long j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * (wv[j] - e[j]);
        /* 4. read out with the updated state: o = S^T q */
        if (J->o) {
            double *ot = J->o + tok * dv;
            for (long j = 0; j < dv; ++j) ot[j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) ot[j] += qt[i] * S[i * dv + j];
        }
    }
    if (J->S_T) memcpy(J->S_T + unit * dk * dv, S, sizeof(double) * dk * dv);
}

static void *run_job(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = malloc(sizeof(double) * J->dk * J->dv);
    double *e = malloc(sizeof(double) * J->dv);
    double *wv = malloc(sizeof(double) * J->dv);
    if (!S || !e || !wv) {
        J->status = 2;
    } else {
        for (long u = J->unit_begin; u < J->unit_end; ++u) run_unit(J, u, S, e, wv);
        J->status = 0;
    }
    free(S); free(e); free(wv);
    return NULL;
}

/*
 * Runs the recurrence over all B*H units, split over nthreads threads.
 * Returns 0 on success, 1 on bad arguments, 2 on allocation failure.
 */
int gdn2_oracle_forward(const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *b, const double *w,
                        const double *S0, double *o, double *S_T,
                        long B, long T, long H, long dk, long dv, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !b || !w) return 1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return 1;
    const long units = B * H;
    if (units == 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = (int)units;

    job_t *jobs = calloc((size_t)nthreads, sizeof(job_t));
    pthread_t *tids = calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tids) { free(jobs); free(tids); return 2; }
    for (int n = 0; n < nthreads; ++n) {
        job_t J = {q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, dk, dv,
                   units * n / nthreads, units * (n + 1) / nthreads, 0};
        jobs[n] = J;
    }
    int rc = 0;
    if (nthreads == 1) {
        run_job(&jobs[0]);
        rc = jobs[0].status;
    } else {
        for (int n = 0; n < nthreads; ++n) pthread_create(&tids[n], NULL, run_job, &jobs[n]);
        for (int n = 0; n < nthreads; ++n) {
            pthread_join(tids[n], NULL);
            if (jobs[n].status) rc = jobs[n].status;
        }
    }
    free(jobs); free(tids);
    return rc;
}

/*
 * One decode step: the same update for a single token per unit, with the state
 * updated in place.  q, k, log_alpha, b are [B, H, d_k]; v, w, o are [B, H, d_v];
 * S is [B, H, d_k, d_v].
 */
int gdn2_oracle_decode_step(const double *q, const double *k, const double *v,
                            const double *log_alpha, const double *b, const double *w,
                            double *S, double *o, long B, long H, long dk, long dv, int nthreads)
{
    if (!S) return 1;
    return gdn2_oracle_forward(q, k, v, log_alpha, b, w, S, o, S, B, 1, H, dk, dv, nthreads);
}
