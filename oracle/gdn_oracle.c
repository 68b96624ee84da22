/*
 * Gated DeltaNet oracle: the token-by-token gated delta rule in fp64 on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker for the CUDA library, not
 * part of it.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline may load it.  It shares no code, header or constant with the CUDA
 * path.
 *
 * What it computes (source: "Qwen3.8-Flash-Next 技术总结 -- Qwen4 架构的探路者",
 * section 2.1 "Gated DeltaNet", the state-update equation and the paragraph
 * right after it):
 *
 *   S_t = alpha_t * S_{t-1} + beta_t * k_t * (v_t - alpha_t * S_{t-1}^T k_t)^T
 *
 * with S_t a dk x dv matrix (row index = key dimension, so that k v^T is
 * dk x dv), alpha_t the data-dependent forget gate and beta_t the write
 * strength.  This is the first of the two equal forms the page prints; the
 * second form, alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, is
 * only used by the tests that pin this file.
 *
 * Read-out (not spelled out on the page, which calls S the "memory matrix" of
 * linear attention; the plainest reading is adopted): o_t = S_t^T q_t, taken
 * with the state AFTER the update of token t, with no 1/sqrt(dk) scale.
 *
 * Head sharing (the page gives 16 QK heads for 48 V heads but not the map):
 * V head h reads q and k of QK head h / (Hv / Hqk), i.e. contiguous groups.
 * Gates are per V head: alpha, beta have layout [B, T, Hv].
 *
 * Layouts (contiguous, row-major):
 *   q, k     [B, T, Hqk, dk]   float  (fp32 values; bf16 inputs are upcast exactly)
 *   v        [B, T, Hv,  dv]   float
 *   alpha    [B, T, Hv]        float  (alpha itself, not its log)
 *   beta     [B, T, Hv]        float
 *   S0       [B, Hv, dk, dv]   float  (NULL means zeros)
 *   o        [B, T, nh, dv]    double (nh = h_end - h_begin, heads h_begin..h_end-1)
 *   S_final  [B, nh, dk, dv]   double (may be NULL)
 *
 * All arithmetic is fp64.  Work is split over (b, h) pairs across POSIX
 * threads; each pair is a plain serial loop over t.
 */
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const float *q, *k, *v, *alpha, *beta, *S0;
    double *o, *S_final;
    long B, T, Hqk, Hv, dk, dv, h_begin, h_end;
    long next_unit;              /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
    int failed;
} oracle_job;

/* One (b, h) sequence: the serial recurrence over t. */
static int run_sequence(oracle_job *job, long b, long h)
{
    const long T = job->T, Hqk = job->Hqk, Hv = job->Hv, dk = job->dk, dv = job->dv;
    const long nh = job->h_end - job->h_begin;
    const long g = Hv / Hqk;
    const long hq = h / g;
    double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv));
    double *p = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !p || !u) {
        free(S); free(p); free(u);
        return -1;
    }
    /* S <- S0 (or zero). */
    for (long i = 0; i < dk; ++i)
        for (long j = 0; j < dv; ++j)
            S[i * dv + j] = job->S0 ? (double)job->S0[((b * Hv + h) * dk + i) * dv + j] : 0.0;

    for (long t = 0; t < T; ++t) {
        const float *kt = job->k + ((b * T + t) * Hqk + hq) * dk;
        const float *qt = job->q + ((b * T + t) * Hqk + hq) * dk;
        const float *vt = job->v + ((b * T + t) * Hv + h) * dv;
        const double a = (double)job->alpha[(b * T + t) * Hv + h];
        const double be = (double)job->beta[(b * T + t) * Hv + h];

        /* p = S_{t-1}^T k_t  (what the memory already predicts for key k_t) */
        for (long j = 0; j < dv; ++j) p[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double ki = (double)kt[i];
            for (long j = 0; j < dv; ++j) p[j] += S[i * dv + j] * ki;
        }
        /* u = beta_t (v_t - alpha_t p): the corrected value that gets written */
        for (long j = 0; j < dv; ++j) u[j] = be * ((double)vt[j] - a * p[j]);
        /* S_t = alpha_t S_{t-1} + k_t u^T */
        for (long i = 0; i < dk; ++i) {
            const double ki = (double)kt[i];
            for (long j = 0; j < dv; ++j) S[i * dv + j] = a * S[i * dv + j] + ki * u[j];
        }
        /* o_t = S_t^T q_t */
        double *ot = job->o + ((b * T + t) * nh + (h - job->h_begin)) * dv;
        for (long j = 0; j < dv; ++j) ot[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double qi = (double)qt[i];
            for (long j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qi;
        }
    }
    if (job->S_final) {
        double *dst = job->S_final + (b * nh + (h - job->h_begin)) * dk * dv;
        memcpy(dst, S, sizeof(double) * (size_t)(dk * dv));
    }
    free(S); free(p); free(u);
    return 0;
}

static void *worker(void *arg)
{
    oracle_job *job = (oracle_job *)arg;
    const long nh = job->h_end - job->h_begin;
    const long units = job->B * nh;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        const long unit = job->next_unit++;
        pthread_mutex_unlock(&job->lock);
        if (unit >= units) break;
        const long b = unit / nh, h = job->h_begin + unit % nh;
        if (run_sequence(job, b, h) != 0) {
            pthread_mutex_lock(&job->lock);
            job->failed = 1;
            pthread_mutex_unlock(&job->lock);
        }
    }
    return NULL;
}

/*
 * Runs the recurrence for V heads [h_begin, h_end) of every batch entry.
 * Returns 0 on success, 1 on a bad argument, 2 if memory or a thread could
 * not be obtained.
 */
int gdn_oracle_forward(const float *q, const float *k, const float *v,
                       const float *alpha, const float *beta, const float *S0,
                       double *o, double *S_final,
                       long B, long T, long Hqk, long Hv, long dk, long dv,
                       long h_begin, long h_end, int nthreads)
{
    if (B < 0 || T < 0 || Hqk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return 1;
    if (Hv % Hqk != 0) return 1;
    if (h_begin < 0 || h_end > Hv || h_begin > h_end) return 1;
    if (nthreads < 1) nthreads = 1;

    oracle_job job;
    job.q = q; job.k = k; job.v = v; job.alpha = alpha; job.beta = beta; job.S0 = S0;
    job.o = o; job.S_final = S_final;
    job.B = B; job.T = T; job.Hqk = Hqk; job.Hv = Hv; job.dk = dk; job.dv = dv;
    job.h_begin = h_begin; job.h_end = h_end;
    job.next_unit = 0;
    job.failed = 0;
    pthread_mutex_init(&job.lock, NULL);

    pthread_t *threads = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!threads) {
        pthread_mutex_destroy(&job.lock);
        return 2;
    }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&threads[i], NULL, worker, &job) != 0) break;
        ++started;
    }
    if (started == 0) worker(&job); /* no thread could start: run inline */
    for (int i = 0; i < started; ++i) pthread_join(threads[i], NULL);
    free(threads);
    pthread_mutex_destroy(&job.lock);
    return job.failed ? 2 : 0;
}
