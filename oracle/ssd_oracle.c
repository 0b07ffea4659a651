/*
 * CPU oracle for the int8-input Mamba-2 SSD scan -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct fp64 C.  Only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg may load it; the CUDA library never does, and the two
 * share no code (no headers, helpers or constants).
 *
 * What it computes (one (batch, head) pair at a time, sequentially over tokens):
 *
 *   dequantize   x_t[p] = s_x[h] * xq[b,t,h,p]
 *                B_t[n] = s_B[g] * Bq[b,t,g,n],  C_t[n] = s_C[g] * Cq[b,t,g,n],  g = h / (H/G)
 *                (ssd_oracle_scan_pern: s_B[g, n] and s_C[g, n], one scale per dstate channel
 *                -- the per-N axis of SSDi8's quantization-axis table, Table 10)
 *   recurrence   h_t = Abar_t * h_{t-1} + Bbar_t x_t
 *                ("Ternary Mamba: Grouped QAT of W1.58A16 SSMs", section 1, the SSM recurrence)
 *   discretised  Abar_t = exp(dt_t * A_h),   Bbar_t x_t = dt_t * x_t B_t^T   (Mamba-2 form)
 *   output       y_t[p] = sum_n C_t[n] * h_t[p, n] + D_h * x_t[p]
 *
 * h_0 is the optional initial state (zero otherwise); the final state is h_L.  The decode
 * update is one step of the same recurrence on a given state ("Quamba2" OpenReview
 * rebuttal, the SSD-update discussion around Tables R7/R8).  Output requantization is the
 * static symmetric rule of the Quamba project page: q = clamp(rne(y / s_y), -127, 127).
 *
 * The chunk matrix of SSDi8's ChunkBMM ("SSDi8", Table 5, "Quant. of ChunkBMM") is
 * CB[t, s] = sum_n Cq[t, n] * Bq[s, n] over the int8 codes of one chunk and one group,
 * computed here in int64.
 *
 * An optional additive perturbation eps[b,t,h,p,n] can be injected into h_t right after
 * each update; it exists so that the tests can check the error-accumulation identity
 * e_T = sum_t Abar^{T-t} eps_t ("Ternary Mamba", section 6.2, eq. 2).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const int8_t *x, *B, *C;
    const float *dt, *A, *D, *sx, *sB, *sC;
    int batch, seqlen, nheads, headdim, dstate, ngroups;
    const double *init_state; /* [b,h,p,n] or NULL */
    const double *eps;        /* [b,l,h,p,n] or NULL */
    double *final_state;      /* [b,h,p,n] or NULL */
    double *y;                /* [b,l,h,p] */
    int next;                 /* next (b,h) work item, taken atomically */
    int status;
    int bc_per_n;             /* sB, sC are [g, n] (per dstate channel) instead of [g] */
} scan_job;

static void scan_pair(scan_job *j, int b, int h)
{
    const int L = j->seqlen, H = j->nheads, P = j->headdim, N = j->dstate, G = j->ngroups;
    const int g = h / (H / G);
    double *state = (double *)calloc((size_t)P * N, sizeof(double));
    double *Bt = (double *)malloc(sizeof(double) * (size_t)N);
    double *Ct = (double *)malloc(sizeof(double) * (size_t)N);
    if (!state || !Bt || !Ct) {
        j->status = 1;
        free(state); free(Bt); free(Ct);
        return;
    }
    if (j->init_state)
        memcpy(state, j->init_state + ((size_t)b * H + h) * P * N, sizeof(double) * (size_t)P * N);

    for (int t = 0; t < L; ++t) {
        const size_t bt = (size_t)b * L + t;
        const double dtv = (double)j->dt[bt * H + h];
        const double abar = exp(dtv * (double)j->A[h]);
        for (int n = 0; n < N; ++n) {
            const double sb = (double)(j->bc_per_n ? j->sB[g * N + n] : j->sB[g]);
            const double sc = (double)(j->bc_per_n ? j->sC[g * N + n] : j->sC[g]);
            Bt[n] = sb * (double)j->B[(bt * G + g) * N + n];
            Ct[n] = sc * (double)j->C[(bt * G + g) * N + n];
        }
        for (int p = 0; p < P; ++p) {
            const double xv = (double)j->sx[h] * (double)j->x[(bt * H + h) * P + p];
            double *row = state + (size_t)p * N;
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                row[n] = abar * row[n] + dtv * xv * Bt[n];
                if (j->eps)
                    row[n] += j->eps[((bt * H + h) * P + p) * N + n];
                acc += Ct[n] * row[n];
            }
            j->y[(bt * H + h) * P + p] = acc + (double)j->D[h] * xv;
        }
    }
    if (j->final_state)
        memcpy(j->final_state + ((size_t)b * H + h) * P * N, state, sizeof(double) * (size_t)P * N);
    free(state); free(Bt); free(Ct);
}

static void *scan_worker(void *arg)
{
    scan_job *j = (scan_job *)arg;
    const int total = j->batch * j->nheads;
    for (;;) {
        int item = __atomic_fetch_add(&j->next, 1, __ATOMIC_RELAXED);
        if (item >= total)
            break;
        scan_pair(j, item / j->nheads, item % j->nheads);
    }
    return NULL;
}

static int pick_threads(int requested, int items)
{
    int n = requested;
    if (n <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        n = c > 0 ? (int)c : 1;
    }
    if (n > items)
        n = items;
    return n < 1 ? 1 : n;
}

static int run_pool(void *(*fn)(void *), void *job, int nthreads)
{
    if (nthreads == 1) {
        fn(job);
        return 0;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th)
        return 1;
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, fn, job) != 0)
            break;
        ++started;
    }
    if (started == 0)
        fn(job);
    for (int i = 0; i < started; ++i)
        pthread_join(th[i], NULL);
    free(th);
    return 0;
}

static int scan_impl(const int8_t *x, const int8_t *B, const int8_t *C, const float *dt,
                     const float *A, const float *D, const float *x_scale, const float *B_scale,
                     const float *C_scale, int batch, int seqlen, int nheads, int headdim,
                     int dstate, int ngroups, const double *init_state, const double *eps,
                     double *final_state, double *y, int nthreads, int bc_per_n)
{
    if (batch < 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        nheads % ngroups != 0)
        return -1;
    scan_job j = {x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, seqlen, nheads, headdim,
                  dstate, ngroups, init_state, eps, final_state, y, 0, 0, bc_per_n};
    const int items = batch * nheads;
    if (items == 0)
        return 0;
    const int nt = pick_threads(nthreads, items);
    if (run_pool(scan_worker, &j, nt) != 0 || j.status != 0)
        return -2;
    return nt;
}

/* Sequential fp64 scan over a whole prefill.  Returns the number of threads used, or a
 * negative value on bad arguments / allocation failure. */
int ssd_oracle_scan(const int8_t *x, const int8_t *B, const int8_t *C, const float *dt,
                    const float *A, const float *D, const float *x_scale, const float *B_scale,
                    const float *C_scale, int batch, int seqlen, int nheads, int headdim,
                    int dstate, int ngroups, const double *init_state, const double *eps,
                    double *final_state, double *y, int nthreads)
{
    return scan_impl(x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, seqlen, nheads,
                     headdim, dstate, ngroups, init_state, eps, final_state, y, nthreads, 0);
}

/* The same scan with B_scale and C_scale given per group and dstate channel, [g, n]. */
int ssd_oracle_scan_pern(const int8_t *x, const int8_t *B, const int8_t *C, const float *dt,
                         const float *A, const float *D, const float *x_scale,
                         const float *B_scale, const float *C_scale, int batch, int seqlen,
                         int nheads, int headdim, int dstate, int ngroups,
                         const double *init_state, const double *eps, double *final_state,
                         double *y, int nthreads)
{
    return scan_impl(x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, seqlen, nheads,
                     headdim, dstate, ngroups, init_state, eps, final_state, y, nthreads, 1);
}

/* One decode step on an fp64 state held by the caller (updated in place). */
int ssd_oracle_step(double *state, const int8_t *x, const int8_t *B, const int8_t *C,
                    const float *dt, const float *A, const float *D, const float *x_scale,
                    const float *B_scale, const float *C_scale, int batch, int nheads,
                    int headdim, int dstate, int ngroups, double *y, int nthreads)
{
    /* A single token of the recurrence is a length-1 scan whose initial and final state is
     * the decode state; run it as such so both share the one definition above. */
    if (batch < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0 ||
        nheads % ngroups != 0)
        return -1;
    const size_t sz = (size_t)batch * nheads * headdim * dstate;
    double *out = (double *)malloc(sizeof(double) * (sz ? sz : 1));
    if (!out)
        return -2;
    int r = ssd_oracle_scan(x, B, C, dt, A, D, x_scale, B_scale, C_scale, batch, 1, nheads,
                            headdim, dstate, ngroups, state, NULL, out, y, nthreads);
    if (r >= 0)
        memcpy(state, out, sizeof(double) * sz);
    free(out);
    return r;
}

/* ChunkBMM: CB[b, c, g, t, s] = sum_n Cq[b, cQ+t, g, n] * Bq[b, cQ+s, g, n] (int64, full
 * Q x Q block, no causal mask); rows / columns past the sequence end are zero. */
int ssd_oracle_chunk_cb(const int8_t *C, const int8_t *B, int batch, int seqlen, int ngroups,
                        int dstate, int chunk_size, int64_t *cb)
{
    if (batch < 0 || seqlen < 0 || ngroups <= 0 || dstate <= 0 || chunk_size <= 0)
        return -1;
    const int Q = chunk_size, nchunks = (seqlen + Q - 1) / Q;
    const int G = ngroups, N = dstate, L = seqlen;
    for (int b = 0; b < batch; ++b)
        for (int c = 0; c < nchunks; ++c)
            for (int g = 0; g < G; ++g) {
                int64_t *blk = cb + ((((size_t)b * nchunks + c) * G + g) * Q) * Q;
                for (int t = 0; t < Q; ++t)
                    for (int s = 0; s < Q; ++s) {
                        const int lt = c * Q + t, ls = c * Q + s;
                        int64_t acc = 0;
                        if (lt < L && ls < L)
                            for (int n = 0; n < N; ++n)
                                acc += (int64_t)C[(((size_t)b * L + lt) * G + g) * N + n] *
                                       (int64_t)B[(((size_t)b * L + ls) * G + g) * N + n];
                        blk[(size_t)t * Q + s] = acc;
                    }
            }
    return 0;
}

/* Static symmetric requantization of the output: q = clamp(rne(y / s_y), -127, 127). */
int ssd_oracle_requant(const double *y, int64_t count, double y_scale, int8_t *q)
{
    if (count < 0 || !(y_scale > 0.0))
        return -1;
    for (int64_t i = 0; i < count; ++i) {
        double r = nearbyint(y[i] / y_scale); /* default rounding mode: half to even */
        if (r > 127.0)
            r = 127.0;
        if (r < -127.0)
            r = -127.0;
        q[i] = (int8_t)r;
    }
    return 0;
}
