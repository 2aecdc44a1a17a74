/*
 * CPU oracle for the Mamba-2 SSD forward layer: the plain sequential recurrence
 * in fp64.  TEST INFRASTRUCTURE ONLY: it is used by tests/, by the smoke check
 * and by the bench's CPU baseline, never by the library's product path.  It
 * shares no code with the CUDA path.
 *
 * What it computes ("Transformers are SSMs", Sec. 2.4 "SSD layer" with the
 * scalar-times-identity A_t, and the linear / recurrent mode of Sec. 3.4.1,
 * eq. (8): expand the input by B, run the scalar recurrence, contract by C):
 *
 *   for every sequence s and head h (group g = h / (nheads / ngroups)):
 *     state = initial_states[s, h]            (zeros when absent)
 *     for t in the sequence, in order:
 *       delta = softplus(dt[t, h])            (or dt itself when dt_softplus == 0)
 *       a     = exp(delta * -exp(A_log[h]))   (scalar decay, in [0, 1])
 *       state = a * state + (delta * x[t, h, :]) (outer) B[t, g, :]     (P x N)
 *       y[t, h, :] = state @ C[t, g, :] + D[h] * x[t, h, :]
 *     final_states[s, h] = state
 *
 * Readings of points the pages leave open (the same in the CUDA path):
 *  - the input is discretised as delta * x (Sec. 2.1 omits the rule; delta
 *    acts as the input gate),
 *  - A = -exp(A_log) per head,
 *  - D multiplies the raw x,
 *  - the initial state is decayed by the first token's a (the algorithm's
 *    state-to-output term uses an inclusive cumulative decay, Sec. 6),
 *  - packed variable-length sequences exchange no state (Sec. 8.3).
 *
 * Inputs are float32 arrays (holding the exact io-dtype values); all
 * arithmetic is double.  Work is split over (sequence, head) pairs with
 * OpenMP; each pair is an independent sequential loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double softplus(double r)
{
    /* log(1 + exp(r)) without overflow, no threshold shortcut */
    return (r > 0.0 ? r : 0.0) + log1p(exp(-fabs(r)));
}

/*
 * One (sequence, head) pair.
 *   tok0, len   : token range of the sequence in the flattened token axis
 *   y_out       : len * P doubles (row t, column p)
 *   final_out   : P * N doubles, may be NULL
 */
static void ssd_ref_one(int64_t tok0, int64_t len, int h, int H, int P, int N, int G,
                        int dt_softplus, const float *x, const float *dt,
                        const float *A_log, const float *B, const float *C,
                        const float *D, const float *init_sh,
                        double *y_out, double *final_out, double *state)
{
    const int g = h / (H / G);
    const double A = -exp((double)A_log[h]);
    const double Dh = D ? (double)D[h] : 0.0;
    const int64_t PN = (int64_t)P * N;
    if (init_sh) {
        for (int64_t i = 0; i < PN; ++i) state[i] = (double)init_sh[i];
    } else {
        memset(state, 0, sizeof(double) * (size_t)PN);
    }
    for (int64_t t = 0; t < len; ++t) {
        const int64_t tok = tok0 + t;
        const double r = (double)dt[tok * H + h];
        const double delta = dt_softplus ? softplus(r) : r;
        const double a = exp(delta * A);
        const float *xt = x + (tok * H + h) * (int64_t)P;
        const float *Bt = B + (tok * G + g) * (int64_t)N;
        const float *Ct = C + (tok * G + g) * (int64_t)N;
        double *yt = y_out + t * (int64_t)P;
        for (int p = 0; p < P; ++p) {
            const double xb = delta * (double)xt[p];
            double *sp = state + (int64_t)p * N;
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                sp[n] = a * sp[n] + xb * (double)Bt[n];
                acc += sp[n] * (double)Ct[n];
            }
            yt[p] = acc + Dh * (double)xt[p];
        }
    }
    if (final_out) memcpy(final_out, state, sizeof(double) * (size_t)PN);
}

/*
 * Compute the recurrence for `npairs` (sequence, head) pairs.
 *
 *   seq_start[s], seq_len[s]   token range of sequence s (s < nseq)
 *   pair_seq[i], pair_head[i]  the pairs to compute
 *   x (tokens, H, P), dt (tokens, H), B and C (tokens, G, N): float32
 *   A_log, D (H): float32, D may be NULL
 *   init (nseq, H, P, N): float32, may be NULL (zeros)
 *   y_out: pair i writes seq_len[pair_seq[i]] * P doubles at offset
 *          y_offset[i] (caller-computed, in doubles)
 *   final_out: pair i writes P*N doubles at i*P*N; may be NULL
 *   nthreads <= 0 uses the OpenMP default
 *
 * Returns 0, or -1 on an invalid argument.
 */
int ssd_ref_pairs(int nseq, const int64_t *seq_start, const int64_t *seq_len,
                  int H, int P, int N, int G, int dt_softplus,
                  const float *x, const float *dt, const float *A_log,
                  const float *B, const float *C, const float *D, const float *init,
                  int npairs, const int32_t *pair_seq, const int32_t *pair_head,
                  const int64_t *y_offset, double *y_out, double *final_out,
                  int nthreads)
{
    if (nseq < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0 || npairs < 0)
        return -1;
    if (!x || !dt || !A_log || !B || !C || !y_out || !y_offset || !seq_start || !seq_len)
        return -1;
    for (int i = 0; i < npairs; ++i) {
        if (pair_seq[i] < 0 || pair_seq[i] >= nseq || pair_head[i] < 0 || pair_head[i] >= H)
            return -1;
    }
    const int64_t PN = (int64_t)P * N;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        double *state = (double *)malloc(sizeof(double) * (size_t)PN);
        if (!state) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int i = 0; i < npairs; ++i) {
                const int s = pair_seq[i], h = pair_head[i];
                const float *init_sh = init ? init + ((int64_t)s * H + h) * PN : NULL;
                ssd_ref_one(seq_start[s], seq_len[s], h, H, P, N, G, dt_softplus, x, dt,
                            A_log, B, C, D, init_sh, y_out + y_offset[i],
                            final_out ? final_out + (int64_t)i * PN : NULL, state);
            }
            free(state);
        }
    }
    return bad ? -1 : 0;
}

int ssd_ref_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Reverse mode of the same recurrence (the gradient of a loss L with respect
 * to every input, given dL/dy and dL/dfinal_state), written by differentiating
 * the per-token update above step by step.  With G_t = dL/dstate_t (P x N):
 *
 *   G_t = dy_t (outer) C_t + a_{t+1} G_{t+1},     G_T = dL/dfinal (or 0), a_T = 1
 *   dC_t   += state_t^T dy_t                        (N; summed over the heads of a group)
 *   dx_t    = D dy_t + delta_t G_t B_t               (P)
 *   dB_t   += delta_t G_t^T x_t                     (N; summed over the heads of a group)
 *   ddelta  = x_t^T G_t B_t + A a_t <G_t, state_{t-1}>
 *   dA     += delta_t a_t <G_t, state_{t-1}>,   dA_log = A dA   (A = -exp(A_log))
 *   dD     += <dy_t, x_t>
 *   ddt_t   = ddelta * sigmoid(dt_t)   (ddelta when dt_softplus == 0)
 *   dinit   = a_0 G_0
 *
 * state_{t-1} is needed in reverse order: states are recomputed forward from
 * checkpoints kept every kCk tokens.
 */
enum { kCk = 64 };

static double sigmoid(double r)
{
    return r >= 0.0 ? 1.0 / (1.0 + exp(-r)) : exp(r) / (1.0 + exp(r));
}

/* One (sequence, head) pair.  dB_out, dC_out: len * N doubles (this head's
 * contribution); dx_out len * P; ddt_out len; dinit_out P * N (may be NULL). */
static int ssd_ref_bwd_one(int64_t tok0, int64_t len, int h, int H, int P, int N, int G,
                           int dt_softplus, const float *x, const float *dt,
                           const float *A_log, const float *B, const float *C,
                           const float *D, const float *init_sh, const float *dy,
                           const float *dfin_sh, double *dx_out, double *ddt_out,
                           double *dB_out, double *dC_out, double *dAlog_out,
                           double *dD_out, double *dinit_out)
{
    const int g = h / (H / G);
    const double A = -exp((double)A_log[h]);
    const double Dh = D ? (double)D[h] : 0.0;
    const int64_t PN = (int64_t)P * N;
    const int64_t nck = (len + kCk - 1) / kCk;
    double *ck = (double *)calloc((size_t)((nck > 0 ? nck : 1) * PN), sizeof(double));
    double *seg = (double *)malloc(sizeof(double) * (size_t)(kCk * PN));
    double *gst = (double *)malloc(sizeof(double) * (size_t)PN);
    if (!ck || !seg || !gst) {
        free(ck); free(seg); free(gst);
        return -1;
    }
    /* forward: checkpoint k holds the state before token k * kCk */
    double *st = gst;   /* scratch for the forward sweep */
    for (int64_t i = 0; i < PN; ++i) st[i] = init_sh ? (double)init_sh[i] : 0.0;
    for (int64_t t = 0; t < len; ++t) {
        if (t % kCk == 0) memcpy(ck + (t / kCk) * PN, st, sizeof(double) * (size_t)PN);
        const int64_t tok = tok0 + t;
        const double r = (double)dt[tok * H + h];
        const double delta = dt_softplus ? softplus(r) : r;
        const double a = exp(delta * A);
        const float *xt = x + (tok * H + h) * (int64_t)P;
        const float *Bt = B + (tok * G + g) * (int64_t)N;
        for (int p = 0; p < P; ++p)
            for (int n = 0; n < N; ++n)
                st[(int64_t)p * N + n] = a * st[(int64_t)p * N + n] + delta * (double)xt[p] * (double)Bt[n];
    }
    /* reverse sweep; gst = a_{t+1} G_{t+1} before step t */
    for (int64_t i = 0; i < PN; ++i) gst[i] = dfin_sh ? (double)dfin_sh[i] : 0.0;
    double dA = 0.0, dDh = 0.0;
    for (int64_t k = nck - 1; k >= 0; --k) {
        const int64_t t0 = k * kCk, t1 = (t0 + kCk < len) ? t0 + kCk : len;
        /* recompute state_t for t in [t0, t1): seg[t - t0] */
        for (int64_t t = t0; t < t1; ++t) {
            const int64_t tok = tok0 + t;
            const double r = (double)dt[tok * H + h];
            const double delta = dt_softplus ? softplus(r) : r;
            const double a = exp(delta * A);
            const float *xt = x + (tok * H + h) * (int64_t)P;
            const float *Bt = B + (tok * G + g) * (int64_t)N;
            const double *prev = (t == t0) ? ck + k * PN : seg + (t - 1 - t0) * PN;
            double *cur = seg + (t - t0) * PN;
            for (int p = 0; p < P; ++p)
                for (int n = 0; n < N; ++n)
                    cur[(int64_t)p * N + n] = a * prev[(int64_t)p * N + n] + delta * (double)xt[p] * (double)Bt[n];
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const int64_t tok = tok0 + t;
            const double r = (double)dt[tok * H + h];
            const double delta = dt_softplus ? softplus(r) : r;
            const double a = exp(delta * A);
            const float *xt = x + (tok * H + h) * (int64_t)P;
            const float *dyt = dy + (tok * H + h) * (int64_t)P;
            const float *Bt = B + (tok * G + g) * (int64_t)N;
            const float *Ct = C + (tok * G + g) * (int64_t)N;
            const double *cur = seg + (t - t0) * PN;
            const double *prev = (t == t0) ? ck + k * PN : seg + (t - 1 - t0) * PN;
            double ddelta = 0.0, gh = 0.0;
            for (int p = 0; p < P; ++p) {
                const double dyp = (double)dyt[p], xp = (double)xt[p];
                double gb = 0.0;
                for (int n = 0; n < N; ++n) {
                    double *gp = gst + (int64_t)p * N + n;
                    *gp += dyp * (double)Ct[n];                 /* G_t */
                    gb += *gp * (double)Bt[n];
                    gh += *gp * prev[(int64_t)p * N + n];
                    dC_out[(t)*N + n] += dyp * cur[(int64_t)p * N + n];
                    dB_out[(t)*N + n] += delta * xp * *gp;
                }
                dx_out[t * P + p] = Dh * dyp + delta * gb;
                ddelta += xp * gb;
                dDh += dyp * xp;
            }
            ddelta += A * a * gh;
            dA += delta * a * gh;
            ddt_out[t] = dt_softplus ? ddelta * sigmoid(r) : ddelta;
            for (int64_t i = 0; i < PN; ++i) gst[i] *= a;   /* a_t G_t, for step t - 1 */
        }
    }
    if (dinit_out) memcpy(dinit_out, gst, sizeof(double) * (size_t)PN);
    *dAlog_out = A * dA;
    *dD_out = dDh;
    free(ck); free(seg); free(gst);
    return 0;
}

/*
 * Gradients for every (sequence, head) pair of a batch.  Inputs as for
 * ssd_ref_pairs plus dy (tokens, H, P) and dfinal (nseq, H, P, N, may be
 * NULL).  Outputs (double, zeroed here): dx (tokens, H, P), ddt (tokens, H),
 * dB and dC (tokens, G, N), dA_log and dD (H), dinit (nseq, H, P, N).
 */
int ssd_ref_bwd(int nseq, const int64_t *seq_start, const int64_t *seq_len,
                int H, int P, int N, int G, int dt_softplus,
                const float *x, const float *dt, const float *A_log,
                const float *B, const float *C, const float *D, const float *init,
                const float *dy, const float *dfinal, int64_t tokens,
                double *dx, double *ddt, double *dB, double *dC, double *dA_log,
                double *dD, double *dinit, int nthreads)
{
    if (nseq < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G != 0 || tokens < 0)
        return -1;
    if (!x || !dt || !A_log || !B || !C || !dy || !dx || !ddt || !dB || !dC || !dA_log || !dD || !dinit)
        return -1;
    const int64_t PN = (int64_t)P * N;
    memset(dx, 0, sizeof(double) * (size_t)(tokens * H * P));
    memset(ddt, 0, sizeof(double) * (size_t)(tokens * H));
    memset(dB, 0, sizeof(double) * (size_t)(tokens * G * N));
    memset(dC, 0, sizeof(double) * (size_t)(tokens * G * N));
    memset(dA_log, 0, sizeof(double) * (size_t)H);
    memset(dD, 0, sizeof(double) * (size_t)H);
    memset(dinit, 0, sizeof(double) * (size_t)(nseq * H * PN));
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int npairs = nseq * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < npairs; ++i) {
        const int s = i / H, h = i % H, g = h / (H / G);
        const int64_t t0 = seq_start[s], len = seq_len[s];
        double *px = (double *)malloc(sizeof(double) * (size_t)((len > 0 ? len : 1) * P));
        double *pdt = (double *)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
        double *pB = (double *)calloc((size_t)((len > 0 ? len : 1) * N), sizeof(double));
        double *pC = (double *)calloc((size_t)((len > 0 ? len : 1) * N), sizeof(double));
        double dal = 0.0, dd = 0.0;
        const float *init_sh = init ? init + ((int64_t)s * H + h) * PN : NULL;
        const float *dfin_sh = dfinal ? dfinal + ((int64_t)s * H + h) * PN : NULL;
        if (!px || !pdt || !pB || !pC ||
            ssd_ref_bwd_one(t0, len, h, H, P, N, G, dt_softplus, x, dt, A_log, B, C, D, init_sh, dy,
                            dfin_sh, px, pdt, pB, pC, &dal, &dd, dinit + ((int64_t)s * H + h) * PN) != 0) {
#pragma omp atomic write
            bad = 1;
        } else {
            for (int64_t t = 0; t < len; ++t) {
                for (int p = 0; p < P; ++p) dx[((t0 + t) * H + h) * P + p] = px[t * P + p];
                ddt[(t0 + t) * H + h] = pdt[t];
                for (int n = 0; n < N; ++n) {
#pragma omp atomic
                    dB[((t0 + t) * G + g) * N + n] += pB[t * N + n];
#pragma omp atomic
                    dC[((t0 + t) * G + g) * N + n] += pC[t * N + n];
                }
            }
#pragma omp atomic
            dA_log[h] += dal;
#pragma omp atomic
            dD[h] += dd;
        }
        free(px); free(pdt); free(pB); free(pC);
    }
    return bad ? -1 : 0;
}
