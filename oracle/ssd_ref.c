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
