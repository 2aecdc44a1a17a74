// CUDA-core (SIMT) path of the SSD forward: the chunked block decomposition
// of "Transformers are SSMs", Sec. 6, as four kernels with fp32 arithmetic.
// It serves float32 inputs (where bf16 tensor-core operands would not meet a
// 1e-4 tolerance) and every shape the tensor-core path does not take.
//
//   chunk_cumsum   delta = softplus(dt), dA = delta * A, inclusive prefix
//                  sum of dA inside each chunk (the 1-SS mask's exponents,
//                  Sec. 3.2.2 / Listing 1 `segsum`)
//   chunk_state    S_c = sum_l exp(cs_last - cs_l) delta_l x_l (outer) B_l:
//                  the chunk's final state from a zero start (Sec. 6.2,
//                  right factor)
//   state_passing  H_c = exp(cs_last(c-1)) H_{c-1} + S_{c-1}, H_0 = initial
//                  state: the state entering every chunk (Sec. 6.2, centre
//                  factor, evaluated as the sequential scalar scan of App. B)
//   chunk_scan     y_l = sum_{s<=l} (C_l . B_s) exp(cs_l - cs_s) delta_s x_s
//                        + exp(cs_l) C_l . H_c + D x_l
//                  (Sec. 6.1 diagonal block + Sec. 6.2 left factor)
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 32;   // rows per smem tile

// ------------------------------------------------------------------ cumsum
template <typename T>
__global__ void __launch_bounds__(256)
chunk_cumsum_kernel(Plan plan, Dims d, const T *__restrict__ dt, const float *__restrict__ A_log,
                    float *__restrict__ cs, float *__restrict__ dv)
{
    __shared__ float s_warp[8];
    const int c = blockIdx.x;
    if (c >= *plan.count) return;
    const ChunkDesc ch = plan.chunks[c];
    const int h = blockIdx.y;
    const int l = threadIdx.x;          // blockDim.x == Q
    const float A = -expf(A_log[h]);
    float delta = 0.0f, dA = 0.0f;
    if (l < ch.len) {
        const float r = to_f32(dt[(size_t)(ch.tok0 + l) * d.H + h]);
        delta = d.dt_softplus ? fmaxf(r, 0.0f) + log1pf(expf(-fabsf(r))) : r;
        dA = delta * A;
    }
    // inclusive scan over the chunk
    float v = dA;
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if ((l & 31) >= o) v += u;
    }
    if ((l & 31) == 31) s_warp[l >> 5] = v;
    __syncthreads();
    float carry = 0.0f;
    for (int w = 0; w < (l >> 5); ++w) carry += s_warp[w];
    const size_t o = ((size_t)c * d.H + h) * d.Q + l;
    cs[o] = v + carry;
    dv[o] = delta;
}

// -------------------------------------------------------------- chunk_state
// Register tiles: each thread accumulates 4 x 4 outputs (four channels by four state columns)
// per item, at most two items at a time, from float4 rows of the shared tiles (rows padded to a
// multiple of 4 with zeros).
constexpr int kStateItems = 2;   // items per thread per pass

template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_state_kernel(Plan plan, Dims d, const T *__restrict__ x, const T *__restrict__ Bm,
                   const float *__restrict__ cs, const float *__restrict__ dv,
                   float *__restrict__ states)
{
    extern __shared__ float smem[];
    const int c = blockIdx.x;
    if (c >= *plan.count) return;
    const ChunkDesc ch = plan.chunks[c];
    const int h = blockIdx.y;
    const int g = h / d.heads_per_group;
    const int P = d.P, N = d.N, Q = d.Q;
    const int PA = (P + 3) & ~3, NA = (N + 3) & ~3;
    float *Xs = smem;                       // kTile x PA (weighted x)
    float *Bs = Xs + kTile * PA;            // kTile x NA
    float *w = Bs + kTile * NA;             // Q
    const float *csc = cs + ((size_t)c * d.H + h) * Q;
    const float *dvc = dv + ((size_t)c * d.H + h) * Q;
    const float cs_last = csc[Q - 1];
    for (int l = threadIdx.x; l < Q; l += kThreads)
        w[l] = l < ch.len ? __expf(fminf(cs_last - csc[l], 0.0f)) * dvc[l] : 0.0f;   // <= 0 up to rounding
    __syncthreads();

    const int NG = NA / 4, items = (PA / 4) * NG;
    float *out = states + ((size_t)c * d.H + h) * (size_t)P * N;
    for (int b0 = 0; b0 < items; b0 += kThreads * kStateItems) {
        float acc[kStateItems][4][4];
#pragma unroll
        for (int k = 0; k < kStateItems; ++k)
#pragma unroll
            for (int a2 = 0; a2 < 4; ++a2)
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) acc[k][a2][b2] = 0.0f;
        for (int l0 = 0; l0 < ch.len; l0 += kTile) {
            for (int i = threadIdx.x; i < kTile * PA; i += kThreads) {
                const int r = i / PA, p = i % PA;
                const int l = l0 + r;
                Xs[i] = l < ch.len && p < P ? w[l] * to_f32(x[((size_t)(ch.tok0 + l) * d.H + h) * P + p]) : 0.0f;
            }
            for (int i = threadIdx.x; i < kTile * NA; i += kThreads) {
                const int r = i / NA, n = i % NA;
                const int l = l0 + r;
                Bs[i] = l < ch.len && n < N ? to_f32(Bm[((size_t)(ch.tok0 + l) * d.G + g) * N + n]) : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kStateItems; ++k) {
                const int it = b0 + threadIdx.x + k * kThreads;
                if (it < items) {
                    const int p0 = 4 * (it / NG), n0 = 4 * (it % NG);
#pragma unroll 4
                    for (int j = 0; j < kTile; ++j) {
                        const float4 x4 = *reinterpret_cast<const float4 *>(&Xs[j * PA + p0]);
                        const float4 b4 = *reinterpret_cast<const float4 *>(&Bs[j * NA + n0]);
                        const float xv[4] = {x4.x, x4.y, x4.z, x4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                        for (int a2 = 0; a2 < 4; ++a2)
#pragma unroll
                            for (int b2 = 0; b2 < 4; ++b2) acc[k][a2][b2] = fmaf(xv[a2], bv[b2], acc[k][a2][b2]);
                    }
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int k = 0; k < kStateItems; ++k) {
            const int it = b0 + threadIdx.x + k * kThreads;
            if (it >= items) continue;
            const int p0 = 4 * (it / NG), n0 = 4 * (it % NG);
#pragma unroll
            for (int a2 = 0; a2 < 4; ++a2) {
                if (p0 + a2 >= P) break;
                float *row = out + (size_t)(p0 + a2) * N + n0;
                if (n0 + 4 <= N && (N & 3) == 0) {
                    *reinterpret_cast<float4 *>(row) = make_float4(acc[k][a2][0], acc[k][a2][1], acc[k][a2][2], acc[k][a2][3]);
                } else {
#pragma unroll
                    for (int b2 = 0; b2 < 4; ++b2)
                        if (n0 + b2 < N) row[b2] = acc[k][a2][b2];
                }
            }
        }
    }
}

// ------------------------------------------------------------ state_passing
__global__ void __launch_bounds__(kThreads)
state_passing_kernel(Plan plan, Dims d, const float *__restrict__ cs, float *__restrict__ states,
                     const float *__restrict__ init, float *__restrict__ final_states)
{
    const int s = blockIdx.x;
    const int h = blockIdx.y;
    const int PN = d.P * d.N;
    const int e = blockIdx.z * kThreads + threadIdx.x;
    if (e >= PN) return;
    const SeqDesc sq = plan.seqs[s];
    float hv = init ? init[((size_t)s * d.H + h) * PN + e] : 0.0f;
    // the chunks' states and decays are loaded in groups before the chain uses them, so the
    // chain waits on memory once per group, not once per chunk
    constexpr int kGroup = 8;
    for (int j0 = 0; j0 < sq.nchunks; j0 += kGroup) {
        float sv[kGroup], dk[kGroup];
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            const int c = sq.chunk0 + j0 + i;
            const bool has = j0 + i < sq.nchunks;
            sv[i] = has ? states[((size_t)c * d.H + h) * PN + e] : 0.0f;
            dk[i] = has ? __expf(cs[((size_t)c * d.H + h) * d.Q + d.Q - 1]) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            if (j0 + i < sq.nchunks) {
                const int c = sq.chunk0 + j0 + i;
                states[((size_t)c * d.H + h) * PN + e] = hv;     // state entering chunk c
                hv = fmaf(dk[i], hv, sv[i]);
            }
        }
    }
    if (final_states) final_states[((size_t)s * d.H + h) * PN + e] = hv;
}

// --------------------------------------------------------------- chunk_scan
template <typename T>
__global__ void __launch_bounds__(kThreads)
chunk_scan_kernel(Plan plan, Dims d, const T *__restrict__ x, const T *__restrict__ Bm,
                  const T *__restrict__ Cm, const float *__restrict__ D,
                  const float *__restrict__ cs, const float *__restrict__ dv,
                  const float *__restrict__ states, T *__restrict__ y)
{
    extern __shared__ float smem[];
    const int c = blockIdx.x;
    if (c >= *plan.count) return;
    const ChunkDesc ch = plan.chunks[c];
    const int l0 = blockIdx.z * kTile;
    if (l0 >= ch.len) return;
    const int h = blockIdx.y;
    const int g = h / d.heads_per_group;
    const int P = d.P, N = d.N, Q = d.Q;
    const int NS = N + 1, PS = P + 1;       // padded strides
    float *Cs = smem;                       // kTile x NS
    float *Bs = Cs + kTile * NS;            // kTile x NS
    float *Xs = Bs + kTile * NS;            // kTile x PS
    float *Hs = Xs + kTile * PS;            // kTile x PS  (32 state rows n, all p)
    float *Gm = Hs + kTile * PS;            // kTile x (kTile + 1)
    float *csl = Gm + kTile * (kTile + 1);  // kTile
    float *css = csl + kTile;               // kTile
    float *dvs = css + kTile;               // kTile
    const float *csc = cs + ((size_t)c * d.H + h) * Q;
    const float *dvc = dv + ((size_t)c * d.H + h) * Q;
    const float *Hc = states + ((size_t)c * d.H + h) * (size_t)P * N;   // state entering chunk

    for (int i = threadIdx.x; i < kTile * N; i += kThreads) {
        const int r = i / N, n = i % N;
        const int l = l0 + r;
        Cs[r * NS + n] = l < ch.len ? to_f32(Cm[((size_t)(ch.tok0 + l) * d.G + g) * N + n]) : 0.0f;
    }
    if (threadIdx.x < kTile) csl[threadIdx.x] = csc[min(l0 + (int)threadIdx.x, Q - 1)];
    __syncthreads();

    // this thread's outputs: e = threadIdx.x + i * kThreads over kTile x P
    constexpr int kMaxEPT = kTile * 128 / kThreads;  // P <= 128
    float acc[kMaxEPT];
#pragma unroll
    for (int i = 0; i < kMaxEPT; ++i) acc[i] = 0.0f;
    const int nout = kTile * P;

    // left factor: exp(cs_l) * sum_n C[l][n] H[p][n], over n tiles of kTile
    for (int n0 = 0; n0 < N; n0 += kTile) {
        for (int i = threadIdx.x; i < kTile * P; i += kThreads) {
            const int p = i / kTile, nn = i % kTile;
            const int n = n0 + nn;
            Hs[nn * PS + p] = n < N ? Hc[(size_t)p * N + n] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kMaxEPT; ++i) {
            const int e = threadIdx.x + i * kThreads;
            if (e < nout) {
                const int r = e / P, p = e % P;
                float a = acc[i];
                const int nmax = min(kTile, N - n0);
                for (int nn = 0; nn < nmax; ++nn) a = fmaf(Cs[r * NS + n0 + nn], Hs[nn * PS + p], a);
                acc[i] = a;
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < kMaxEPT; ++i) {
        const int e = threadIdx.x + i * kThreads;
        if (e < nout) acc[i] *= __expf(csl[e / P]);
    }

    // diagonal block: sum over s <= l of (C_l . B_s) exp(cs_l - cs_s) delta_s x_s
    for (int s0 = 0; s0 <= l0; s0 += kTile) {
        for (int i = threadIdx.x; i < kTile * N; i += kThreads) {
            const int r = i / N, n = i % N;
            const int s = s0 + r;
            Bs[r * NS + n] = s < ch.len ? to_f32(Bm[((size_t)(ch.tok0 + s) * d.G + g) * N + n]) : 0.0f;
        }
        for (int i = threadIdx.x; i < kTile * P; i += kThreads) {
            const int r = i / P, p = i % P;
            const int s = s0 + r;
            Xs[r * PS + p] = s < ch.len ? to_f32(x[((size_t)(ch.tok0 + s) * d.H + h) * P + p]) : 0.0f;
        }
        if (threadIdx.x < kTile) {
            const int s = s0 + threadIdx.x;
            css[threadIdx.x] = csc[min(s, Q - 1)];
            dvs[threadIdx.x] = s < ch.len ? dvc[s] : 0.0f;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kTile * kTile; i += kThreads) {
            const int r = i / kTile, j = i % kTile;
            const int l = l0 + r, s = s0 + j;
            float v = 0.0f;
            if (s <= l && s < ch.len) {
                float dot = 0.0f;
                for (int n = 0; n < N; ++n) dot = fmaf(Cs[r * NS + n], Bs[j * NS + n], dot);
                v = dot * __expf(fminf(csl[r] - css[j], 0.0f)) * dvs[j];   // s <= l: <= 0 up to rounding
            }
            Gm[r * (kTile + 1) + j] = v;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kMaxEPT; ++i) {
            const int e = threadIdx.x + i * kThreads;
            if (e < nout) {
                const int r = e / P, p = e % P;
                float a = acc[i];
                for (int j = 0; j < kTile; ++j) a = fmaf(Gm[r * (kTile + 1) + j], Xs[j * PS + p], a);
                acc[i] = a;
            }
        }
        __syncthreads();
    }

    const float Dh = D ? D[h] : 0.0f;
#pragma unroll
    for (int i = 0; i < kMaxEPT; ++i) {
        const int e = threadIdx.x + i * kThreads;
        if (e < nout) {
            const int r = e / P, p = e % P;
            const int l = l0 + r;
            if (l < ch.len) {
                const size_t o = ((size_t)(ch.tok0 + l) * d.H + h) * P + p;
                y[o] = from_f32<T>(acc[i] + Dh * to_f32(x[o]));
            }
        }
    }
}

size_t state_smem(const Dims &d)
{
    return sizeof(float) * (kTile * ((d.P + 3) & ~3) + kTile * ((d.N + 3) & ~3) + d.Q);
}
size_t scan_smem(const Dims &d)
{
    return sizeof(float) * (2 * kTile * (d.N + 1) + 2 * kTile * (d.P + 1) + kTile * (kTile + 1) + 3 * kTile);
}

template <typename T>
cudaError_t launch_typed(const Plan &plan, const Dims &d, const SimtArgs &a, cudaStream_t st, const Instr &ins)
{
    const T *x = static_cast<const T *>(a.x);
    const T *dt = static_cast<const T *>(a.dt);
    const T *Bm = static_cast<const T *>(a.B);
    const T *Cm = static_cast<const T *>(a.C);
    T *y = static_cast<T *>(a.y);
    const dim3 gc(plan.max_chunks, d.H);
    if (ins.begin) cudaEventRecord(ins.begin, st);
    chunk_cumsum_kernel<T><<<gc, d.Q, 0, st>>>(plan, d, dt, a.A_log, a.cs, a.dv);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    const size_t ss = state_smem(d);
    e = cudaFuncSetAttribute(chunk_state_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ss);
    if (e != cudaSuccess) return e;
    chunk_state_kernel<T><<<gc, kThreads, ss, st>>>(plan, d, x, Bm, a.cs, a.dv, a.states);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const dim3 gp(plan.nseq, d.H, (d.P * d.N + kThreads - 1) / kThreads);
    state_passing_kernel<<<gp, kThreads, 0, st>>>(plan, d, a.cs, a.states, a.init, a.final_states);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    const size_t sc = scan_smem(d);
    e = cudaFuncSetAttribute(chunk_scan_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc);
    if (e != cudaSuccess) return e;
    const dim3 gs(plan.max_chunks, d.H, (d.Q + kTile - 1) / kTile);
    if (ins.main) cudaEventRecord(ins.main, st);
    chunk_scan_kernel<T><<<gs, kThreads, sc, st>>>(plan, d, x, Bm, Cm, a.D, a.cs, a.dv, a.states, y);
    if (ins.end) cudaEventRecord(ins.end, st);
    return cudaGetLastError();
}

// Total log decay sum_t delta_t A of every (sequence, head): the sum of its
// chunks' last prefix sums.
__global__ void __launch_bounds__(kThreads)
seq_logdecay_kernel(Plan plan, Dims d, const float *__restrict__ cs, float *__restrict__ logdecay)
{
    const int i = blockIdx.x * kThreads + threadIdx.x;
    if (i >= plan.nseq * d.H) return;
    const int s = i / d.H, h = i % d.H;
    const SeqDesc sq = plan.seqs[s];
    float v = 0.0f;
    for (int j = 0; j < sq.nchunks; ++j) v += cs[((size_t)(sq.chunk0 + j) * d.H + h) * d.Q + d.Q - 1];
    logdecay[i] = v;
}

}  // namespace

cudaError_t launch_simt_states(const Plan &plan, const Dims &d, const SimtArgs &a, cudaStream_t st,
                               float *final_states)
{
    if (plan.max_chunks == 0) return cudaSuccess;
    const dim3 gc(plan.max_chunks, d.H);
    const size_t ss = state_smem(d);
    cudaError_t e;
    if (a.bf16) {
        chunk_cumsum_kernel<__nv_bfloat16><<<gc, d.Q, 0, st>>>(plan, d, static_cast<const __nv_bfloat16 *>(a.dt),
                                                                a.A_log, a.cs, a.dv);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = cudaFuncSetAttribute(chunk_state_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ss);
        if (e != cudaSuccess) return e;
        chunk_state_kernel<__nv_bfloat16><<<gc, kThreads, ss, st>>>(
            plan, d, static_cast<const __nv_bfloat16 *>(a.x), static_cast<const __nv_bfloat16 *>(a.B), a.cs, a.dv,
            a.states);
    } else {
        chunk_cumsum_kernel<float><<<gc, d.Q, 0, st>>>(plan, d, static_cast<const float *>(a.dt), a.A_log, a.cs,
                                                       a.dv);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        e = cudaFuncSetAttribute(chunk_state_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ss);
        if (e != cudaSuccess) return e;
        chunk_state_kernel<float><<<gc, kThreads, ss, st>>>(plan, d, static_cast<const float *>(a.x),
                                                            static_cast<const float *>(a.B), a.cs, a.dv, a.states);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 gp(plan.nseq, d.H, (d.P * d.N + kThreads - 1) / kThreads);
    state_passing_kernel<<<gp, kThreads, 0, st>>>(plan, d, a.cs, a.states, a.init, final_states);
    return cudaGetLastError();
}

cudaError_t launch_simt_summary(const Plan &plan, const Dims &d, const SimtArgs &a, float *end_states,
                                float *logdecay, cudaStream_t st)
{
    cudaError_t e = launch_simt_states(plan, d, a, st, end_states);
    if (e != cudaSuccess) return e;
    if (plan.max_chunks == 0) {
        // no tokens: zero end states (no initial state is applied in a summary)
        const dim3 gp(plan.nseq, d.H, (d.P * d.N + kThreads - 1) / kThreads);
        if (plan.nseq > 0)
            state_passing_kernel<<<gp, kThreads, 0, st>>>(plan, d, a.cs, a.states, nullptr, end_states);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const int n = plan.nseq * d.H;
    if (n > 0) seq_logdecay_kernel<<<(n + kThreads - 1) / kThreads, kThreads, 0, st>>>(plan, d, a.cs, logdecay);
    return cudaGetLastError();
}

cudaError_t launch_simt(const Plan &plan, const Dims &d, const SimtArgs &a, cudaStream_t stream,
                        const Instr &ins)
{
    if (plan.max_chunks == 0) {
        // nothing to compute; final states still equal the initial states
        const dim3 gp(plan.nseq, d.H, (d.P * d.N + kThreads - 1) / kThreads);
        if (a.final_states && plan.nseq > 0)
            state_passing_kernel<<<gp, kThreads, 0, stream>>>(plan, d, a.cs, a.states, a.init, a.final_states);
        return cudaGetLastError();
    }
    return a.bf16 ? launch_typed<__nv_bfloat16>(plan, d, a, stream, ins) : launch_typed<float>(plan, d, a, stream, ins);
}

}  // namespace ssd
