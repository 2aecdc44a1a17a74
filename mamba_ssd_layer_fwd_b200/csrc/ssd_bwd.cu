// Backward pass of the SSD layer on CUDA cores (fp32 arithmetic): the chunked
// block decomposition of "Transformers are SSMs", Sec. 6, run in reverse.
//
// With 32-token chunks c, per head: cs_l the inclusive cumsum of delta * A
// inside the chunk, H_c the state entering chunk c (recomputed with the
// forward's cumsum / chunk-state / state-passing kernels), and G_c = dL/dH_c:
//
//   U_c      = sum_l exp(cs_l) dy_l (outer) C_l                      (dstate kernel)
//   G_c      = U_c + exp(cs_last) G_{c+1},  G_nc = dL/dfinal,  dL/dinit = G_0
//                                                                    (reverse state passing)
// and inside chunk c (L[l,s] = exp(cs_l - cs_s) for s <= l, W = L o C B^T,
// e2_s = exp(cs_last - cs_s), Gn = G_{c+1}):
//
//   dx_s  = D dy_s + delta_s (sum_l W[l,s] dy_l + e2_s Gn B_s)
//   dB_s  = delta_s (sum_l L[l,s] (dy_l . x_s) C_l + e2_s Gn^T x_s)   (summed over the group's heads)
//   dC_l  = sum_s L[l,s] delta_s (dy_l . x_s) B_s + exp(cs_l) H_c^T dy_l
//   dcs_l = sum_{s<l} E[l,s] - sum_{l'>l} E[l',l] + exp(cs_l) dy_l . (H_c C_l) - F_l
//           + [l last] (sum_s F_s + exp(cs_last) <Gn, H_c>),
//           E[l,s] = W[l,s] delta_s (dy_l . x_s),  F_s = e2_s delta_s x_s . (Gn B_s)
//   d(dA)_k = sum_{l >= k} dcs_l          (dA = delta * A enters cs_l for every l >= k)
//   ddelta_k = A d(dA)_k + sum_l W[l,k] (dy_l . x_k) + e2_k x_k . (Gn B_k)
//   ddt = ddelta * sigmoid(dt) (softplus), dA_log = A sum_k delta_k d(dA)_k, dD = sum <dy, x>
//
// Every exponent above is a difference cs_l - cs_s with s <= l, <= 0 in exact
// arithmetic; the fp32 prefix sums can round it above 0 when |A| is huge, so
// it is clamped at 0.
//
// One CTA per (chunk, B/C group) loops over the group's heads, keeping the
// group's dB and dC tiles in shared memory, so they are written once, without
// atomics; dA_log and dD are summed with one atomic per (chunk, head).
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kBQ = 32;         // chunk length of the backward
constexpr int kBThreads = 256;
constexpr int kNT = 32;         // dstate columns per tile of H_c and G_{c+1}
// the chunk kernel's register tiles map 256 threads onto 32 x 32 token pairs and token x column tiles
static_assert(kBQ == 32 && kNT == 32 && kBThreads == 256, "the chunk kernel's thread mappings assume these sizes");

__device__ __forceinline__ float sigmoid_f32(float r)
{
    // 1 / (1 + e^-r), evaluated without overflow
    const float e = __expf(-fabsf(r));
    return r >= 0.0f ? 1.0f / (1.0f + e) : e / (1.0f + e);
}

// U_c[p][n] = sum_l exp(cs_l) dy_l[p] C_l[n], written into `ubuf` (the layout of the chunk states).
// Rows of the shared tiles are padded to a multiple of 4 (zeros); each thread accumulates a
// 4 x 4 register tile (four channels by four state columns) from float4 rows.
template <typename T>
__global__ void __launch_bounds__(kBThreads)
bwd_dstate_kernel(Plan plan, Dims d, const T *__restrict__ dy, const T *__restrict__ Cm,
                  const float *__restrict__ cs, float *__restrict__ ubuf)
{
    extern __shared__ float smem[];
    const int c = blockIdx.x;
    if (c >= *plan.count) return;
    const ChunkDesc ch = plan.chunks[c];
    const int h = blockIdx.y, g = h / d.heads_per_group;
    const int P = d.P, N = d.N;
    const int PA = (P + 3) & ~3, NA = (N + 3) & ~3;
    float *Ys = smem;                 // kBQ x PA (weighted dy)
    float *Cs = Ys + kBQ * PA;        // kBQ x NA
    const float *csc = cs + ((size_t)c * d.H + h) * kBQ;
    for (int i = threadIdx.x; i < kBQ * PA; i += kBThreads) {
        const int l = i / PA, p = i % PA;
        Ys[i] = l < ch.len && p < P ? __expf(csc[l]) * to_f32(dy[((size_t)(ch.tok0 + l) * d.H + h) * P + p]) : 0.0f;
    }
    for (int i = threadIdx.x; i < kBQ * NA; i += kBThreads) {
        const int l = i / NA, n = i % NA;
        Cs[i] = l < ch.len && n < N ? to_f32(Cm[((size_t)(ch.tok0 + l) * d.G + g) * N + n]) : 0.0f;
    }
    __syncthreads();
    const int NG = NA / 4, items = (PA / 4) * NG;
    float *out = ubuf + ((size_t)c * d.H + h) * (size_t)P * N;
    for (int it = threadIdx.x; it < items; it += kBThreads) {
        const int p0 = 4 * (it / NG), n0 = 4 * (it % NG);
        float acc[4][4];
#pragma unroll
        for (int a2 = 0; a2 < 4; ++a2)
#pragma unroll
            for (int b2 = 0; b2 < 4; ++b2) acc[a2][b2] = 0.0f;
#pragma unroll 4
        for (int l = 0; l < kBQ; ++l) {
            const float4 y4 = *reinterpret_cast<const float4 *>(&Ys[l * PA + p0]);
            const float4 c4 = *reinterpret_cast<const float4 *>(&Cs[l * NA + n0]);
            const float yv[4] = {y4.x, y4.y, y4.z, y4.w}, cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int a2 = 0; a2 < 4; ++a2)
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2) acc[a2][b2] = fmaf(yv[a2], cv[b2], acc[a2][b2]);
        }
#pragma unroll
        for (int a2 = 0; a2 < 4; ++a2) {
            if (p0 + a2 >= P) break;
            float *row = out + (size_t)(p0 + a2) * N + n0;
            if (n0 + 4 <= N && (N & 3) == 0) {
                *reinterpret_cast<float4 *>(row) = make_float4(acc[a2][0], acc[a2][1], acc[a2][2], acc[a2][3]);
            } else {
#pragma unroll
                for (int b2 = 0; b2 < 4; ++b2)
                    if (n0 + b2 < N) row[b2] = acc[a2][b2];
            }
        }
    }
}

// G_c = U_c + exp(cs_last(c)) G_{c+1} from the last chunk of each sequence to
// the first; the buffer slot of chunk c receives G_{c+1} (dL/d of the state
// leaving the chunk), and dL/dinit = G_0.
__global__ void __launch_bounds__(kBThreads)
bwd_state_passing_kernel(Plan plan, Dims d, const float *__restrict__ cs, float *__restrict__ gbuf,
                         const float *__restrict__ dfinal, float *__restrict__ dinit)
{
    const int s = blockIdx.x, h = blockIdx.y;
    const int PN = d.P * d.N;
    const int e = blockIdx.z * kBThreads + threadIdx.x;
    if (e >= PN) return;
    const SeqDesc sq = plan.seqs[s];
    float gv = dfinal ? dfinal[((size_t)s * d.H + h) * PN + e] : 0.0f;
    // loads in groups of chunks ahead of the chain (see state_passing_kernel)
    constexpr int kGroup = 8;
    for (int j0 = sq.nchunks - 1; j0 >= 0; j0 -= kGroup) {
        float uv[kGroup], dk[kGroup];
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            const int c = sq.chunk0 + j0 - i;
            const bool has = j0 - i >= 0;
            uv[i] = has ? gbuf[((size_t)c * d.H + h) * PN + e] : 0.0f;
            dk[i] = has ? __expf(cs[((size_t)c * d.H + h) * kBQ + kBQ - 1]) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            if (j0 - i >= 0) {
                gbuf[((size_t)(sq.chunk0 + j0 - i) * d.H + h) * PN + e] = gv;
                gv = fmaf(dk[i], gv, uv[i]);
            }
        }
    }
    if (dinit) dinit[((size_t)s * d.H + h) * PN + e] = gv;
}

struct BwdArgs {
    const void *x, *dt, *B, *C, *dy;
    const float *A_log, *D;
    const float *cs, *dv, *states, *gbuf;
    float *dx, *ddt, *dA_log, *dB, *dC, *dD;
};

// Head-channel rows are padded to PA = P rounded up to 4 (zeros) plus 4, so that the
// register-tiled products read them as float4.
size_t chunk_smem_floats(int P, int N)
{
    const int PA = (P + 3) & ~3, PS = PA + 4, NS = N + 1, QS = kBQ + 1;
    return (size_t)2 * kBQ * NS        // B, C
           + 2 * kBQ * NS              // dB, dC accumulators
           + 2 * kBQ * PS              // x, dy
           + 3 * kBQ * QS              // C B^T, L, dy . x
           + 2 * kNT * PS              // H_c, G_{c+1} tiles, transposed
           + 8 * kBQ + 32;             // per-token vectors, reductions
}

__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc)
{
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}

template <typename T>
__global__ void __launch_bounds__(kBThreads, 2)   // two CTAs per SM (registers and shared memory)
bwd_chunk_kernel(Plan plan, Dims d, BwdArgs a)
{
    extern __shared__ float smem[];
    const int c = blockIdx.x;
    if (c >= *plan.count) return;
    const ChunkDesc ch = plan.chunks[c];
    const int g = blockIdx.y;
    const int P = d.P, N = d.N, H = d.H, G = d.G;
    const int PA = (P + 3) & ~3, PG = PA / 4, PS = PA + 4, NS = N + 1, QS = kBQ + 1;
    const int len = ch.len;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *Bs = smem;                      // kBQ x NS
    float *Cs = Bs + kBQ * NS;
    float *dBs = Cs + kBQ * NS;            // group accumulators
    float *dCs = dBs + kBQ * NS;
    float *Xs = dCs + kBQ * NS;            // kBQ x PS (current head)
    float *DYs = Xs + kBQ * PS;
    float *CB = DYs + kBQ * PS;            // kBQ x QS: C_l . B_s
    float *Lm = CB + kBQ * QS;             // exp(cs_l - cs_s), s <= l < len
    float *DX = Lm + kBQ * QS;             // M = L o (dy . x): L[l, s] (dy_l . x_s)
    float *Ht = DX + kBQ * QS;             // kNT x PS: Ht[nn][p] = H_c[p][n0 + nn]
    float *Gt = Ht + kNT * PS;             // the same for G_{c+1}
    float *css = Gt + kNT * PS;            // kBQ
    float *dls = css + kBQ;                // delta (0 past the chunk's end)
    float *fxs = dls + kBQ;                // x_s . (Gn B_s)
    float *dhc = fxs + kBQ;                // dy_l . (H C_l)
    float *rowv = dhc + kBQ;
    float *colv = rowv + kBQ;
    float *red = colv + kBQ;               // [0] <Gn, H>, [1] dD partial

    const T *x = static_cast<const T *>(a.x), *dy = static_cast<const T *>(a.dy);
    const T *Bm = static_cast<const T *>(a.B), *Cm = static_cast<const T *>(a.C);
    const T *dtp = static_cast<const T *>(a.dt);

    for (int i = tid; i < kBQ * N; i += kBThreads) {
        const int r = i / N, n = i % N;
        const bool v = r < len;
        const size_t o = ((size_t)(ch.tok0 + r) * G + g) * N + n;
        Bs[r * NS + n] = v ? to_f32(Bm[o]) : 0.0f;
        Cs[r * NS + n] = v ? to_f32(Cm[o]) : 0.0f;
        dBs[r * NS + n] = 0.0f;
        dCs[r * NS + n] = 0.0f;
    }
    __syncthreads();
    // C_l . B_s for the whole group
    for (int i = tid; i < kBQ * kBQ; i += kBThreads) {
        const int l = i / kBQ, s = i % kBQ;
        float v = 0.0f;
        for (int n = 0; n < N; ++n) v = fmaf(Cs[l * NS + n], Bs[s * NS + n], v);
        CB[l * QS + s] = v;
    }

    // pad columns p in [P, PA) of the x, dy, H and G tiles: zero, never written again
    for (int i = tid; i < (2 * kBQ + 2 * kNT) * (PA - P); i += kBThreads) {
        const int r = i / (PA - P), p = P + i % (PA - P);
        (r < 2 * kBQ ? Xs : Ht)[(r % (2 * kBQ)) * PS + p] = 0.0f;   // Xs, DYs and Ht, Gt are adjacent
    }
    // the dx terms are computed in (token pair, 4-channel group) items, at most two per thread
    constexpr int kMaxItems = (kBQ / 2) * (128 / 4) / kBThreads;
    const int n_items = (kBQ / 2) * PG;
    for (int h = g * d.heads_per_group; h < (g + 1) * d.heads_per_group; ++h) {
        const float A = -__expf(a.A_log[h]);
        const float Dh = a.D ? a.D[h] : 0.0f;
        const float *csc = a.cs + ((size_t)c * H + h) * kBQ;
        const float *dvc = a.dv + ((size_t)c * H + h) * kBQ;
        __syncthreads();   // previous head done with Xs, DYs, Lm, DX, per-token vectors
        for (int i = tid; i < kBQ * P; i += kBThreads) {
            const int r = i / P, p = i % P;
            const bool v = r < len;
            const size_t o = ((size_t)(ch.tok0 + r) * H + h) * P + p;
            Xs[r * PS + p] = v ? to_f32(x[o]) : 0.0f;
            DYs[r * PS + p] = v ? to_f32(dy[o]) : 0.0f;
        }
        if (tid < kBQ) {
            css[tid] = csc[tid];
            dls[tid] = tid < len ? dvc[tid] : 0.0f;
            fxs[tid] = 0.0f;
            dhc[tid] = 0.0f;
        }
        if (tid < 2) red[tid] = 0.0f;
        __syncthreads();
        // dy_l . x_s for tokens l, l + 16 by s, s + 16 per thread (float4 rows; the lanes of a
        // warp read rows 17 float4 apart, which fall in distinct bank groups)
        {
            const int l0 = tid >> 4, s0 = tid & 15;
            float v[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
            for (int p0 = 0; p0 < PA; p0 += 4) {
                const float4 ya = *reinterpret_cast<const float4 *>(&DYs[l0 * PS + p0]);
                const float4 yb = *reinterpret_cast<const float4 *>(&DYs[(l0 + 16) * PS + p0]);
                const float4 xa = *reinterpret_cast<const float4 *>(&Xs[s0 * PS + p0]);
                const float4 xb = *reinterpret_cast<const float4 *>(&Xs[(s0 + 16) * PS + p0]);
                v[0][0] = dot4(ya, xa, v[0][0]); v[0][1] = dot4(ya, xb, v[0][1]);
                v[1][0] = dot4(yb, xa, v[1][0]); v[1][1] = dot4(yb, xb, v[1][1]);
            }
#pragma unroll
            for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
                for (int b2 = 0; b2 < 2; ++b2) {
                    const int l = l0 + 16 * a2, s = s0 + 16 * b2;
                    const float lm = (s <= l && l < len) ? __expf(fminf(css[l] - css[s], 0.0f)) : 0.0f;
                    Lm[l * QS + s] = lm;
                    DX[l * QS + s] = lm * v[a2][b2];
                }
        }
        __syncthreads();
        // per token: row and column sums of E and of W o (dy . x); dD.  The sums for d(cs)
        // leave out the diagonal, whose terms cancel exactly (d exp(cs_l - cs_l) = 0): left in,
        // their rounding would be multiplied by A, which can be large
        if (tid < kBQ) {
            const int t = tid;
            float row = 0.0f, col = 0.0f;
            for (int s = 0; s < t; ++s) row = fmaf(CB[t * QS + s] * DX[t * QS + s], dls[s], row);
            for (int l = t + 1; l < kBQ; ++l) col = fmaf(CB[l * QS + t], DX[l * QS + t], col);
            rowv[t] = row;
            colv[t] = col;
            float dd = t < len ? DX[t * QS + t] : 0.0f;       // L[t, t] = 1
            for (int o = 16; o > 0; o >>= 1) dd += __shfl_xor_sync(0xffffffffu, dd, o);
            if (t == 0) red[1] = dd;
        }
        // intra terms of dx (into registers): sum over l >= s of W[l, s] dy_l, W = L o CB (zero above
        // the diagonal), two tokens by four channels per item
        float dxa[kMaxItems][2][4], gba[kMaxItems][2][4];
#pragma unroll
        for (int k = 0; k < kMaxItems; ++k) {
#pragma unroll
            for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
                for (int i = 0; i < 4; ++i) dxa[k][a2][i] = gba[k][a2][i] = 0.0f;
            const int item = tid + k * kBThreads;
            if (item < n_items) {
                const int s0 = 2 * (item / PG), p0 = 4 * (item % PG);
                for (int l = s0; l < kBQ; ++l) {
                    const float w0 = Lm[l * QS + s0] * CB[l * QS + s0];
                    const float w1 = Lm[l * QS + s0 + 1] * CB[l * QS + s0 + 1];
                    const float4 y4 = *reinterpret_cast<const float4 *>(&DYs[l * PS + p0]);
                    dxa[k][0][0] = fmaf(w0, y4.x, dxa[k][0][0]); dxa[k][0][1] = fmaf(w0, y4.y, dxa[k][0][1]);
                    dxa[k][0][2] = fmaf(w0, y4.z, dxa[k][0][2]); dxa[k][0][3] = fmaf(w0, y4.w, dxa[k][0][3]);
                    dxa[k][1][0] = fmaf(w1, y4.x, dxa[k][1][0]); dxa[k][1][1] = fmaf(w1, y4.y, dxa[k][1][1]);
                    dxa[k][1][2] = fmaf(w1, y4.z, dxa[k][1][2]); dxa[k][1][3] = fmaf(w1, y4.w, dxa[k][1][3]);
                }
            }
        }
        // intra terms of dB, dC
        // dB_s += delta_s sum_{l >= s} M[l, s] C_l and dC_s += sum_{t <= s} M[s, t] delta_t B_t
        // (M zero above the diagonal): two tokens by four state columns nq + NQ k per item, so
        // that the lanes of a warp read consecutive columns
        const int NQ = (N + 3) / 4;
        for (int it = tid; it < (kBQ / 2) * NQ; it += kBThreads) {
            const int s0 = 2 * (it / NQ), nq = it % NQ;
            float vb[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
            float vc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
            for (int l = s0; l < kBQ; ++l) {
                const float m0 = DX[l * QS + s0], m1 = DX[l * QS + s0 + 1];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = nq + NQ * k;
                    const float cv = n < N ? Cs[l * NS + n] : 0.0f;
                    vb[0][k] = fmaf(m0, cv, vb[0][k]);
                    vb[1][k] = fmaf(m1, cv, vb[1][k]);
                }
            }
            for (int t = 0; t <= s0 + 1; ++t) {
                const float q0 = DX[s0 * QS + t] * dls[t], q1 = DX[(s0 + 1) * QS + t] * dls[t];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = nq + NQ * k;
                    const float bv = n < N ? Bs[t * NS + n] : 0.0f;
                    vc[0][k] = fmaf(q0, bv, vc[0][k]);
                    vc[1][k] = fmaf(q1, bv, vc[1][k]);
                }
            }
#pragma unroll
            for (int a2 = 0; a2 < 2; ++a2) {
                const int s = s0 + a2;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int n = nq + NQ * k;
                    if (n < N) {
                        dBs[s * NS + n] += dls[s] * vb[a2][k];
                        dCs[s * NS + n] += vc[a2][k];
                    }
                }
            }
        }
        // inter terms, over tiles of kNT dstate columns of H_c and G_{c+1} (stored transposed)
        const float *Hc = a.states + ((size_t)c * H + h) * (size_t)P * N;
        const float *Gn = a.gbuf + ((size_t)c * H + h) * (size_t)P * N;
        float ghp = 0.0f;
        // each tile is fetched into registers one tile ahead, so its global loads are in flight
        // while the previous tile's products run
        constexpr int kTL = 128 * kNT / kBThreads;     // tile elements per thread (P <= 128)
        float hn[kTL], gn[kTL];
        auto fetch = [&](int t0) {
            const int tn = min(kNT, N - t0);
#pragma unroll
            for (int k = 0; k < kTL; ++k) {
                const int i = tid + k * kBThreads, p = i / kNT, nn = i % kNT;
                const bool v = i < P * kNT && nn < tn;
                hn[k] = v ? Hc[(size_t)p * N + t0 + nn] : 0.0f;
                gn[k] = v ? Gn[(size_t)p * N + t0 + nn] : 0.0f;
            }
        };
        fetch(0);
        for (int n0 = 0; n0 < N; n0 += kNT) {
            const int nt = min(kNT, N - n0);
            __syncthreads();
#pragma unroll
            for (int k = 0; k < kTL; ++k) {
                const int i = tid + k * kBThreads, p = i / kNT, nn = i % kNT;
                if (i < P * kNT) {
                    Ht[nn * PS + p] = hn[k];
                    Gt[nn * PS + p] = gn[k];
                    ghp = fmaf(hn[k], gn[k], ghp);
                }
            }
            if (n0 + kNT < N) fetch(n0 + kNT);
            __syncthreads();
            // (Gn B_s)[p] over this tile, per (token pair, channel group) item
#pragma unroll
            for (int k = 0; k < kMaxItems; ++k) {
                const int item = tid + k * kBThreads;
                if (item < n_items) {
                    const int s0 = 2 * (item / PG), p0 = 4 * (item % PG);
                    for (int nn = 0; nn < nt; ++nn) {
                        const float b0 = Bs[s0 * NS + n0 + nn], b1 = Bs[(s0 + 1) * NS + n0 + nn];
                        const float4 g4 = *reinterpret_cast<const float4 *>(&Gt[nn * PS + p0]);
                        gba[k][0][0] = fmaf(b0, g4.x, gba[k][0][0]); gba[k][0][1] = fmaf(b0, g4.y, gba[k][0][1]);
                        gba[k][0][2] = fmaf(b0, g4.z, gba[k][0][2]); gba[k][0][3] = fmaf(b0, g4.w, gba[k][0][3]);
                        gba[k][1][0] = fmaf(b1, g4.x, gba[k][1][0]); gba[k][1][1] = fmaf(b1, g4.y, gba[k][1][1]);
                        gba[k][1][2] = fmaf(b1, g4.z, gba[k][1][2]); gba[k][1][3] = fmaf(b1, g4.w, gba[k][1][3]);
                    }
                }
            }
            // x_s . Gn[:, n] and dy_s . H[:, n]: tokens s0, s0 + 1 by columns nn, nn + 16 per thread
            {
                const int s0 = 2 * (tid >> 4), nb = tid & 15;
                float xg[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}}, dh[2][2] = {{0.0f, 0.0f}, {0.0f, 0.0f}};
                for (int p0 = 0; p0 < PA; p0 += 4) {
                    const float4 xa = *reinterpret_cast<const float4 *>(&Xs[s0 * PS + p0]);
                    const float4 xb = *reinterpret_cast<const float4 *>(&Xs[(s0 + 1) * PS + p0]);
                    const float4 ya = *reinterpret_cast<const float4 *>(&DYs[s0 * PS + p0]);
                    const float4 yb = *reinterpret_cast<const float4 *>(&DYs[(s0 + 1) * PS + p0]);
                    const float4 g0 = *reinterpret_cast<const float4 *>(&Gt[nb * PS + p0]);
                    const float4 g1 = *reinterpret_cast<const float4 *>(&Gt[(nb + 16) * PS + p0]);
                    const float4 h0 = *reinterpret_cast<const float4 *>(&Ht[nb * PS + p0]);
                    const float4 h1 = *reinterpret_cast<const float4 *>(&Ht[(nb + 16) * PS + p0]);
                    xg[0][0] = dot4(xa, g0, xg[0][0]); xg[0][1] = dot4(xa, g1, xg[0][1]);
                    xg[1][0] = dot4(xb, g0, xg[1][0]); xg[1][1] = dot4(xb, g1, xg[1][1]);
                    dh[0][0] = dot4(ya, h0, dh[0][0]); dh[0][1] = dot4(ya, h1, dh[0][1]);
                    dh[1][0] = dot4(yb, h0, dh[1][0]); dh[1][1] = dot4(yb, h1, dh[1][1]);
                }
                float fx[2] = {0.0f, 0.0f}, dc[2] = {0.0f, 0.0f};
#pragma unroll
                for (int a2 = 0; a2 < 2; ++a2) {
                    const int s = s0 + a2;
                    const float e2 = __expf(fminf(css[kBQ - 1] - css[s], 0.0f));
                    const float ec = s < len ? __expf(css[s]) : 0.0f;
#pragma unroll
                    for (int b2 = 0; b2 < 2; ++b2) {
                        const int nn = nb + 16 * b2;
                        if (nn < nt) {
                            const int n = n0 + nn;
                            dBs[s * NS + n] += dls[s] * e2 * xg[a2][b2];
                            dCs[s * NS + n] += ec * dh[a2][b2];
                            fx[a2] = fmaf(xg[a2][b2], Bs[s * NS + n], fx[a2]);
                            dc[a2] = fmaf(dh[a2][b2], Cs[s * NS + n], dc[a2]);
                        }
                    }
                }
                // over the 16 lanes holding this token pair (lanes 16 t .. 16 t + 15 of the warp)
#pragma unroll
                for (int o = 8; o > 0; o >>= 1)
#pragma unroll
                    for (int a2 = 0; a2 < 2; ++a2) {
                        fx[a2] += __shfl_xor_sync(0xffffffffu, fx[a2], o);
                        dc[a2] += __shfl_xor_sync(0xffffffffu, dc[a2], o);
                    }
                if (nb == 0) {
                    atomicAdd(&fxs[s0], fx[0]);
                    atomicAdd(&fxs[s0 + 1], fx[1]);
                    atomicAdd(&dhc[s0], dc[0]);
                    atomicAdd(&dhc[s0 + 1], dc[1]);
                }
            }
        }
        for (int o = 16; o > 0; o >>= 1) ghp += __shfl_xor_sync(0xffffffffu, ghp, o);
        if (lane == 0) atomicAdd(&red[0], ghp);
        __syncthreads();
        // dx = D dy + delta (intra + e2 Gn B)
#pragma unroll
        for (int k = 0; k < kMaxItems; ++k) {
            const int item = tid + k * kBThreads;
            if (item < n_items) {
                const int s0 = 2 * (item / PG), p0 = 4 * (item % PG);
#pragma unroll
                for (int a2 = 0; a2 < 2; ++a2) {
                    const int s = s0 + a2;
                    if (s < len) {
                        const float e2 = __expf(fminf(css[kBQ - 1] - css[s], 0.0f));
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (p0 + i < P)
                                a.dx[((size_t)(ch.tok0 + s) * H + h) * P + p0 + i] =
                                    fmaf(Dh, DYs[s * PS + p0 + i], dls[s] * (dxa[k][a2][i] + e2 * gba[k][a2][i]));
                    }
                }
            }
        }
        // d(cs) -> d(dA) (reverse cumsum) -> ddelta, ddt, dA_log, dD
        if (warp == 0) {
            const int t = lane;            // kBQ == 32
            const float e2 = __expf(fminf(css[kBQ - 1] - css[t], 0.0f));
            const float F = e2 * dls[t] * fxs[t];
            float Fsum = F;
            for (int o = 16; o > 0; o >>= 1) Fsum += __shfl_xor_sync(0xffffffffu, Fsum, o);
            float dcs = rowv[t] - dls[t] * colv[t] + (t < len ? __expf(css[t]) : 0.0f) * dhc[t] - F;
            const float colx = colv[t] + CB[t * QS + t] * DX[t * QS + t];   // with the diagonal
            if (t == kBQ - 1) dcs += Fsum + __expf(css[kBQ - 1]) * red[0];
            // reverse inclusive scan: ddA_k = sum_{l >= k} dcs_l
            float v = dcs;
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_down_sync(0xffffffffu, v, o);
                if (t + o < 32) v += u;
            }
            const float ddelta = A * v + colx + e2 * fxs[t];
            float da = dls[t] * v;
            for (int o = 16; o > 0; o >>= 1) da += __shfl_xor_sync(0xffffffffu, da, o);
            if (t < len) {
                const size_t o = (size_t)(ch.tok0 + t) * H + h;
                const float r = to_f32(dtp[o]);
                a.ddt[o] = d.dt_softplus ? ddelta * sigmoid_f32(r) : ddelta;
            }
            if (t == 0) {
                atomicAdd(&a.dA_log[h], A * da);
                atomicAdd(&a.dD[h], red[1]);
            }
        }
    }
    __syncthreads();
    for (int i = tid; i < len * N; i += kBThreads) {
        const int r = i / N, n = i % N;
        const size_t o = ((size_t)(ch.tok0 + r) * G + g) * N + n;
        a.dB[o] = dBs[r * NS + n];
        a.dC[o] = dCs[r * NS + n];
    }
}

}  // namespace

bool bwd_supported(const ssd_fwd_params &p)
{
    const size_t smem = chunk_smem_floats(p.headdim, p.dstate) * sizeof(float);
    return p.path != SSD_PATH_TENSOR && p.headdim <= 128 && smem <= 227 * 1024;
}

size_t bwd_chunk_count(const ssd_fwd_params &p)
{
    const long long Q = kBQ;
    return p.num_seqs > 0 ? (size_t)((p.seqlen + Q - 1) / Q + p.num_seqs)
                          : (size_t)p.batch * (size_t)((p.seqlen + Q - 1) / Q);
}

int bwd_chunk_len() { return kBQ; }

cudaError_t launch_bwd(const Plan &plan, const Dims &d, const SimtArgs &fa, const void *dy, const float *dfinal,
                       float *gbuf, float *dx, float *ddt, float *dA_log, float *dB, float *dC, float *dD,
                       float *dinit, bool bf16, cudaStream_t st)
{
    cudaError_t e;
    const long long tokens = d.tokens;
    if ((e = cudaMemsetAsync(dA_log, 0, sizeof(float) * d.H, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dD, 0, sizeof(float) * d.H, st)) != cudaSuccess) return e;
    if (tokens > 0 && (e = cudaMemsetAsync(dB, 0, sizeof(float) * tokens * d.G * d.N, st)) != cudaSuccess) return e;
    if (tokens > 0 && (e = cudaMemsetAsync(dC, 0, sizeof(float) * tokens * d.G * d.N, st)) != cudaSuccess) return e;
    if ((e = launch_simt_states(plan, d, fa, st)) != cudaSuccess) return e;
    const int PN = d.P * d.N;
    if (plan.max_chunks > 0) {
        const dim3 gc(plan.max_chunks, d.H);
        const size_t sd = sizeof(float) * kBQ * (((d.P + 3) & ~3) + ((d.N + 3) & ~3));
        if (bf16) {
            e = cudaFuncSetAttribute(bwd_dstate_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sd);
            if (e != cudaSuccess) return e;
            bwd_dstate_kernel<__nv_bfloat16><<<gc, kBThreads, sd, st>>>(
                plan, d, static_cast<const __nv_bfloat16 *>(dy), static_cast<const __nv_bfloat16 *>(fa.C), fa.cs, gbuf);
        } else {
            e = cudaFuncSetAttribute(bwd_dstate_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sd);
            if (e != cudaSuccess) return e;
            bwd_dstate_kernel<float><<<gc, kBThreads, sd, st>>>(plan, d, static_cast<const float *>(dy),
                                                                static_cast<const float *>(fa.C), fa.cs, gbuf);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (plan.nseq > 0) {
        const dim3 gp(plan.nseq, d.H, (PN + kBThreads - 1) / kBThreads);
        bwd_state_passing_kernel<<<gp, kBThreads, 0, st>>>(plan, d, fa.cs, gbuf, dfinal, dinit);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (plan.max_chunks == 0) return cudaSuccess;
    BwdArgs a;
    a.x = fa.x; a.dt = fa.dt; a.B = fa.B; a.C = fa.C; a.dy = dy;
    a.A_log = fa.A_log; a.D = fa.D;
    a.cs = fa.cs; a.dv = fa.dv; a.states = fa.states; a.gbuf = gbuf;
    a.dx = dx; a.ddt = ddt; a.dA_log = dA_log; a.dB = dB; a.dC = dC; a.dD = dD;
    const size_t sm = chunk_smem_floats(d.P, d.N) * sizeof(float);
    const dim3 gk(plan.max_chunks, d.G);
    if (bf16) {
        e = cudaFuncSetAttribute(bwd_chunk_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        bwd_chunk_kernel<__nv_bfloat16><<<gk, kBThreads, sm, st>>>(plan, d, a);
    } else {
        e = cudaFuncSetAttribute(bwd_chunk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        bwd_chunk_kernel<float><<<gk, kBThreads, sm, st>>>(plan, d, a);
    }
    return cudaGetLastError();
}

}  // namespace ssd
