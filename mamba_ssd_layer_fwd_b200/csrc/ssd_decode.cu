// ssd_decode_step: one token of the SSD's recurrent (linear) mode for every
// (batch row, head) - the decoding counterpart of ssd_fwd ("Transformers are
// SSMs", Sec. 3.4.1 eq. (8): the scalar recurrence with the state expanded by
// B and contracted by C; Sec. 2.4 for the selective parameters).
//
//     delta = softplus(dt[b, h])       a = exp(delta * -exp(A_log[h]))
//     state[b, h] <- a * state[b, h] + (delta * x[b, h, :]) (outer) B[b, g, :]
//     y[b, h, :]   = state[b, h] @ C[b, g, :] + D[h] * x[b, h, :]
//
// The state (P x N fp32 per row and head) is read and written once per call:
// the kernel is bound by HBM.  One CTA of 4 warps per (row, head); each warp owns P/4 state
// rows and walks them in groups of eight, so eight 16-byte loads per lane (16
// for dstate > 128) are in flight before any arithmetic; lane i covers columns 4i, 4i+1, ... of every
// 128-column slice, which makes each row access one coalesced 512-byte sweep.
// B and C of the row's group are loaded once per CTA into registers.
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecRows = 8;        // state rows in flight per warp

template <typename T> __device__ __forceinline__ void load4(const T *p, float (&v)[4]);
template <> __device__ __forceinline__ void load4<float>(const float *p, float (&v)[4])
{
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
template <> __device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4])
{
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&q.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&q.y);
    v[0] = __low2float(lo); v[1] = __high2float(lo);
    v[2] = __low2float(hi); v[3] = __high2float(hi);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// KS: 128-column slices of a state row per lane (1: N <= 128, 2: N <= 256)
template <typename T, int KS>
__global__ void __launch_bounds__(kDecThreads)
ssd_decode_kernel(const T *__restrict__ x, const T *__restrict__ dt, const float *__restrict__ A_log,
                  const T *__restrict__ Bm, const T *__restrict__ Cm, const float *__restrict__ D,
                  float *__restrict__ state, T *__restrict__ y, int H, int P, int N, int G, int hpg,
                  int dt_softplus)
{
    const int bh = blockIdx.x;              // row * H + head
    const int row = bh / H, h = bh - row * H, g = h / hpg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // exact softplus and exponentials: the kernel waits on memory, not on arithmetic
    const float r = to_f32(dt[bh]);
    const float delta = dt_softplus ? fmaxf(r, 0.0f) + log1pf(expf(-fabsf(r))) : r;
    const float a = expf(delta * -expf(A_log[h]));
    const float Dh = D ? D[h] : 0.0f;

    float bv[KS][4], cv[KS][4];
    const size_t gofs = ((size_t)row * G + g) * N;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
        const int n0 = 128 * k + 4 * lane;
        if (n0 < N) {
            load4(Bm + gofs + n0, bv[k]);
            load4(Cm + gofs + n0, cv[k]);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) bv[k][i] = cv[k][i] = 0.0f;
        }
    }

    float *const st = state + (size_t)bh * P * N;
    for (int p0 = warp * kDecRows; p0 < P; p0 += kDecWarps * kDecRows) {
        float s[kDecRows][KS][4];
        float xp[kDecRows];
#pragma unroll
        for (int j = 0; j < kDecRows; ++j) {
            const int p = p0 + j;
            xp[j] = p < P ? to_f32(x[(size_t)bh * P + p]) : 0.0f;
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                const int n0 = 128 * k + 4 * lane;
                if (p < P && n0 < N) {
                    const float4 q = *reinterpret_cast<const float4 *>(st + (size_t)p * N + n0);
                    s[j][k][0] = q.x; s[j][k][1] = q.y; s[j][k][2] = q.z; s[j][k][3] = q.w;
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) s[j][k][i] = 0.0f;
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kDecRows; ++j) {
            const int p = p0 + j;
            const float dx = delta * xp[j];
            float acc = 0.0f;
#pragma unroll
            for (int k = 0; k < KS; ++k) {
                const int n0 = 128 * k + 4 * lane;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    s[j][k][i] = fmaf(a, s[j][k][i], dx * bv[k][i]);
                    acc = fmaf(s[j][k][i], cv[k][i], acc);
                }
                if (p < P && n0 < N)
                    *reinterpret_cast<float4 *>(st + (size_t)p * N + n0) =
                        make_float4(s[j][k][0], s[j][k][1], s[j][k][2], s[j][k][3]);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0 && p < P) y[(size_t)bh * P + p] = from_f32<T>(acc + Dh * xp[j]);
        }
    }
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T>
void launch_decode(bool two_slices, unsigned blocks, cudaStream_t st, const T *x, const T *dt, const float *A_log,
                   const T *B, const T *C, const float *D, float *state, T *y, const ssd_step_params &q, int hpg)
{
    if (two_slices)
        ssd_decode_kernel<T, 2><<<blocks, kDecThreads, 0, st>>>(x, dt, A_log, B, C, D, state, y, q.nheads, q.headdim,
                                                               q.dstate, q.ngroups, hpg, q.dt_softplus);
    else
        ssd_decode_kernel<T, 1><<<blocks, kDecThreads, 0, st>>>(x, dt, A_log, B, C, D, state, y, q.nheads, q.headdim,
                                                               q.dstate, q.ngroups, hpg, q.dt_softplus);
}

}  // namespace
}  // namespace ssd

extern "C" SSD_API ssd_status ssd_decode_step(const ssd_step_params *p, const void *x, const void *dt,
                                              const float *A_log, const void *B, const void *C, const float *D,
                                              float *state, void *y, void *stream)
{
    using namespace ssd;
    if (!p) return SSD_ERR_INVALID_ARG;
    const ssd_step_params q = *p;
    if (q.batch < 0 || q.nheads < 1 || q.headdim < 1 || q.dstate < 1 || q.ngroups < 1 ||
        q.nheads % q.ngroups != 0 || (q.io_dtype != SSD_DTYPE_F32 && q.io_dtype != SSD_DTYPE_BF16) ||
        (q.dt_softplus != 0 && q.dt_softplus != 1))
        return SSD_ERR_INVALID_ARG;
    if (q.dstate % 4 != 0 || q.dstate > 256 || q.headdim > 4096) return SSD_ERR_UNSUPPORTED;
    if (q.batch == 0) return SSD_OK;
    if (!x || !dt || !A_log || !B || !C || !state || !y) return SSD_ERR_INVALID_ARG;
    // vector accesses: B and C rows (4 elements), state rows (float4); x, dt, y are scalar
    if (!aligned16(B) || !aligned16(C) || !aligned16(state)) return SSD_ERR_INVALID_ARG;
    const long long blocks = (long long)q.batch * q.nheads;
    if (blocks > 0x7fffffffLL) return SSD_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int hpg = q.nheads / q.ngroups;
    const bool two = q.dstate > 128;
    if (q.io_dtype == SSD_DTYPE_BF16)
        launch_decode<__nv_bfloat16>(two, (unsigned)blocks, st, static_cast<const __nv_bfloat16 *>(x),
                                     static_cast<const __nv_bfloat16 *>(dt), A_log,
                                     static_cast<const __nv_bfloat16 *>(B), static_cast<const __nv_bfloat16 *>(C), D,
                                     state, static_cast<__nv_bfloat16 *>(y), q, hpg);
    else
        launch_decode<float>(two, (unsigned)blocks, st, static_cast<const float *>(x), static_cast<const float *>(dt),
                             A_log, static_cast<const float *>(B), static_cast<const float *>(C), D, state,
                             static_cast<float *>(y), q, hpg);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
