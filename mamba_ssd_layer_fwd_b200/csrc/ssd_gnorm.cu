// Output normalisation of the Mamba-2 block ("Transformers are SSMs",
// Sec. 7.1: an extra normalisation before the block's output projection;
// Sec. 8.1: a GroupNorm whose group count divides by the tensor-parallel
// degree): out = GroupNorm(y * silu(z)) with one group per head (its headdim
// channels) and per-channel weight and bias.  This kernel runs it as a pass of
// its own after the SIMT forward; the tensor-core walk fuses it into its
// output epilogue instead.
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kGnWarps = 8;

// one warp per (token, head) row of P <= 128 channels, in place on y
template <typename T>
__global__ void __launch_bounds__(kGnWarps * 32)
gated_norm_kernel(long long rows, int H, int P, T *__restrict__ y, const T *__restrict__ z,
                  const float *__restrict__ w, const float *__restrict__ b, float eps)
{
    const long long row = (long long)blockIdx.x * kGnWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31;
    const int h = (int)(row % H);
    T *yr = y + row * P;
    const T *zr = z + row * P;
    float g[4];
    float s = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        float v = 0.0f;
        if (c < P) {
            const float zv = to_f32(zr[c]);
            v = to_f32(yr[c]) * (zv / (1.0f + expf(-zv)));
        }
        g[k] = v;
        s += v;
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float mean = s / P;
    float q = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if (lane + 32 * k < P) q = fmaf(g[k] - mean, g[k] - mean, q);
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    const float rstd = rsqrtf(q / P + eps);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int c = lane + 32 * k;
        if (c < P) {
            float o = (g[k] - mean) * rstd * w[(size_t)h * P + c];
            if (b) o += b[(size_t)h * P + c];
            yr[c] = from_f32<T>(o);
        }
    }
}

}  // namespace

cudaError_t launch_gated_norm(long long rows, int H, int P, bool bf16, void *y, const void *z, const float *w,
                              const float *b, float eps, cudaStream_t st)
{
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kGnWarps - 1) / kGnWarps);
    if (bf16)
        gated_norm_kernel<__nv_bfloat16><<<grid, kGnWarps * 32, 0, st>>>(
            rows, H, P, static_cast<__nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(z), w, b, eps);
    else
        gated_norm_kernel<float><<<grid, kGnWarps * 32, 0, st>>>(rows, H, P, static_cast<float *>(y),
                                                                 static_cast<const float *>(z), w, b, eps);
    return cudaGetLastError();
}

}  // namespace ssd
