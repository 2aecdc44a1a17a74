// State passing between pieces of a sequence held by different workers
// ("Transformers are SSMs", Sec. 8.2, context parallelism: a worker receives
// an initial state, runs the SSM on its piece and hands its final state to the
// next worker; Fig. 7 right).  Worker r's piece maps its entering state H to
// exp(L_r) H + S_r, with S_r the piece's end state from a zero state and L_r
// its total log decay (one (nseq, nheads) scalar each), so the state entering
// worker `rank` is the ordered fold of the summaries of workers 0..rank-1
// starting from the initial state.
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kCombineThreads = 256;

__global__ void __launch_bounds__(kCombineThreads)
state_combine_kernel(int world, int rank, long long nsh, int PN, const float *__restrict__ S_all,
                     const float *__restrict__ L_all, const float *__restrict__ init, float *__restrict__ H_in)
{
    const long long i = (long long)blockIdx.x * kCombineThreads + threadIdx.x;
    if (i >= nsh * PN) return;
    const long long sh = i / PN;
    float v = init ? init[i] : 0.0f;
    for (int r = 0; r < rank && r < world; ++r)
        v = fmaf(__expf(L_all[(size_t)r * nsh + sh]), v, S_all[(size_t)r * nsh * PN + i]);
    H_in[i] = v;
}

}  // namespace

cudaError_t launch_state_combine(int world, int rank, long long nsh, int PN, const float *S_all, const float *L_all,
                                 const float *init, float *H_in, cudaStream_t st)
{
    const long long n = nsh * PN;
    if (n == 0) return cudaSuccess;
    state_combine_kernel<<<(unsigned)((n + kCombineThreads - 1) / kCombineThreads), kCombineThreads, 0, st>>>(
        world, rank, nsh, PN, S_all, L_all, init, H_in);
    return cudaGetLastError();
}

}  // namespace ssd
