// Shared definitions of the SSD forward CUDA library (host + device).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "ssd_fwd.h"

namespace ssd {

// Device-side status codes written into the workspace's status word.  The
// first error wins (atomicCAS from 0).
enum DeviceStatus : int {
    kDevOk = 0,
    kDevTimeout = 1,
    kDevBadSeqlens = 2,
};

// Chunk / sequence tables, built on the device from cu_seqlens (or from the
// uniform batch) so that no host synchronisation is needed.
struct ChunkDesc {
    int seq;      // sequence index
    int tok0;     // first token in the flattened token axis
    int len;      // tokens in this chunk (1..Q)
    int idx;      // chunk index inside its sequence
};

struct SeqDesc {
    int chunk0;   // first chunk of the sequence in the chunk table
    int nchunks;  // ceil(len / Q)
    int tok0;
    int len;
};

// The forward's workspace starts with this many bytes: the status word, and
// from kSyncOffsetInts on, counters that CTAs of one launch use to wait for one
// another (zeroed with the status word before such a launch).
constexpr size_t kStatusRegion = 2048;
constexpr int kSyncOffsetInts = 64;

struct Plan {
    int *status;        // device status word
    int *count;         // number of valid chunk entries
    ChunkDesc *chunks;  // max_chunks entries
    SeqDesc *seqs;      // nseq entries
    int nseq;
    int max_chunks;
};

// Shapes as seen by the kernels.
struct Dims {
    int H, P, N, G, Q;
    int heads_per_group;  // H / G
    int tokens;           // batch * seqlen
    int dt_softplus;
};

__device__ __forceinline__ void set_status(int *status, int code)
{
    atomicCAS(status, 0, code);
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v)
{
    return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// softplus(r) = log(1 + e^r), evaluated without overflow and without a
// threshold shortcut.
__device__ __forceinline__ float softplus_f32(float r)
{
    return fmaxf(r, 0.0f) + log1pf(__expf(-fabsf(r)));
}

// Events and the failure-injection switch of ssd_fwd_instrumented (all null /
// zero for plain ssd_fwd).
struct Instr {
    cudaEvent_t begin = nullptr, main = nullptr, end = nullptr;
    int withhold_first_tile = 0;
};

// Host-side launchers (one per translation unit).
cudaError_t launch_build_plan(const Plan &plan, const int32_t *cu_seqlens, int batch, int seqlen,
                              int chunk_len, cudaStream_t stream);

struct SimtArgs {
    const void *x, *dt, *B, *C;
    const float *A_log, *D, *init;
    void *y;
    float *final_states;
    float *cs, *dv, *states;   // workspace
    int bf16;
};
cudaError_t launch_simt(const Plan &plan, const Dims &d, const SimtArgs &a, cudaStream_t stream,
                        const Instr &ins);
// Gated GroupNorm of the block output, in place on y (ssd_gnorm.cu).
cudaError_t launch_gated_norm(long long rows, int H, int P, bool bf16, void *y, const void *z, const float *w,
                              const float *b, float eps, cudaStream_t st);

// Ordered fold of per-worker state summaries (ssd_cp.cu).
cudaError_t launch_state_combine(int world, int rank, long long nsh, int PN, const float *S_all, const float *L_all,
                                 const float *init, float *H_in, cudaStream_t st);

// Backward pass (ssd_bwd.cu): 32-token chunks, fp32 gradients.
bool bwd_supported(const ssd_fwd_params &p);
size_t bwd_chunk_count(const ssd_fwd_params &p);
int bwd_chunk_len();
cudaError_t launch_bwd(const Plan &plan, const Dims &d, const SimtArgs &fa, const void *dy, const float *dfinal,
                       float *gbuf, float *dx, float *ddt, float *dA_log, float *dB, float *dC, float *dD,
                       float *dinit, bool bf16, cudaStream_t st);

// The first three SIMT kernels only (chunk cumsum, chunk states, state
// passing): cs, dv and, in `states`, the state entering every chunk.
cudaError_t launch_simt_states(const Plan &plan, const Dims &d, const SimtArgs &a, cudaStream_t stream,
                               float *final_states = nullptr);
// Every sequence's end state from a zero state and its total log decay
// sum_t delta_t A (SIMT kernels).
cudaError_t launch_simt_summary(const Plan &plan, const Dims &d, const SimtArgs &a, float *end_states,
                                float *logdecay, cudaStream_t stream);

}  // namespace ssd
