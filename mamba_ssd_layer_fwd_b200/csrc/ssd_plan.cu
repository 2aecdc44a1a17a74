// Chunk and sequence tables for the SSD forward ("Transformers are SSMs",
// Sec. 6: the sequence axis is split into chunks of length Q; Sec. 8.3: a
// packed batch is one long token axis in which no state crosses a sequence
// boundary, so chunks never straddle two sequences).
//
// One block builds both tables from cu_seqlens (or from the uniform batch)
// on the device, so the host never waits for the lengths.
#include "ssd_common.cuh"

namespace ssd {
namespace {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
build_plan_kernel(Plan plan, const int32_t *__restrict__ cu_seqlens, int batch, int seqlen, int Q)
{
    __shared__ int s_bad;
    __shared__ int s_carry;
    __shared__ int s_warp[kPlanThreads / 32];
    const int tid = threadIdx.x;
    const int nseq = plan.nseq;
    if (tid == 0) {
        *plan.status = 0;
        s_bad = 0;
        s_carry = 0;
    }
    __syncthreads();

    // Validate cu_seqlens: 0 = c0 <= c1 <= ... <= c_nseq = seqlen.
    if (cu_seqlens) {
        for (int i = tid; i < nseq; i += kPlanThreads) {
            const int a = cu_seqlens[i], b = cu_seqlens[i + 1];
            if (b < a || (i == 0 && a != 0) || (i == nseq - 1 && b != seqlen)) s_bad = 1;
        }
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) {
            set_status(plan.status, kDevBadSeqlens);
            *plan.count = 0;
        }
        for (int i = tid; i < nseq; i += kPlanThreads) plan.seqs[i] = SeqDesc{0, 0, 0, 0};
        return;
    }

    // Exclusive scan of chunks-per-sequence, one tile of kPlanThreads at a time.
    for (int base = 0; base < nseq; base += kPlanThreads) {
        const int i = base + tid;
        int tok0 = 0, len = 0, nch = 0;
        if (i < nseq) {
            if (cu_seqlens) {
                tok0 = cu_seqlens[i];
                len = cu_seqlens[i + 1] - tok0;
            } else {
                tok0 = i * seqlen;
                len = seqlen;
            }
            nch = (len + Q - 1) / Q;
        }
        // block-wide inclusive scan of nch
        int v = nch;
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, v, o);
            if ((tid & 31) >= o) v += u;
        }
        if ((tid & 31) == 31) s_warp[tid >> 5] = v;
        __syncthreads();
        if (tid < 32) {
            int w = s_warp[tid];
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, w, o);
                if (tid >= o) w += u;
            }
            s_warp[tid] = w;
        }
        __syncthreads();
        const int incl = v + ((tid >> 5) ? s_warp[(tid >> 5) - 1] : 0) + s_carry;
        const int chunk0 = incl - nch;
        if (i < nseq) {
            plan.seqs[i] = SeqDesc{chunk0, nch, tok0, len};
            for (int j = 0; j < nch; ++j) {
                const int c = chunk0 + j;
                if (c < plan.max_chunks)
                    plan.chunks[c] = ChunkDesc{i, tok0 + j * Q, min(Q, len - j * Q), j};
            }
        }
        __syncthreads();
        if (tid == kPlanThreads - 1) s_carry = incl;
        __syncthreads();
    }
    if (tid == 0) *plan.count = min(s_carry, plan.max_chunks);
}

}  // namespace

cudaError_t launch_build_plan(const Plan &plan, const int32_t *cu_seqlens, int batch, int seqlen,
                              int chunk_len, cudaStream_t stream)
{
    (void)batch;
    build_plan_kernel<<<1, kPlanThreads, 0, stream>>>(plan, cu_seqlens, batch, seqlen, chunk_len);
    return cudaGetLastError();
}

}  // namespace ssd
