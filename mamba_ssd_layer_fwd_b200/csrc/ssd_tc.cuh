// Tensor-core (tcgen05 / TMEM / TMA) path of the SSD forward for sm_100a.
#pragma once

#include "ssd_common.cuh"

namespace ssd {

struct TcArgs {
    const void *x, *dt, *B, *C;
    const float *A_log, *D, *init;
    const int32_t *cu_seqlens;
    void *y;
    float *final_states;
    void *scratch;
    size_t scratch_bytes;
    // gated norm of the block output (z == nullptr: plain y)
    const void *z = nullptr;
    const float *gn_w = nullptr, *gn_b = nullptr;
    float gn_eps = 0.0f;
};

bool tc_supported(const ssd_fwd_params &p);
size_t tc_workspace_bytes(const ssd_fwd_params &p);
int tc_launch_count(const ssd_fwd_params &p);
cudaError_t launch_tc(const ssd_fwd_params &p, const Plan &plan, const Dims &d, const TcArgs &a,
                      cudaStream_t stream, const Instr &ins);
cudaError_t launch_tc_summary(const ssd_fwd_params &p, const Plan &plan, const TcArgs &a, float *end_states,
                              float *logdecay, cudaStream_t stream);
size_t tc_summary_workspace_bytes(const ssd_fwd_params &p);

}  // namespace ssd
