// ssd_fwd_noalloc: the SSD forward for callers that cannot allocate device
// memory.  Its workspace is a fixed file-scope __device__ array that lives in
// this library's module, so the call itself allocates nothing.
//
// Who needs this: code that runs where cudaMalloc is off limits, for example
// inside a custom allocator's own callbacks, a real-time loop that must not
// take the allocator's locks or risk an out-of-memory failure mid-run, or an
// embedding runtime that hands out only the tensors it owns.  Such callers
// pass inputs and outputs as usual; the scratch space comes from here.
//
// Rules of use (also stated in include/ssd_fwd.h):
//  - The array holds SSD_NOALLOC_SCRATCH_BYTES bytes on every GPU that loads
//    the library, for as long as the process lives.
//  - Problems whose workspace (ssd_fwd_workspace_size) exceeds that size are
//    rejected with SSD_ERR_UNSUPPORTED before anything is launched.
//  - The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    before any stream capture.
//  - All calls share the one array.  The kernels clear what must start at
//    zero (the status word) and overwrite everything else they read, so the
//    previous call's leftovers do no harm, but calls that overlap on the GPU
//    (different streams, or threads racing on one device) race on it.
#include <mutex>

#include "ssd_common.cuh"

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array for the current device (looked up once).
cudaError_t scratch_for_current_device(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ssd_status ssd_fwd_noalloc(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log,
                                      const void *B, const void *C, const float *D, const float *initial_states,
                                      const int32_t *cu_seqlens, void *y, float *final_states, void *stream,
                                      int sync_status)
{
    void *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return SSD_ERR_CUDA;
    // invalid parameters report 0 here and are then rejected by ssd_fwd's own checks
    if (ssd_fwd_workspace_size(p) > (size_t)SSD_NOALLOC_SCRATCH_BYTES) return SSD_ERR_UNSUPPORTED;
    const ssd_status s = ssd_fwd(p, x, dt, A_log, B, C, D, initial_states, cu_seqlens, y, final_states, scratch,
                                 (size_t)SSD_NOALLOC_SCRATCH_BYTES, stream);
    if (s != SSD_OK || !sync_status) return s;
    return ssd_get_status(scratch, stream);
}
