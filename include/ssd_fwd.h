/*
 * ssd_fwd.h - C ABI of the Mamba-2 SSD (structured state space duality)
 * forward layer for NVIDIA B200 (sm_100a).
 *
 * The operation ("Transformers are SSMs: Generalized Models and Efficient
 * Algorithms Through Structured State Space Duality", Sec. 2.4 "SSD layer",
 * Sec. 3.4.1 eq. (8), Sec. 6 "SSD algorithm", Sec. 7.2 grouped heads,
 * Sec. 8.3 variable length), per sequence s and head h, with B/C group
 * g = h / (nheads / ngroups):
 *
 *     delta_t = softplus(dt[t, h])        (dt itself when dt_softplus == 0)
 *     a_t     = exp(delta_t * A_h),  A_h = -exp(A_log[h])
 *     state_t = a_t * state_{t-1} + (delta_t * x[t, h, :]) (outer) B[t, g, :]   (P x N, fp32)
 *     y[t, h, :] = state_t @ C[t, g, :] + D[h] * x[t, h, :]
 *
 * with state_{-1} = initial_states[s, h] (zeros when NULL) and
 * final_states[s, h] = the state after the sequence's last token.  It is
 * evaluated by the chunked block decomposition of the semiseparable matrix
 * M = L o (C B^T) (Sec. 6): quadratic form inside chunks, chunk states,
 * a scan over chunk states, state-to-output.  The result does not depend on
 * chunk_len except through rounding.
 *
 * Layouts (row-major, contiguous, every pointer 16-byte aligned):
 *     x, y             (batch, seqlen, nheads, headdim)     io dtype
 *     dt               (batch, seqlen, nheads)              io dtype
 *     B, C             (batch, seqlen, ngroups, dstate)     io dtype
 *     A_log, D         (nheads)                             float32
 *     initial_states,
 *     final_states     (nseq, nheads, headdim, dstate)      float32
 *     cu_seqlens       (num_seqs + 1)                       int32
 * nseq = num_seqs when cu_seqlens is given (packed variable-length batch:
 * batch == 1, seqlen == total tokens, sequence i = tokens
 * [cu_seqlens[i], cu_seqlens[i+1]) with no state crossing a boundary),
 * else nseq = batch.
 *
 * Ownership and threading: every data pointer is a DEVICE pointer owned by
 * the caller; the library allocates and frees nothing and keeps no mutable
 * global state.  Calls are asynchronous on `stream` (a cudaStream_t passed as
 * void*, NULL = legacy default stream); calls on different streams with
 * different workspaces may run concurrently.
 *
 * Errors: arguments are validated on the host before anything is launched,
 * and no C++ exception crosses this boundary.  Problems the host cannot see
 * (a malformed cu_seqlens, a device-side wait that ran out of its bound) are
 * recorded in the workspace's status word; read it with ssd_get_status().
 */
#ifndef SSD_FWD_H_
#define SSD_FWD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SSD_ABI_VERSION 2

#if defined(__GNUC__)
#define SSD_API __attribute__((visibility("default")))
#else
#define SSD_API
#endif

typedef enum ssd_status {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = -1,   /* null/misaligned pointer, bad dimension, workspace too small */
    SSD_ERR_UNSUPPORTED = -2,   /* valid shape the library does not implement (see limits) */
    SSD_ERR_CUDA = -3,          /* a CUDA runtime call or launch failed */
    SSD_ERR_TIMEOUT = -4,       /* device-side bounded wait gave up (status word) */
    SSD_ERR_BAD_SEQLENS = -5    /* cu_seqlens not 0 = c0 <= c1 <= ... = seqlen (status word) */
} ssd_status;

typedef enum ssd_dtype {
    SSD_DTYPE_F32 = 0,          /* x, dt, B, C, y in float32 */
    SSD_DTYPE_BF16 = 1          /* x, dt, B, C, y in bfloat16 (states stay float32) */
} ssd_dtype;

/* Limits ("see limits" above).  SIMT path: headdim 1..128, dstate 1..256,
 * float32 or bf16.  Tensor-core path: bf16, headdim 64, dstate 64, 128 or
 * 256, dt_softplus == 1, chunk_len 128 or 256, at least 128 tokens in the
 * call; it evaluates the decomposition on 128-token blocks whatever
 * chunk_len is (the result does not depend on chunk_len beyond rounding).
 * AUTO takes the tensor-core path whenever these hold.  Requesting a path the
 * shape does not allow returns SSD_ERR_UNSUPPORTED, and so do problems with
 * 2^31 or more elements in x or in B, or more than 2^20 packed sequences. */
typedef enum ssd_path {
    SSD_PATH_AUTO = 0,          /* tensor-core path when the shape allows it, else SIMT */
    SSD_PATH_SIMT = 1,          /* CUDA-core path: any supported shape, float32 or bf16 */
    SSD_PATH_TENSOR = 2         /* tcgen05/TMEM path: bf16, headdim 64, dstate 64/128/256 */
} ssd_path;

typedef struct ssd_fwd_params {
    int batch;                  /* >= 1 (1 when num_seqs > 0) */
    int seqlen;                 /* >= 0, tokens per row (total tokens when num_seqs > 0) */
    int nheads;                 /* H >= 1 */
    int headdim;                /* P: 1..128 (tensor path: 64) */
    int dstate;                 /* N: 1..256 (tensor path: 64, 128 or 256) */
    int ngroups;                /* G >= 1, nheads % ngroups == 0 */
    int chunk_len;              /* Q: 64, 128 or 256 */
    int num_seqs;               /* > 0 iff cu_seqlens != NULL */
    ssd_dtype io_dtype;
    int dt_softplus;            /* 1: delta = softplus(dt); 0: delta = dt (must be >= 0) */
    ssd_path path;
} ssd_fwd_params;

/* Bytes of device workspace ssd_fwd needs for these parameters (0 on invalid
 * parameters), for the device current at the time of the query: the schedule
 * of equal-length rows depends on that device's SM count (at most 148 are
 * used), so ask with the device current that the call will run on.  ssd_fwd
 * recomputes the size and returns SSD_ERR_INVALID_ARG for a smaller workspace.
 * The workspace must be 256-byte aligned; its contents need no initialisation
 * and may be reused by the next call on the same stream. */
SSD_API size_t ssd_fwd_workspace_size(const ssd_fwd_params *p);

/* SSD forward.  D, initial_states, cu_seqlens and final_states may be NULL
 * (D = 0, zero initial state, batch of equal rows, no final state written).
 * Returns SSD_OK once every kernel is enqueued; see ssd_get_status for the
 * device-side outcome. */
SSD_API ssd_status ssd_fwd(const ssd_fwd_params *p,
                   const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D,
                   const float *initial_states, const int32_t *cu_seqlens,
                   void *y, float *final_states,
                   void *workspace, size_t workspace_bytes, void *stream);

/* Measurement and failure-injection hooks for ssd_fwd_instrumented (profiling
 * tools and the library's own tests; ordinary callers use ssd_fwd). */
typedef struct ssd_fwd_instrumentation {
    void *ev_begin;             /* cudaEvent_t or NULL: recorded on `stream` before the first compute
                                   kernel (after the work planner / status reset) */
    void *ev_main;              /* cudaEvent_t or NULL: recorded before the kernel that writes y (equals
                                   ev_begin unless a state-only pass and segment scan run first) */
    void *ev_end;               /* cudaEvent_t or NULL: recorded after the last kernel */
    int withhold_first_tile;    /* 0 normally; nonzero makes the tensor-core path withhold the first x tile
                                   of work item 0, so that item's bounded waits run out and the call reports
                                   SSD_ERR_TIMEOUT through ssd_get_status (no fault, the context survives) */
} ssd_fwd_instrumentation;

/* ssd_fwd with instrumentation; `ins` may be NULL (then identical to ssd_fwd). */
SSD_API ssd_status ssd_fwd_instrumented(const ssd_fwd_params *p,
                   const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D,
                   const float *initial_states, const int32_t *cu_seqlens,
                   void *y, float *final_states,
                   void *workspace, size_t workspace_bytes, void *stream,
                   const ssd_fwd_instrumentation *ins);

/* Size of the fixed scratch array behind ssd_fwd_noalloc: 16 MiB of device
 * memory on every GPU that loads this library, held until the process exits. */
#define SSD_NOALLOC_SCRATCH_BYTES (16u << 20)

/* Allocation-free SSD forward, for callers that cannot allocate device memory
 * (inside an allocator's own callbacks, in a real-time loop that must not take
 * allocator locks or risk running out of memory mid-run, in a runtime that
 * only lends out the tensors it owns).  No counterpart in the paper: it is the
 * same operation as ssd_fwd, with the workspace taken from a file-scope
 * __device__ array of SSD_NOALLOC_SCRATCH_BYTES instead of the caller.
 *   - Arguments are those of ssd_fwd minus the workspace; inputs and outputs
 *     are still the caller's device buffers.
 *   - Returns SSD_ERR_UNSUPPORTED (nothing launched) when the problem needs
 *     more workspace than SSD_NOALLOC_SCRATCH_BYTES (ssd_fwd_workspace_size).
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's address with that
 *     device current; make it before any stream capture.  The address is kept
 *     for the life of the process: after cudaDeviceReset (or any other
 *     teardown of the device's primary context) it is stale, and this entry
 *     point must not be called again on that device.
 *   - Every call shares the array.  The kernels clear what must start at zero
 *     and overwrite the rest before reading it, but calls that overlap on the
 *     GPU (other streams, other threads on the same device) race on it.
 *   - sync_status != 0: synchronise `stream` and return the device-side status
 *     (what ssd_get_status reports for ssd_fwd). */
SSD_API ssd_status ssd_fwd_noalloc(const ssd_fwd_params *p,
                   const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D,
                   const float *initial_states, const int32_t *cu_seqlens,
                   void *y, float *final_states, void *stream, int sync_status);

/* One decoding step: the recurrent (linear) mode of the same layer
 * ("Transformers are SSMs", Sec. 3.4.1 eq. (8)) applied to a single new token
 * of every row, with the state carried in place between calls:
 *
 *     delta = softplus(dt[b, h])  (dt itself when dt_softplus == 0)
 *     a     = exp(delta * -exp(A_log[h]))
 *     state[b, h] <- a * state[b, h] + (delta * x[b, h, :]) (outer) B[b, g, :]
 *     y[b, h, :]   = state[b, h] @ C[b, g, :] + D[h] * x[b, h, :]
 *
 * A prefill with ssd_fwd(..., final_states) followed by steps from that state
 * reproduces ssd_fwd over the concatenated tokens.
 * Layouts (row-major, contiguous): x, y (batch, nheads, headdim) and
 * dt (batch, nheads) in io dtype; B, C (batch, ngroups, dstate) io dtype;
 * A_log, D (nheads) float32; state (batch, nheads, headdim, dstate) float32,
 * read and overwritten.  B, C and state must be 16-byte aligned; x, dt, y
 * naturally aligned.  D may be NULL (0).  All pointers are caller-owned device
 * pointers; no workspace, nothing allocated, asynchronous on `stream`.
 * Returns SSD_ERR_INVALID_ARG (bad dimension or pointer), SSD_ERR_UNSUPPORTED
 * (dstate not a multiple of 4 or above 256), SSD_ERR_CUDA (launch failed). */
typedef struct ssd_step_params {
    int batch;                  /* rows >= 0 (0: nothing to do) */
    int nheads;                 /* H >= 1 */
    int headdim;                /* P >= 1 */
    int dstate;                 /* N: multiple of 4, <= 256 */
    int ngroups;                /* G >= 1, nheads % ngroups == 0 */
    ssd_dtype io_dtype;
    int dt_softplus;            /* 1: delta = softplus(dt); 0: delta = dt */
} ssd_step_params;

SSD_API ssd_status ssd_decode_step(const ssd_step_params *p,
                   const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D,
                   float *state, void *y, void *stream);

/* The SSD forward followed by the Mamba-2 block's output normalisation
 * ("Transformers are SSMs", Sec. 7.1: an extra normalisation layer before the
 * block's output projection; Sec. 8.1: a GroupNorm whose group count divides
 * by the tensor-parallel degree), with the gate of the block's z branch:
 *
 *     g   = y * silu(z),   silu(z) = z / (1 + exp(-z))
 *     out = (g - mean) / sqrt(var + eps) * norm_weight + norm_bias
 *
 * mean and var over each group of headdim channels of one token and head (one
 * group per head).  z has y's layout and io dtype; norm_weight and norm_bias
 * (NULL = 0) are float32 (nheads * headdim); out receives the normalised
 * output in y's layout (y itself is not written).  The tensor-core path fuses
 * the gate and the norm into its output epilogue; the SIMT path runs them as
 * one more pass over out.  Other arguments, limits, errors and the workspace
 * are ssd_fwd's; eps must be >= 0. */
SSD_API ssd_status ssd_fwd_gated_norm(const ssd_fwd_params *p,
                   const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D,
                   const float *initial_states, const int32_t *cu_seqlens,
                   const void *z, const float *norm_weight, const float *norm_bias, float eps,
                   void *out, float *final_states, void *workspace, size_t workspace_bytes, void *stream);

/* Context parallelism ("Transformers are SSMs", Sec. 8.2 item 2, Fig. 7
 * right): a long sequence is cut into pieces held by different workers; a
 * worker takes the state entering its piece, runs the SSM on it and passes
 * its final state on.  Since a piece maps an entering state H to
 * exp(L) H + S, with S its end state from a zero state and L its total log
 * decay (sum over its tokens of delta_t * A), the workers can summarise their
 * pieces at the same time, exchange the summaries once, and each fold the
 * summaries of the pieces before its own:
 *
 *   1. ssd_fwd_summary on the local piece          -> S (nseq, nheads, headdim, dstate), L (nseq, nheads)
 *   2. all-gather S and L over the workers         (the caller's collective, e.g. NCCL)
 *   3. ssd_state_combine(world, rank, ...)         -> the state entering this piece
 *   4. ssd_fwd on the local piece from that state  -> y of the piece (and, on the last worker, the
 *                                                     final state)
 *
 * ssd_fwd_summary takes ssd_fwd's parameters and inputs (C and D are not
 * needed) and writes, for every sequence of the call, its end state from a
 * zero state (end_states, float32) and its total log decay (logdecay,
 * float32, (nseq, nheads)).  Its workspace is ssd_fwd's
 * (ssd_fwd_summary_workspace_size).  Errors and asynchrony as for ssd_fwd.
 *
 * ssd_state_combine folds the summaries of workers 0 .. rank-1, in order,
 * starting from initial_states (NULL = 0): H <- exp(L_r) H + S_r.
 * end_states_all is (world, nseq, nheads, headdim, dstate) and logdecay_all
 * (world, nseq, nheads), float32 device arrays; entering_states receives
 * (nseq, nheads, headdim, dstate).  rank == world gives the state after the
 * whole sequence.  Returns SSD_ERR_INVALID_ARG for a bad size or NULL array,
 * SSD_ERR_CUDA if the launch fails. */
SSD_API size_t ssd_fwd_summary_workspace_size(const ssd_fwd_params *p);

SSD_API ssd_status ssd_fwd_summary(const ssd_fwd_params *p,
                   const void *x, const void *dt, const float *A_log, const void *B,
                   const int32_t *cu_seqlens, float *end_states, float *logdecay,
                   void *workspace, size_t workspace_bytes, void *stream);

SSD_API ssd_status ssd_state_combine(int world, int rank, int nseq, int nheads, int headdim, int dstate,
                   const float *end_states_all, const float *logdecay_all,
                   const float *initial_states, float *entering_states, void *stream);

/* Backward pass: the gradients of a loss L given dy = dL/dy and
 * dfinal_states = dL/dfinal_states, for training ("Transformers are SSMs",
 * Thm. 6.1 counts the training cost of the SSD algorithm; the gradient is the
 * same block decomposition of Sec. 6 run in reverse).  With the forward's
 * per-token update (see the top of this file) and G_t = dL/dstate_t:
 *
 *     G_t = dy_t (outer) C_t + a_{t+1} G_{t+1},   G_last = dL/dfinal_states
 *     dx_t = D dy_t + delta_t G_t B_t,   dB_t = sum over the group's heads of delta_t G_t^T x_t,
 *     dC_t = sum over the group's heads of state_t^T dy_t,
 *     ddelta_t = x_t^T G_t B_t + A a_t <G_t, state_{t-1}>,   ddt_t = ddelta_t sigmoid(dt_t)
 *     (ddelta_t itself when dt_softplus == 0),   dA_log = A sum_t delta_t a_t <G_t, state_{t-1}>,
 *     dD = sum_t <dy_t, x_t>,   dinitial_states = a_first G_first
 *
 * Inputs are those of ssd_fwd plus dy (y's layout and io dtype) and
 * dfinal_states ((nseq, nheads, headdim, dstate) float32, NULL = 0).
 * Every gradient is float32, in the layout of its input: dx (batch, seqlen,
 * nheads, headdim), ddt (batch, seqlen, nheads) with respect to the raw dt,
 * dA_log and dD (nheads), dB and dC (batch, seqlen, ngroups, dstate),
 * dinitial_states (nseq, nheads, headdim, dstate; NULL: not written).  D and
 * initial_states may be NULL as in ssd_fwd; dD is written either way.  The
 * pass recomputes the forward's chunk states on CUDA cores with 32-token
 * chunks (chunk_len is not used; the result does not depend on it) and holds
 * two fp32 states per chunk and head in the workspace.  Supported: float32
 * or bf16 inputs, headdim <= 128, dstate <= 256, path AUTO or SIMT
 * (SSD_PATH_TENSOR returns SSD_ERR_UNSUPPORTED).  Errors and asynchrony as
 * for ssd_fwd; ssd_get_status reads the workspace's status word. */
SSD_API size_t ssd_bwd_workspace_size(const ssd_fwd_params *p);

SSD_API ssd_status ssd_bwd(const ssd_fwd_params *p,
                   const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D,
                   const float *initial_states, const int32_t *cu_seqlens,
                   const void *dy, const float *dfinal_states,
                   float *dx, float *ddt, float *dA_log, float *dB, float *dC, float *dD,
                   float *dinitial_states, void *workspace, size_t workspace_bytes, void *stream);

/* Device-side status of the last ssd_fwd that used `workspace` on `stream`:
 * synchronises `stream`, then returns SSD_OK, SSD_ERR_TIMEOUT or
 * SSD_ERR_BAD_SEQLENS (or SSD_ERR_CUDA if the copy fails). */
SSD_API ssd_status ssd_get_status(const void *workspace, void *stream);

/* Number of kernels one ssd_fwd call with these parameters launches. */
SSD_API int ssd_fwd_launch_count(const ssd_fwd_params *p);

/* The path ssd_fwd takes for these parameters (AUTO resolved), or -1. */
SSD_API int ssd_fwd_resolved_path(const ssd_fwd_params *p);

/* Static description of a status code. */
SSD_API const char *ssd_status_string(ssd_status s);

SSD_API int ssd_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_FWD_H_ */
