// C ABI of the SSD forward library: argument validation, workspace carving,
// path selection and the launch sequence.  Declarations and the contract of
// every entry point are in include/ssd_fwd.h.
#include <new>

#include "ssd_common.cuh"
#include "ssd_tc.cuh"

namespace ssd {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int nseq_of(const ssd_fwd_params &p) { return p.num_seqs > 0 ? p.num_seqs : p.batch; }

// Upper bound on the number of chunks: each sequence adds at most one partial chunk.
int max_chunks_of(const ssd_fwd_params &p)
{
    const long long Q = p.chunk_len;
    long long m;
    if (p.num_seqs > 0)
        m = (p.seqlen + Q - 1) / Q + p.num_seqs;
    else
        m = (long long)p.batch * ((p.seqlen + Q - 1) / Q);
    return (int)m;
}

// Host-side validation; returns SSD_OK or the error to report.
ssd_status validate(const ssd_fwd_params *p)
{
    if (!p) return SSD_ERR_INVALID_ARG;
    if (p->batch < 1 || p->seqlen < 0 || p->nheads < 1 || p->headdim < 1 || p->dstate < 1 ||
        p->ngroups < 1 || p->nheads % p->ngroups != 0 || p->num_seqs < 0)
        return SSD_ERR_INVALID_ARG;
    if (p->chunk_len != 64 && p->chunk_len != 128 && p->chunk_len != 256) return SSD_ERR_INVALID_ARG;
    if (p->num_seqs > 0 && p->batch != 1) return SSD_ERR_INVALID_ARG;
    if (p->io_dtype != SSD_DTYPE_F32 && p->io_dtype != SSD_DTYPE_BF16) return SSD_ERR_INVALID_ARG;
    if (p->path != SSD_PATH_AUTO && p->path != SSD_PATH_SIMT && p->path != SSD_PATH_TENSOR)
        return SSD_ERR_INVALID_ARG;
    if (p->dt_softplus != 0 && p->dt_softplus != 1) return SSD_ERR_INVALID_ARG;
    // 32-bit token and element indices inside the kernels
    const long long tokens = (long long)p->batch * p->seqlen;
    if (tokens * p->nheads * p->headdim >= (1LL << 31) || tokens * p->ngroups * p->dstate >= (1LL << 31))
        return SSD_ERR_UNSUPPORTED;
    if (p->headdim > 128 || p->dstate > 256) return SSD_ERR_UNSUPPORTED;
    if (p->num_seqs > (1 << 20)) return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

int resolve_path(const ssd_fwd_params &p)
{
    const bool tc_ok = tc_supported(p);
    if (p.path == SSD_PATH_SIMT) return SSD_PATH_SIMT;
    if (p.path == SSD_PATH_TENSOR) return tc_ok ? SSD_PATH_TENSOR : -1;
    return tc_ok ? SSD_PATH_TENSOR : SSD_PATH_SIMT;
}

// Workspace layout (all regions 256-byte aligned).
struct Layout {
    size_t status, count, chunks, seqs;   // common
    size_t cs, dv, states;                // SIMT path
    size_t tc;                            // tensor-core path scratch
    size_t total;
};

Layout layout_of(const ssd_fwd_params &p, int path)
{
    Layout L{};
    size_t off = 0;
    L.status = off; off += kStatusRegion;
    L.count = off; off += kAlign;
    const size_t mc = (size_t)max_chunks_of(p);
    const size_t ns = (size_t)nseq_of(p);
    L.chunks = off; off = align_up(off + mc * sizeof(ChunkDesc));
    L.seqs = off; off = align_up(off + ns * sizeof(SeqDesc));
    if (path == SSD_PATH_SIMT) {
        const size_t cq = mc * p.nheads * p.chunk_len * sizeof(float);
        L.cs = off; off = align_up(off + cq);
        L.dv = off; off = align_up(off + cq);
        L.states = off; off = align_up(off + mc * p.nheads * (size_t)p.headdim * p.dstate * sizeof(float));
    } else {
        L.tc = off; off = align_up(off + tc_workspace_bytes(p));
    }
    L.total = off;
    return L;
}

}  // namespace
}  // namespace ssd

using namespace ssd;

extern "C" {

int ssd_abi_version(void) { return SSD_ABI_VERSION; }

const char *ssd_status_string(ssd_status s)
{
    switch (s) {
    case SSD_OK: return "ok";
    case SSD_ERR_INVALID_ARG: return "invalid argument";
    case SSD_ERR_UNSUPPORTED: return "unsupported shape or path";
    case SSD_ERR_CUDA: return "CUDA error";
    case SSD_ERR_TIMEOUT: return "device-side wait timed out";
    case SSD_ERR_BAD_SEQLENS: return "cu_seqlens is not a non-decreasing 0..seqlen sequence";
    }
    return "unknown status";
}

int ssd_fwd_resolved_path(const ssd_fwd_params *p)
{
    if (validate(p) != SSD_OK) return -1;
    return resolve_path(*p);
}

size_t ssd_fwd_workspace_size(const ssd_fwd_params *p)
{
    if (validate(p) != SSD_OK) return 0;
    const int path = resolve_path(*p);
    if (path < 0) return 0;
    return layout_of(*p, path).total;
}

int ssd_fwd_launch_count(const ssd_fwd_params *p)
{
    if (validate(p) != SSD_OK) return -1;
    const int path = resolve_path(*p);
    if (path < 0) return -1;
    if (path == SSD_PATH_SIMT) return max_chunks_of(*p) == 0 ? 2 : 5;   // chunk table + kernels
    return (long long)p->batch * p->seqlen == 0 ? 1 : tc_launch_count(*p);
}

ssd_status ssd_fwd(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log,
                   const void *B, const void *C, const float *D, const float *initial_states,
                   const int32_t *cu_seqlens, void *y, float *final_states, void *workspace,
                   size_t workspace_bytes, void *stream)
{
    return ssd_fwd_instrumented(p, x, dt, A_log, B, C, D, initial_states, cu_seqlens, y, final_states, workspace,
                                workspace_bytes, stream, nullptr);
}

}  // extern "C"

namespace {

struct GnArgs {
    const void *z;
    const float *w, *b;
    float eps;
};

ssd_status fwd_impl(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log, const void *B,
                    const void *C, const float *D, const float *initial_states, const int32_t *cu_seqlens, void *y,
                    float *final_states, void *workspace, size_t workspace_bytes, void *stream,
                    const ssd_fwd_instrumentation *instr, const GnArgs *gn)
{
    try {
        const ssd_status v = validate(p);
        if (v != SSD_OK) return v;
        const bool has_tokens = (long long)p->batch * p->seqlen > 0;
        if (!A_log || !workspace) return SSD_ERR_INVALID_ARG;
        if (has_tokens && (!x || !dt || !B || !C || !y)) return SSD_ERR_INVALID_ARG;
        if ((p->num_seqs > 0) != (cu_seqlens != nullptr)) return SSD_ERR_INVALID_ARG;
        const void *ptrs[] = {x, dt, A_log, B, C, y, D, initial_states, final_states, cu_seqlens};
        for (const void *q : ptrs)
            if (q && !aligned16(q)) return SSD_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return SSD_ERR_INVALID_ARG;
        const int path = resolve_path(*p);
        if (path < 0) return SSD_ERR_UNSUPPORTED;
        const Layout L = layout_of(*p, path);
        if (workspace_bytes < L.total) return SSD_ERR_INVALID_ARG;

        cudaStream_t st = static_cast<cudaStream_t>(stream);
        char *ws = static_cast<char *>(workspace);
        Plan plan;
        plan.status = reinterpret_cast<int *>(ws + L.status);
        plan.count = reinterpret_cast<int *>(ws + L.count);
        plan.chunks = reinterpret_cast<ChunkDesc *>(ws + L.chunks);
        plan.seqs = reinterpret_cast<SeqDesc *>(ws + L.seqs);
        plan.nseq = nseq_of(*p);
        plan.max_chunks = max_chunks_of(*p);

        Dims d;
        d.H = p->nheads;
        d.P = p->headdim;
        d.N = p->dstate;
        d.G = p->ngroups;
        d.Q = p->chunk_len;
        d.heads_per_group = p->nheads / p->ngroups;
        d.tokens = p->batch * p->seqlen;
        d.dt_softplus = p->dt_softplus;

        Instr ins;
        if (instr) {
            ins.begin = static_cast<cudaEvent_t>(instr->ev_begin);
            ins.main = static_cast<cudaEvent_t>(instr->ev_main);
            ins.end = static_cast<cudaEvent_t>(instr->ev_end);
            ins.withhold_first_tile = instr->withhold_first_tile;
        }
        cudaError_t e;
        if (path == SSD_PATH_SIMT) {
            // the chunk table kernel also clears the status word
            if (launch_build_plan(plan, cu_seqlens, p->batch, p->seqlen, p->chunk_len, st) != cudaSuccess)
                return SSD_ERR_CUDA;
            SimtArgs a;
            a.x = x; a.dt = dt; a.B = B; a.C = C;
            a.A_log = A_log; a.D = D; a.init = initial_states;
            a.y = y; a.final_states = final_states;
            a.cs = reinterpret_cast<float *>(ws + L.cs);
            a.dv = reinterpret_cast<float *>(ws + L.dv);
            a.states = reinterpret_cast<float *>(ws + L.states);
            a.bf16 = p->io_dtype == SSD_DTYPE_BF16;
            e = launch_simt(plan, d, a, st, ins);
            if (e == cudaSuccess && gn)
                e = launch_gated_norm((long long)d.tokens * d.H, d.H, d.P, a.bf16, y, gn->z, gn->w, gn->b, gn->eps,
                                      st);
        } else {
            TcArgs a;
            a.x = x; a.dt = dt; a.B = B; a.C = C;
            a.A_log = A_log; a.D = D; a.init = initial_states;
            a.cu_seqlens = cu_seqlens;
            a.y = y; a.final_states = final_states;
            a.scratch = ws + L.tc;
            a.scratch_bytes = L.total - L.tc;
            if (gn) {
                a.z = gn->z;
                a.gn_w = gn->w;
                a.gn_b = gn->b;
                a.gn_eps = gn->eps;
            }
            e = launch_tc(*p, plan, d, a, st, ins);
        }
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    } catch (const std::bad_alloc &) {
        return SSD_ERR_CUDA;
    } catch (...) {
        return SSD_ERR_CUDA;
    }
}

}  // namespace

extern "C" {

ssd_status ssd_fwd_instrumented(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log,
                                const void *B, const void *C, const float *D, const float *initial_states,
                                const int32_t *cu_seqlens, void *y, float *final_states, void *workspace,
                                size_t workspace_bytes, void *stream, const ssd_fwd_instrumentation *instr)
{
    return fwd_impl(p, x, dt, A_log, B, C, D, initial_states, cu_seqlens, y, final_states, workspace,
                    workspace_bytes, stream, instr, nullptr);
}

ssd_status ssd_fwd_gated_norm(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log,
                              const void *B, const void *C, const float *D, const float *initial_states,
                              const int32_t *cu_seqlens, const void *z, const float *norm_weight,
                              const float *norm_bias, float eps, void *out, float *final_states, void *workspace,
                              size_t workspace_bytes, void *stream)
{
    if (!p || !norm_weight || !(eps >= 0.0f)) return SSD_ERR_INVALID_ARG;
    if ((long long)p->batch * p->seqlen > 0 && !z) return SSD_ERR_INVALID_ARG;
    if ((z && !aligned16(z)) || !aligned16(norm_weight) || (norm_bias && !aligned16(norm_bias)))
        return SSD_ERR_INVALID_ARG;
    const GnArgs gn{z, norm_weight, norm_bias, eps};
    return fwd_impl(p, x, dt, A_log, B, C, D, initial_states, cu_seqlens, out, final_states, workspace,
                    workspace_bytes, stream, nullptr, &gn);
}

size_t ssd_fwd_summary_workspace_size(const ssd_fwd_params *p)
{
    return ssd_fwd_workspace_size(p);
}

ssd_status ssd_fwd_summary(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log, const void *B,
                           const int32_t *cu_seqlens, float *end_states, float *logdecay, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    try {
        const ssd_status v = validate(p);
        if (v != SSD_OK) return v;
        const bool has_tokens = (long long)p->batch * p->seqlen > 0;
        if (!A_log || !workspace || !end_states || !logdecay) return SSD_ERR_INVALID_ARG;
        if (has_tokens && (!x || !dt || !B)) return SSD_ERR_INVALID_ARG;
        if ((p->num_seqs > 0) != (cu_seqlens != nullptr)) return SSD_ERR_INVALID_ARG;
        const void *ptrs[] = {x, dt, A_log, B, cu_seqlens, end_states, logdecay};
        for (const void *q : ptrs)
            if (q && !aligned16(q)) return SSD_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return SSD_ERR_INVALID_ARG;
        const int path = resolve_path(*p);
        if (path < 0) return SSD_ERR_UNSUPPORTED;
        const Layout L = layout_of(*p, path);
        if (workspace_bytes < L.total) return SSD_ERR_INVALID_ARG;
        cudaStream_t st = static_cast<cudaStream_t>(stream);
        char *ws = static_cast<char *>(workspace);
        Plan plan;
        plan.status = reinterpret_cast<int *>(ws + L.status);
        plan.count = reinterpret_cast<int *>(ws + L.count);
        plan.chunks = reinterpret_cast<ChunkDesc *>(ws + L.chunks);
        plan.seqs = reinterpret_cast<SeqDesc *>(ws + L.seqs);
        plan.nseq = nseq_of(*p);
        plan.max_chunks = max_chunks_of(*p);
        cudaError_t e;
        if (path == SSD_PATH_SIMT) {
            Dims d;
            d.H = p->nheads;
            d.P = p->headdim;
            d.N = p->dstate;
            d.G = p->ngroups;
            d.Q = p->chunk_len;
            d.heads_per_group = p->nheads / p->ngroups;
            d.tokens = p->batch * p->seqlen;
            d.dt_softplus = p->dt_softplus;
            if (launch_build_plan(plan, cu_seqlens, p->batch, p->seqlen, p->chunk_len, st) != cudaSuccess)
                return SSD_ERR_CUDA;
            SimtArgs a;
            a.x = x; a.dt = dt; a.B = B; a.C = nullptr;
            a.A_log = A_log; a.D = nullptr; a.init = nullptr;
            a.y = nullptr; a.final_states = nullptr;
            a.cs = reinterpret_cast<float *>(ws + L.cs);
            a.dv = reinterpret_cast<float *>(ws + L.dv);
            a.states = reinterpret_cast<float *>(ws + L.states);
            a.bf16 = p->io_dtype == SSD_DTYPE_BF16;
            e = launch_simt_summary(plan, d, a, end_states, logdecay, st);
        } else {
            TcArgs a;
            a.x = x; a.dt = dt; a.B = B; a.C = nullptr;
            a.A_log = A_log; a.D = nullptr; a.init = nullptr;
            a.cu_seqlens = cu_seqlens;
            a.y = nullptr; a.final_states = nullptr;
            a.scratch = ws + L.tc;
            a.scratch_bytes = L.total - L.tc;
            e = launch_tc_summary(*p, plan, a, end_states, logdecay, st);
        }
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    } catch (...) {
        return SSD_ERR_CUDA;
    }
}

ssd_status ssd_state_combine(int world, int rank, int nseq, int nheads, int headdim, int dstate,
                             const float *end_states_all, const float *logdecay_all, const float *initial_states,
                             float *entering_states, void *stream)
{
    if (world < 1 || rank < 0 || rank > world || nseq < 0 || nheads < 1 || headdim < 1 || dstate < 1)
        return SSD_ERR_INVALID_ARG;
    if (!end_states_all || !logdecay_all || !entering_states) return SSD_ERR_INVALID_ARG;
    const long long nsh = (long long)nseq * nheads;
    if (nsh * headdim * dstate * (long long)world >= (1LL << 40)) return SSD_ERR_UNSUPPORTED;
    const cudaError_t e = launch_state_combine(world, rank, nsh, headdim * dstate, end_states_all, logdecay_all,
                                               initial_states, entering_states, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

namespace {

struct BwdLayout {
    size_t status, count, chunks, seqs, cs, dv, states, gbuf, total;
};

BwdLayout bwd_layout(const ssd_fwd_params &p)
{
    BwdLayout L{};
    size_t off = 0;
    const size_t mc = bwd_chunk_count(p), ns = (size_t)nseq_of(p), Q = (size_t)bwd_chunk_len();
    const size_t pn = (size_t)p.headdim * p.dstate;
    L.status = off; off += kAlign;
    L.count = off; off += kAlign;
    L.chunks = off; off = align_up(off + mc * sizeof(ChunkDesc));
    L.seqs = off; off = align_up(off + ns * sizeof(SeqDesc));
    L.cs = off; off = align_up(off + mc * p.nheads * Q * sizeof(float));
    L.dv = off; off = align_up(off + mc * p.nheads * Q * sizeof(float));
    L.states = off; off = align_up(off + mc * p.nheads * pn * sizeof(float));
    L.gbuf = off; off = align_up(off + mc * p.nheads * pn * sizeof(float));
    L.total = off;
    return L;
}

}  // namespace

size_t ssd_bwd_workspace_size(const ssd_fwd_params *p)
{
    if (validate(p) != SSD_OK || !bwd_supported(*p)) return 0;
    return bwd_layout(*p).total;
}

ssd_status ssd_bwd(const ssd_fwd_params *p, const void *x, const void *dt, const float *A_log, const void *B,
                   const void *C, const float *D, const float *initial_states, const int32_t *cu_seqlens,
                   const void *dy, const float *dfinal_states, float *dx, float *ddt, float *dA_log, float *dB,
                   float *dC, float *dD, float *dinitial_states, void *workspace, size_t workspace_bytes,
                   void *stream)
{
    try {
        const ssd_status v = validate(p);
        if (v != SSD_OK) return v;
        if (!bwd_supported(*p)) return SSD_ERR_UNSUPPORTED;
        const bool has_tokens = (long long)p->batch * p->seqlen > 0;
        if (!A_log || !workspace || !dA_log || !dD) return SSD_ERR_INVALID_ARG;
        if (has_tokens && (!x || !dt || !B || !C || !dy || !dx || !ddt || !dB || !dC)) return SSD_ERR_INVALID_ARG;
        if ((p->num_seqs > 0) != (cu_seqlens != nullptr)) return SSD_ERR_INVALID_ARG;
        const void *ptrs[] = {x, dt, A_log, B, C, D, initial_states, cu_seqlens, dy, dfinal_states, dx, ddt,
                              dA_log, dB, dC, dD, dinitial_states};
        for (const void *q : ptrs)
            if (q && !aligned16(q)) return SSD_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return SSD_ERR_INVALID_ARG;
        const BwdLayout L = bwd_layout(*p);
        if (workspace_bytes < L.total) return SSD_ERR_INVALID_ARG;

        cudaStream_t st = static_cast<cudaStream_t>(stream);
        char *ws = static_cast<char *>(workspace);
        Plan plan;
        plan.status = reinterpret_cast<int *>(ws + L.status);
        plan.count = reinterpret_cast<int *>(ws + L.count);
        plan.chunks = reinterpret_cast<ChunkDesc *>(ws + L.chunks);
        plan.seqs = reinterpret_cast<SeqDesc *>(ws + L.seqs);
        plan.nseq = nseq_of(*p);
        plan.max_chunks = (int)bwd_chunk_count(*p);
        Dims d;
        d.H = p->nheads;
        d.P = p->headdim;
        d.N = p->dstate;
        d.G = p->ngroups;
        d.Q = bwd_chunk_len();
        d.heads_per_group = p->nheads / p->ngroups;
        d.tokens = p->batch * p->seqlen;
        d.dt_softplus = p->dt_softplus;
        if (launch_build_plan(plan, cu_seqlens, p->batch, p->seqlen, d.Q, st) != cudaSuccess) return SSD_ERR_CUDA;
        SimtArgs fa;
        fa.x = x; fa.dt = dt; fa.B = B; fa.C = C;
        fa.A_log = A_log; fa.D = D; fa.init = initial_states;
        fa.y = nullptr; fa.final_states = nullptr;
        fa.cs = reinterpret_cast<float *>(ws + L.cs);
        fa.dv = reinterpret_cast<float *>(ws + L.dv);
        fa.states = reinterpret_cast<float *>(ws + L.states);
        fa.bf16 = p->io_dtype == SSD_DTYPE_BF16;
        const cudaError_t e = launch_bwd(plan, d, fa, dy, dfinal_states, reinterpret_cast<float *>(ws + L.gbuf), dx,
                                         ddt, dA_log, dB, dC, dD, dinitial_states, fa.bf16, st);
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    } catch (...) {
        return SSD_ERR_CUDA;
    }
}

ssd_status ssd_get_status(const void *workspace, void *stream)
{
    if (!workspace) return SSD_ERR_INVALID_ARG;
    int code = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&code, workspace, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSD_ERR_CUDA;
    switch (code) {
    case kDevOk: return SSD_OK;
    case kDevTimeout: return SSD_ERR_TIMEOUT;
    case kDevBadSeqlens: return SSD_ERR_BAD_SEQLENS;
    default: return SSD_ERR_CUDA;
    }
}

}  // extern "C"
