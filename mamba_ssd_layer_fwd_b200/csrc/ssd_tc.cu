// Tensor-core path of the SSD forward for sm_100a (tcgen05 / TMEM / TMA).
//
// Method ("Transformers are SSMs", Sec. 6, block decomposition of the
// semiseparable matrix M = L o (C B^T)), evaluated by one CTA per work item
// = (sequence, block of KH heads sharing a B/C group, token segment).  The
// CTA walks its segment in 128-token blocks, keeping every head's P x N
// state in tensor memory (fp32) between blocks, so chunk states never go
// through HBM.  Per block c and head h (q = 128 tokens, rows l, columns s):
//
//   cs_l   = sum_{k<=l} delta_k A_h                     (cumsum warp, fp32)
//   CB     = C_c B_c^T                    (UMMA, K = N; once per block, shared by the KH heads)
//   Pm     = CB o exp(cs_l - cs_s) delta_s  (s <= l), + D_h on the diagonal
//                                          (mask warps, TMEM -> regs -> TMEM as bf16)
//   Yd     = Pm X_c                       (UMMA, A operand from TMEM)  Sec. 6.1
//   Yo     = C_c Hbf^T,  Hbf = bf16(H)    (UMMA)                       Sec. 6.2 left factor
//   y_l    = Yd_l + exp(cs_l) Yo_l        (epilogue warps -> HBM)
//   H     <- exp(cs_last) H + B_c^T (w o X_c),  w_s = exp(cs_last - cs_s) delta_s
//                                          (state warps rescale H in TMEM, UMMA accumulates)
//                                          Sec. 6.2 right + centre factors
//
// Exponents that are <= 0 in exact arithmetic (cs_l - cs_s with s <= l) are
// clamped at 0: with a huge decay rate the fp32 prefix sums can round them
// above 0, and the exponential would overflow.
//
// Each diagonal block of the caller's chunk length Q (128 or 256) is thereby
// computed by the same decomposition one level down with 128-token blocks;
// Sec. 6.1 leaves the method for a diagonal block free, and the result is
// the same up to rounding.
//
// Warp roles (16 warps; warp w runs on SM sub-partition w % 4 and may only
// touch TMEM lanes 32*(w%4) .. +31): 0 cumsum, 1 UMMA issuer for the state
// path (H += B^T (w o X); also C Hbf^T when dstate is 256), 2 TMA producer,
// 3 UMMA issuer for the output path (CB, C Hbf^T, Pm X) + TMEM owner, 4-7
// and 10-11 mask (the causal work of rows 96-127 is four times that of rows
// 0-31, so sub-partitions 0-1 also get the w o X pass, warps 8-9), 12-15
// state rescale + output epilogue.  Two issuers keep the state and output paths from waiting on
// each other.  Every mbarrier wait is bounded (2 s); on a timeout the CTA
// records SSD_ERR_TIMEOUT in the status word, drains, frees TMEM and exits.
//
// Equal-length rows take their work item from the block index (no planner
// kernel): whole waves of the SMs walk whole rows; the pairs left over run as
// one-head items in a second launch, or (rows of many blocks, or fewer pairs
// than SMs) are cut into segments and run by ssd_tc_fused, in which each
// segment's CTA computes its end state from zero (state-only walk), the CTAs
// of a pair chain the segment states between them, and every CTA then walks
// its segment from its true entering state (Sec. 8.2: state passing between
// pieces of a sequence).  Packed sequences take items from a planner kernel;
// when they must be cut, a state-only launch, a scan kernel and the full walk
// do the same in three launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstddef>

#include "ssd_tc.cuh"
#include "ssd_tc_prims.cuh"

namespace ssd {
namespace {

using namespace tc;

constexpr int kQ = 128;          // tokens per block (TMEM lanes, UMMA M)
constexpr int kP = 64;           // head dim
constexpr int kThreadsTc = 512;  // 16 warps
constexpr int kMaskWarps = 6;    // warps 4-7, 10, 11
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kCsd = 4;          // depth of the per-(block, head) cumsum ring
constexpr int kPrefetch = 1;     // blocks of L2 prefetch ahead of the TMA loads

struct TcItem {
    int seq;     // sequence index
    int tok0;    // first token of the segment (flattened token axis)
    int len;     // tokens in the segment (>= 1)
    int gseg;    // global segment index (segment-state buffer row)
    int seg;     // segment index inside the sequence
    int nseg;    // segments of the sequence
    int h0;      // first head of the block
    int pad;
};

// Gated norm of the block output (walk variant GN): out = GroupNorm(y * silu(z))
// over each head's 64 channels, with per-channel weight and bias.  A kernel
// argument of its own, so that the other variants' parameter block is unchanged.
struct GnParams {
    const __nv_bfloat16 *z;
    const float *w, *b;
    float eps;
};

struct TcParams {
    const __nv_bfloat16 *dt;
    const float *A_log, *D, *init;
    __nv_bfloat16 *y;
    float *final_states;
    float *segstate;      // [max_segments][H][P][N]: pass-1 end states, then entering states
    float *seglogdec;     // [max_segments][H]: sum of delta*A over the segment
    const TcItem *items;  // null: equal-length rows of one segment each (see direct_base)
    const int *count;
    int *status;
    // items == null: item i of this launch covers heads row * H + h0 .. + KH - 1 of
    // the flattened (row, head) index g = direct_base + i * KH; n_items items
    int n_items, direct_base, seqlen;
    int H, G, N, heads_per_group;
    int dt_softplus;
    int withhold_x0;      // testing: work item 0 never loads its first x tile (bounded waits expire)
    int summary;          // state-only mode over whole sequences: end state from zero and total
                          // log decay of every sequence, written to row `seq` of segstate / seglogdec
};

// softplus(v) = max(v, 0) + log1p(e), e = exp(-|v|) in (0, 1], in a dozen
// instructions (the cumsum warp evaluates it for every token and head, on the
// path that feeds the mask).  log1p(e) = log(w) * e / (w - 1), w = 1 + e
// rounded (e itself when w rounds to 1): the factor e / (w - 1) cancels the
// rounding of w (Goldberg, "What every computer scientist should know about
// floating-point arithmetic", 1991, the log(1 + x) theorem), so the error is
// that of the hardware logarithm, below 4e-7 absolute on [1, 2].  Summed over
// a 128-token block with |A| <= 16 that moves a decay exponent by < 1e-3, far
// inside the bf16 rounding of the block's products.
__device__ __forceinline__ float softplus_fast(float v)
{
    const float e = __expf(-fabsf(v));
    const float w = 1.0f + e;
    const float lp = w == 1.0f ? e : __logf(w) * __fdividef(e, w - 1.0f);
    return fmaxf(v, 0.0f) + lp;
}

// --------------------------------------------------------------- smem layout
// The mbarriers of one walk.
struct TcBars {
    uint64_t bc_full[2], bc_empty[2], x_full[2], x_empty[2], cs_full[kCsd], cs_empty[kCsd];
    uint64_t cb_full, cb_empty, pm_full[2], pm_empty[2], hb_full, hb_empty, xw_full[2], xw_empty[2], xw_free[2];
    uint64_t yo_full;
    uint64_t h_ready[2], hs_full[2], y_full, yo_empty, yd_empty, drain_o, drain_s;
    uint64_t xs_full[4], xs_empty[4], xws_full[4];   // state-only mode's X ring (w o X in place)
};

template <int NST>
struct __align__(1024) TcSmem {
    static constexpr int kBoxes = NST / 64;
    static constexpr int kStages = NST >= 256 ? 1 : 2;   // B/C ring depth (dstate 256: one stage fits)
    static constexpr int kXw = NST >= 256 ? 1 : 2;       // w o X ring depth
    uint8_t bc[kStages][2][kBoxes][16384];   // [stage][0 = C, 1 = B][64-column box][128 rows x 128 B]
    uint8_t x[2][16384];               // X blocks (ring over (block, head))
    uint8_t xw[kXw][16384];            // w o X (ring over (block, head))
    uint8_t hbf[NST * 128];            // bf16(H)^T: rows n, 64 p per 128 B row
    float cs2[kCsd][kQ];               // log2-scaled inclusive cumsum of delta*A
    float dl[kCsd][kQ];                // delta_s (0 on padding rows)
    float w[kCsd][kQ];                 // exp(cs_last - cs_s) * delta_s
    float e[kCsd][kQ];                 // exp(cs_l)
    float u[kCsd][kQ];                 // exp(cs_{s0} - cs_s) * delta_s, s0 = start of s's 16-column chunk
    int exact[kCsd];                   // 1: some 16-token chunk decays too fast for the factorised mask
    float alpha[kCsd];                 // exp(cs_last)
    float ldec[kCsd];                  // cs_last (natural log of the block decay)
    TcBars bar[2];                     // one barrier set per walk of the CTA
    uint32_t tmem_base;
    int abort;
};

template <int NST>
constexpr size_t tc_smem_bytes()
{
    return sizeof(TcSmem<NST>) + 1024;   // + alignment slack
}
// opt-in shared memory per block on sm_100 (227 KB)
static_assert(tc_smem_bytes<64>() <= 232448 && tc_smem_bytes<128>() <= 232448 && tc_smem_bytes<256>() <= 232448,
              "walk kernel shared memory exceeds the per-block limit");

__device__ __forceinline__ void record_timeout(int *status) { set_status(status, kDevTimeout); }

// TMEM column map (512 columns): CB at 0, the Pm buffers from 128, every
// head's state from 256.  With two heads at dstate 256 the states fill
// 256..511, so Pm is single-buffered and Yd and Yo share one accumulator at
// 192 (the epilogue reads Yo before Pm X overwrites it); otherwise Pm is
// double-buffered and Yd, Yo sit at 384 and 448.
constexpr uint32_t kColCB = 0, kColPm = 128, kColH = 256;
template <int NST, int KH>
struct TmemMap {
    static constexpr int kMT = NST >= 256 ? 2 : 1;                 // 128-row state tiles per head
    static constexpr bool kSharedY = KH * kMT * 64 > 128;
    static constexpr int kPmBufs = kSharedY ? 1 : 2;
    static constexpr uint32_t kColYd = kSharedY ? 192u : 384u;
    static constexpr uint32_t kColYo = kSharedY ? 192u : 448u;
    static_assert(kColH + KH * kMT * 64 <= 512, "states do not fit in tensor memory");
};

// Optional per-CTA event timeline (SM clock), compiled only with -DSSD_TRACE.
#ifdef SSD_TRACE
constexpr int kTraceEvents = 28, kTraceUnits = 64, kTraceCtas = 8;
__device__ long long *g_trace = nullptr;
#define SSD_TRACE_EV(ev, idx)                                                                           \
    do {                                                                                                \
        if (trace_buf && (idx) < kTraceUnits)                                                           \
            trace_buf[((size_t)blockIdx.x * kTraceEvents + (ev)) * kTraceUnits + (idx)] = clock64() - t_start; \
    } while (0)
#else
#define SSD_TRACE_EV(ev, idx) \
    do {                      \
    } while (0)
#endif

// One walk over a work item's segment: the state-only walk (end state from
// zero, backwards) or the full walk (outputs and the end state), by the CTA's
// 512 threads with barrier set Bb (initialised here), TMEM columns from tb.
// srow: row of segstate / seglogdec that holds head it.h0 of this segment
// (the heads of the item are srow .. srow + KH - 1).
template <int NST, int KH, bool STATE_ONLY, bool GN>
__device__ __forceinline__ void walk_body(const CUtensorMap &mapX, const CUtensorMap &mapB, const CUtensorMap &mapC,
                                          const CUtensorMap &mapY, const TcParams &prm, const GnParams &gnp,
                                          TcSmem<NST> &S, TcBars &Bb, const uint32_t tb, const TcItem &it,
                                          const int item_idx, const int srow)
{
    // dstate 256 keeps more live registers: there the out-of-line wait call spills
    constexpr bool kInlW = NST >= 256;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q = warp & 3;                             // SM sub-partition = TMEM lane quarter
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const int nblk = (it.len + kQ - 1) / kQ;
    const int nunits = nblk * KH;
    const int g = it.h0 / prm.heads_per_group;
    volatile int *abort = &S.abort;
    constexpr int kSt = TcSmem<NST>::kStages, kXwD = TcSmem<NST>::kXw;
    // Whole 128-token output blocks are staged in the unit's w o X slot (free once the
    // state UMMA has read it) and written by TMA stores, one 32-row slab per epilogue
    // warp: coalesced full-line writes instead of 16-byte pieces of 32 rows.  Needs
    // two w o X slots, so the next unit's w o X pass runs meanwhile.
    constexpr bool kTmaY = !STATE_ONLY && kXwD >= 2;
    // dstate 256 (one head per item): C bf16(H)^T is issued by the state issuer, so it
    // never queues behind the mask-bound Pm X (+3 % there; slower with two heads)
    constexpr bool kYoOnState = !STATE_ONLY && NST >= 256;
    constexpr int kMT = TmemMap<NST, KH>::kMT;     // 128-row state tiles per head (H^T rows = n)
    constexpr bool kSharedY = !STATE_ONLY && TmemMap<NST, KH>::kSharedY;
    constexpr int kPmB = TmemMap<NST, KH>::kPmBufs;
    constexpr uint32_t kColYd = TmemMap<NST, KH>::kColYd, kColYo = TmemMap<NST, KH>::kColYo;
    // the shared Y accumulator needs Yo issued by the state issuer (its own yo_full commit)
    static_assert(!kSharedY || kYoOnState, "shared Yd/Yo accumulator needs the state issuer to issue Yo");
    // state-only mode at dstate 256 runs a two-stage B ring in the C and B slots of the single B/C stage
    constexpr int kBR = (STATE_ONLY && kSt == 1) ? 2 : kSt;
    // one B/C stage with outputs: B and C have their own full/empty barriers (C: bc_*[0], B: bc_*[1]),
    // so the next block's B loads once the last state UMMA is done, while C still feeds C Hbf^T
    constexpr bool kSplitBC = !STATE_ONLY && kSt == 1;
    static_assert(!kSplitBC || kYoOnState, "a split B/C stage assumes the state issuer issues C Hbf^T");
    // two heads sharing Yd/Yo: the second head's Pm is written over the CB columns its mask has
    // just read (K steps 0-3 at columns 0-31, 4-7 at 64-95), so it does not wait for the first
    // head's Pm X; the next CB waits for that Pm X instead
    constexpr bool kInPlace = kSharedY && KH == 2;
    // state-only mode: one state UMMA per block for both heads (N = 128, the B^T operand read once);
    // the heads' states are adjacent per 128-row tile (column kColH + 64 (j + KH mt)) and so are
    // their w o X tiles (at dstate 256 in the bf16(H) tile, which state-only mode does not use)
    constexpr bool kMergeSt = STATE_ONLY && KH == 2;
    constexpr int kXwR = kXwD;                                      // w o X ring depth (full walk)
    auto xw_tile = [&](int i) -> uint8_t * { return S.xw[i]; };
    // X ring: two slots; in state-only mode four (barriers xs_*), laid over the x, w o X and
    // (dstate 256) bf16(H) tiles, contiguous and otherwise unused there, with w o X written
    // over X in place and the slot freed by the state UMMA, so X loads run two blocks ahead
    constexpr int kXR = STATE_ONLY ? 4 : 2;
    static_assert(offsetof(TcSmem<NST>, xw) == offsetof(TcSmem<NST>, x) + sizeof(S.x) &&
                      offsetof(TcSmem<NST>, hbf) == offsetof(TcSmem<NST>, xw) + sizeof(S.xw) &&
                      sizeof(S.x) + sizeof(S.xw) + sizeof(S.hbf) >= 4 * 16384,
                  "the state-only X ring needs four contiguous 16 KB tiles");
    auto x_tile = [&](int i) -> uint8_t * { return STATE_ONLY ? S.x[0] + 16384 * i : S.x[i]; };
    uint64_t *const x_full_b = STATE_ONLY ? Bb.xs_full : Bb.x_full;
    uint64_t *const x_empty_b = STATE_ONLY ? Bb.xs_empty : Bb.x_empty;
    auto b_tile = [&](int stage) -> uint8_t * {
        return (STATE_ONLY && kSt == 1) ? S.bc[0][stage][0] : S.bc[stage][1][0];
    };

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&Bb.bc_full[i], 1);
            mbar_init(&Bb.bc_empty[i], STATE_ONLY ? 1 : 2);    // state issuer (+ output issuer)
            mbar_init(&Bb.x_full[i], 1);
            mbar_init(&Bb.x_empty[i], STATE_ONLY ? 2 : 3);     // w o X warps (+ output issuer)
            mbar_init(&Bb.xw_full[i], 2);
            mbar_init(&Bb.xw_empty[i], kTmaY ? 4 : 1);       // epilogue warps, else the state issuer
            mbar_init(&Bb.xw_free[i], 1);
            mbar_init(&Bb.pm_full[i], kMaskWarps);
            mbar_init(&Bb.pm_empty[i], 1);
            mbar_init(&Bb.h_ready[i], 1);
            mbar_init(&Bb.hs_full[i], 4);      // per head: H rescaled for its next block
        }
        for (int i = 0; i < kCsd; ++i) {
            mbar_init(&Bb.cs_full[i], 32);
            mbar_init(&Bb.cs_empty[i], STATE_ONLY ? 6 : 6 + kMaskWarps);
        }
        mbar_init(&Bb.cb_full, 1);
        mbar_init(&Bb.cb_empty, kMaskWarps);
        mbar_init(&Bb.hb_full, 4);
        mbar_init(&Bb.hb_empty, 1);
        mbar_init(&Bb.y_full, 1);
        mbar_init(&Bb.yo_full, 1);
        mbar_init(&Bb.yo_empty, 4);
        mbar_init(&Bb.yd_empty, 4);
        mbar_init(&Bb.drain_o, 1);
        mbar_init(&Bb.drain_s, 1);
        if (STATE_ONLY)
            for (int i = 0; i < 4; ++i) {
                mbar_init(&Bb.xs_full[i], 1);
                mbar_init(&Bb.xs_empty[i], 1);     // the state UMMA
                mbar_init(&Bb.xws_full[i], 2);     // w o X warps
            }
        mbar_fence_init();
    }
    __syncthreads();
#ifdef SSD_TRACE
    const long long t_start = clock64();
    long long *const trace_buf = (blockIdx.x < kTraceCtas && !STATE_ONLY) ? g_trace : nullptr;
#endif

    // state-only mode with two heads: the idle mask warp 4 takes the second head's units, so the
    // cumsum (about a global-load latency plus ~1k cycles per unit) keeps pace with the walk
    constexpr bool kCs2 = STATE_ONLY && KH == 2;
    if (warp == 0 || (kCs2 && warp == 4)) {
        // ----------------------------------------------------------- cumsum
        // dt of a unit is loaded before waiting for its ring slot.
        const int H = prm.H;
        float Areg[KH];
#pragma unroll
        for (int j = 0; j < KH; ++j) Areg[j] = -expf(prm.A_log[it.h0 + j]);
        // state-only mode walks the segment backwards: rsum[j] = log decay of the blocks
        // already walked (those after the current one), folded into w
        float rsum[KH];
#pragma unroll
        for (int j = 0; j < KH; ++j) rsum[j] = 0.0f;
        bool ok = true;
        for (int u = kCs2 && warp == 4 ? 1 : 0; u < nunits && ok; u += kCs2 ? 2 : 1) {
            const int c = STATE_ONLY ? nblk - 1 - u / KH : u / KH, j = u % KH, slot = u % kCsd;
            const int row0 = it.tok0 + c * kQ;
            const int valid = min(kQ, it.len - c * kQ);
            const int h = it.h0 + j;
            float r[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int l = lane * 4 + i;
                r[i] = l < valid ? __bfloat162float(prm.dt[(size_t)(row0 + l) * H + h]) : 0.0f;
            }
            float A = Areg[0];
#pragma unroll
            for (int jj = 1; jj < KH; ++jj)
                if (j == jj) A = Areg[jj];
            if (u >= kCsd) ok = mbar_wait<kInlW>(&Bb.cs_empty[slot], ((u / kCsd) + 1) & 1, abort);
            if (!ok) break;
            // lane owns tokens 4*lane .. 4*lane+3
            float dl[4], pre[4];
            float run = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int l = lane * 4 + i;
                float d = 0.0f;
                if (l < valid) d = prm.dt_softplus ? softplus_fast(r[i]) : r[i];
                dl[i] = d;
                run += d * A;
                pre[i] = run;
            }
            float incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const float excl = incl - run;
            const float last = __shfl_sync(0xffffffffu, incl, 31);
            float rs = 0.0f;
            if (STATE_ONLY) {
#pragma unroll
                for (int jj = 0; jj < KH; ++jj)
                    if (j == jj) {
                        rs = rsum[jj];
                        rsum[jj] += last;
                    }
            }
            float c2v[4], wv[4], ev[4], uv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float csn = excl + pre[i];
                c2v[i] = csn * kLog2e;
                // decay from token s to the block end (and, walking backwards, on to the segment end)
                wv[i] = ex2_approx(fminf(STATE_ONLY ? last - csn + rs : last - csn, 0.0f) * kLog2e) * dl[i];
                ev[i] = ex2_approx(c2v[i]);
            }
            // factorised mask: exp2(cs2_l - cs2_s) = exp2(cs2_l - R) * exp2(R - cs2_s) with R the
            // cs2 of the first token of s's 16-token chunk (lanes 4k..4k+3 hold chunk k)
            const float Rk = __shfl_sync(0xffffffffu, c2v[0], lane & ~3);
            const float chunk_end = __shfl_sync(0xffffffffu, c2v[3], lane | 3);
#pragma unroll
            for (int i = 0; i < 4; ++i) uv[i] = ex2_approx(Rk - c2v[i]) * dl[i];
            const int exact = __any_sync(0xffffffffu, Rk - chunk_end > 96.0f) ? 1 : 0;
            *reinterpret_cast<float4 *>(&S.cs2[slot][lane * 4]) = make_float4(c2v[0], c2v[1], c2v[2], c2v[3]);
            *reinterpret_cast<float4 *>(&S.dl[slot][lane * 4]) = make_float4(dl[0], dl[1], dl[2], dl[3]);
            *reinterpret_cast<float4 *>(&S.w[slot][lane * 4]) = make_float4(wv[0], wv[1], wv[2], wv[3]);
            *reinterpret_cast<float4 *>(&S.e[slot][lane * 4]) = make_float4(ev[0], ev[1], ev[2], ev[3]);
            *reinterpret_cast<float4 *>(&S.u[slot][lane * 4]) = make_float4(uv[0], uv[1], uv[2], uv[3]);
            if (lane == 0) {
                S.alpha[slot] = ex2_approx(last * kLog2e);
                S.ldec[slot] = last;
                S.exact[slot] = exact;
            }
            mbar_arrive(&Bb.cs_full[slot]);
            if (lane == 0) SSD_TRACE_EV(6, u);
        }
    } else if (warp == 1) {
        // ---------------------------------------------- UMMA issuer: state path
        // H_j <- H_j + B_c^T (w o X)   (H_j already rescaled by exp(cs_last) by the state warps)
        {
            // the whole warp runs the loop; one elected lane issues
            const bool leader = elect_one();
            const uint32_t id_h = idesc_bf16_f32(128, kP, true, true);
            const uint32_t id_y = idesc_bf16_f32(128, kP, false, true);
            const uint32_t id_h2 = idesc_bf16_f32(128, 2 * kP, true, true);
            const uint32_t lbo_m = NST >= 128 ? 16384u : 0u;   // N = 64: rows 64..127 repeat rows 0..63
            bool ok = true;
            for (int c = 0; c < nblk && ok; ++c) {
                const int bs = c % kBR;
                ok = mbar_wait<kInlW>(&Bb.bc_full[kSplitBC ? 1 : bs], (c / kBR) & 1, abort);
                if (!ok) break;
                const uint32_t sB = smem_u32(b_tile(bs));
                if (kMergeSt) {
                    // both heads: the w o X tiles of u = 2c, 2c + 1 (adjacent slots) form one N = 128 operand
                    const int s0 = (2 * c) % kXR, ph = ((2 * c) / kXR) & 1;
                    ok = mbar_wait<kInlW>(&Bb.xws_full[s0], ph, abort) && mbar_wait<kInlW>(&Bb.xws_full[s0 + 1], ph, abort) &&
                         (c > 0 || (mbar_wait<kInlW>(&Bb.hs_full[0], 0, abort) && mbar_wait<kInlW>(&Bb.hs_full[1], 0, abort)));
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t b0 = sdesc_sw128(smem_u32(x_tile(s0)), 16384, 1024);
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        const uint64_t a0 = sdesc_sw128(sB + mt * 32768, lbo_m, 1024);
#pragma unroll
                        for (int kk = 0; kk < kQ / 16; ++kk)
                            if (leader)
                                umma_ss(tb + kColH + 64 * KH * mt, desc_adv(a0, kk * 2048), desc_adv(b0, kk * 2048),
                                        id_h2, 1);
                    }
                    if (leader) {
                        umma_commit(&Bb.xs_empty[s0]);
                        umma_commit(&Bb.xs_empty[s0 + 1]);
                        umma_commit(&Bb.h_ready[0]);
                        umma_commit(&Bb.h_ready[1]);
                        umma_commit(&Bb.bc_empty[bs]);
                    }
                    continue;
                }
                for (int j = 0; j < KH && ok; ++j) {
                    const int u = c * KH + j;
                    // w o X: its own ring, or (state-only mode) in place in the X ring
                    const int wi = STATE_ONLY ? u % kXR : u % kXwR;
                    // state-only mode never rescales: hs_full[j] completes once, when the zeroed state is in place
                    ok = (STATE_ONLY ? mbar_wait<kInlW>(&Bb.xws_full[wi], (u / kXR) & 1, abort)
                                     : mbar_wait<kInlW>(&Bb.xw_full[wi], (u / kXwR) & 1, abort)) &&
                         (STATE_ONLY ? (c > 0 || mbar_wait<kInlW>(&Bb.hs_full[j], 0, abort))
                                     : mbar_wait<kInlW>(&Bb.hs_full[j], c & 1, abort));
                    SSD_TRACE_EV(15, u);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t b0 = sdesc_sw128(smem_u32(STATE_ONLY ? x_tile(wi) : xw_tile(wi)), 16384, 1024);
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        const uint64_t a0 = sdesc_sw128(sB + mt * 32768, lbo_m, 1024);
#pragma unroll
                        for (int kk = 0; kk < kQ / 16; ++kk)
                            if (leader)
                                umma_ss(tb + kColH + 64 * (j + KH * mt), desc_adv(a0, kk * 2048),
                                        desc_adv(b0, kk * 2048), id_h, 1);
                    }
                    if (leader) umma_commit(STATE_ONLY ? &Bb.xs_empty[wi] : kTmaY ? &Bb.xw_free[wi] : &Bb.xw_empty[wi]);
                    if (leader) umma_commit(&Bb.h_ready[j]);
                    if (kSplitBC && j == KH - 1 && leader) umma_commit(&Bb.bc_empty[1]);   // B of block c done
                    SSD_TRACE_EV(4, u);
                    if (kYoOnState) {
                        // the accumulator is free once the epilogue has read the previous unit's
                        // Yo (its own columns) or Yd (columns shared with Yo)
                        ok = mbar_wait<kInlW>(&Bb.hb_full, u & 1, abort) &&
                             (u == 0 || mbar_wait<kInlW>(kSharedY ? &Bb.yd_empty : &Bb.yo_empty, (u - 1) & 1, abort)) &&
                             (!kSplitBC || j > 0 || mbar_wait<kInlW>(&Bb.bc_full[0], c & 1, abort));
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t c0 = sdesc_sw128(smem_u32(S.bc[bs][0][0]), 16, 1024);
                        const uint64_t h0 = sdesc_sw128(smem_u32(S.hbf), 16384, 1024);
#pragma unroll
                        for (int kk = 0; kk < NST / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            if (leader)
                                umma_ss(tb + kColYo, desc_adv(c0, off), desc_adv(h0, kk * 2048), id_y, kk > 0);
                        }
                        if (leader) umma_commit(&Bb.hb_empty);
                        if (leader) umma_commit(&Bb.yo_full);
                        SSD_TRACE_EV(27, u);
                    }
                }
                if (leader) umma_commit(&Bb.bc_empty[kSplitBC ? 0 : bs]);   // (C of block c done)
            }
            if (leader) umma_commit(&Bb.drain_s);
            mbar_wait<kInlW>(&Bb.drain_s, 0, abort, 200000000ull);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&mapX);
            tma_prefetch_desc(&mapB);
            if (!STATE_ONLY) tma_prefetch_desc(&mapC);
            constexpr uint32_t kBoxBytes = 16384;
            constexpr uint32_t kBcBytes = (STATE_ONLY ? 1 : 2) * (NST / 64) * kBoxBytes;
            int issued_bc[2] = {-1, -1}, issued_x[kXR];
#pragma unroll
            for (int i = 0; i < kXR; ++i) issued_x[i] = -1;
            bool ok = true;
            // L2 prefetch runs kPF blocks ahead of the shared-memory ring
            constexpr int kPF = STATE_ONLY ? 1 : (NST >= 256 ? 2 : kPrefetch);
            auto prefetch = [&](int c) {
                const int blk = STATE_ONLY ? nblk - 1 - c : c;
                const int row = it.tok0 + blk * kQ;   // state-only: backwards
                {
                    // the block's dt rows (every head), read by the cumsum warp with plain loads:
                    // 16-byte aligned and inside the segment
                    const int rows = min(kQ, it.len - blk * kQ);
                    const uintptr_t b0 = reinterpret_cast<uintptr_t>(prm.dt + (size_t)row * prm.H);
                    const uintptr_t e0 = reinterpret_cast<uintptr_t>(prm.dt + (size_t)(row + rows) * prm.H);
                    const uintptr_t a0 = (b0 + 15) & ~(uintptr_t)15, a1 = e0 & ~(uintptr_t)15;
                    if (a1 > a0) prefetch_l2_bulk(reinterpret_cast<const void *>(a0), (uint32_t)(a1 - a0));
                }
                for (int b = 0; b < NST / 64; ++b) {
                    if (!STATE_ONLY) tma_prefetch_l2_2d(&mapC, g * NST + 64 * b, row);
                    tma_prefetch_l2_2d(&mapB, g * NST + 64 * b, row);
                }
                for (int j = 0; j < KH; ++j) tma_prefetch_l2_2d(&mapX, (it.h0 + j) * kP, row);
            };
            // split B/C stage: one half (1 = B, 0 = C) of block c
            auto load_half = [&](int c, int half) -> bool {
                const int row = it.tok0 + (STATE_ONLY ? nblk - 1 - c : c) * kQ;   // state-only: backwards
                if (c >= 1 && !mbar_wait<kInlW>(&Bb.bc_empty[half], (c + 1) & 1, abort)) return false;
                mbar_arrive_expect_tx(&Bb.bc_full[half], (NST / 64) * 16384u);
                for (int b = 0; b < NST / 64; ++b)
                    tma_load_2d(S.bc[0][half][b], half ? &mapB : &mapC, &Bb.bc_full[half], g * NST + 64 * b, row);
                issued_bc[half] = c;
                if (half == 0) SSD_TRACE_EV(0, c);
                return true;
            };
            auto load_bc = [&](int c) -> bool {
                const int row = it.tok0 + (STATE_ONLY ? nblk - 1 - c : c) * kQ;   // state-only: backwards
                const int bs = c % kBR;
                if (c >= kBR && !mbar_wait<kInlW>(&Bb.bc_empty[bs], ((c / kBR) + 1) & 1, abort)) return false;
                mbar_arrive_expect_tx(&Bb.bc_full[bs], kBcBytes);
                uint8_t *bdst = b_tile(bs);
                for (int b = 0; b < NST / 64; ++b) {
                    if (!STATE_ONLY) tma_load_2d(S.bc[bs][0][b], &mapC, &Bb.bc_full[bs], g * NST + 64 * b, row);
                    tma_load_2d(bdst + 16384 * b, &mapB, &Bb.bc_full[bs], g * NST + 64 * b, row);
                }
                issued_bc[bs] = c;
                SSD_TRACE_EV(0, c);
                return true;
            };
            auto load_x = [&](int c, int j0, int j1) -> bool {
                const int row = it.tok0 + (STATE_ONLY ? nblk - 1 - c : c) * kQ;   // state-only: backwards
                for (int j = j0; j < j1; ++j) {
                    const int u = c * KH + j, xs = u % kXR;
                    if (u >= kXR && !mbar_wait<kInlW>(&x_empty_b[xs], ((u / kXR) + 1) & 1, abort)) return false;
                    if (prm.withhold_x0 && item_idx == 0 && u == 0) continue;
                    mbar_arrive_expect_tx(&x_full_b[xs], kBoxBytes);
                    tma_load_2d(x_tile(xs), &mapX, &x_full_b[xs], (it.h0 + j) * kP, row);
                    issued_x[xs] = u;
                    SSD_TRACE_EV(1, u);
                }
                return true;
            };
            for (int c = 0; c < nblk && ok; ++c) {
#pragma unroll 1
                for (int pc = c == 0 ? 0 : c + kPF; pc <= c + kPF && pc < nblk; ++pc) prefetch(pc);
                // the single-threaded producer requests tiles in the order their slots free up:
                // with a split B/C stage B (last state UMMA), x of the first heads (their Pm X),
                // C (last C Hbf^T), x of the last head (the block's final Pm X)
                if (kSplitBC)
                    ok = load_half(c, 1) && load_x(c, 0, KH - 1) && load_half(c, 0) && load_x(c, KH - 1, KH);
                else if (kBR == 1)
                    ok = load_x(c, 0, KH) && load_bc(c);
                else
                    ok = load_bc(c) && load_x(c, 0, KH);
            }
            if (!ok) {
                // drain: wait (bounded) for copies still in flight before the CTA exits
                for (int i = 0; i < 2; ++i) {
                    if (kSplitBC && issued_bc[i] >= 0)
                        mbar_wait<kInlW>(&Bb.bc_full[i], issued_bc[i] & 1, abort, 200000000ull);
                    else if (i < kBR && issued_bc[i] >= 0)
                        mbar_wait<kInlW>(&Bb.bc_full[i], (issued_bc[i] / kBR) & 1, abort, 200000000ull);
                }
                for (int i = 0; i < kXR; ++i)
                    if (issued_x[i] >= 0) mbar_wait<kInlW>(&x_full_b[i], (issued_x[i] / kXR) & 1, abort, 200000000ull);
            }
        }
    } else if (warp == 3) {
        // --------------------------------------------- UMMA issuer: output path
        if (!STATE_ONLY) {
            // the whole warp runs the loop; one elected lane issues
            const bool leader = elect_one();
            const uint32_t id_cb = idesc_bf16_f32(128, 128, false, false);
            const uint32_t id_y = idesc_bf16_f32(128, kP, false, true);
            bool ok = true;
            // CB = C_c B_c^T into the single CB accumulator
            auto issue_cb = [&](int c) -> bool {
                const int bs = c % kSt;
                if (!mbar_wait<kInlW>(&Bb.bc_full[bs], (c / kSt) & 1, abort)) return false;
                if (kSplitBC && !mbar_wait<kInlW>(&Bb.bc_full[1], c & 1, abort)) return false;
                if (c >= 1 && !mbar_wait<kInlW>(&Bb.cb_empty, (c - 1) & 1, abort)) return false;
                // the previous block's last Pm lives in the CB columns until its Pm X is done
                if (kInPlace && c >= 1 && !mbar_wait<kInlW>(&Bb.pm_empty[1], (c - 1) & 1, abort)) return false;
                tc_fence_after();
                const uint64_t a0 = sdesc_sw128(smem_u32(S.bc[bs][0][0]), 16, 1024);
                const uint64_t b0 = sdesc_sw128(smem_u32(S.bc[bs][1][0]), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < NST / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                    if (leader) umma_ss(tb + kColCB, desc_adv(a0, off), desc_adv(b0, off), id_cb, kk > 0);
                }
                if (leader) umma_commit(&Bb.cb_full);
                if (kYoOnState && leader) {
                    // CB is this issuer's only use of B and C
                    umma_commit(&Bb.bc_empty[0]);
                    if (kSplitBC) umma_commit(&Bb.bc_empty[1]);
                }
                SSD_TRACE_EV(2, c);
                return true;
            };
            // With two B/C stages the next block's CB is issued early (below); with one
            // stage its operands only arrive after this block is released, so it waits.
            if (kSt > 1 && nblk > 0) ok = issue_cb(0);
            for (int c = 0; c < nblk && ok; ++c) {
                const int bs = c % kSt;
                const uint32_t sC = smem_u32(S.bc[bs][0][0]);
                if (kSt == 1) {
                    ok = issue_cb(c);
                    if (!ok) break;
                }
                for (int j = 0; j < KH && ok; ++j) {
                    const int u = c * KH + j, xs = u & 1;
                    // Pm buffer (barrier index) of this unit and the phase it completes
                    const int pi = kInPlace ? j : u % kPmB;
                    const int pph = kInPlace ? (c & 1) : ((u / kPmB) & 1);
                    // Yo = C Hbf^T (issued by the state issuer when kYoOnState)
                    if (!kYoOnState) {
                        ok = mbar_wait<kInlW>(&Bb.hb_full, u & 1, abort);
                        SSD_TRACE_EV(14, u);
                        ok = ok && (u == 0 || mbar_wait<kInlW>(&Bb.yo_empty, (u - 1) & 1, abort));
                        SSD_TRACE_EV(17, u);
                        if (!ok) break;
                        tc_fence_after();
                        const uint64_t a0 = sdesc_sw128(sC, 16, 1024), b0 = sdesc_sw128(smem_u32(S.hbf), 16384, 1024);
#pragma unroll
                        for (int kk = 0; kk < NST / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                            if (leader) umma_ss(tb + kColYo, desc_adv(a0, off), desc_adv(b0, kk * 2048), id_y, kk > 0);
                        }
                        if (leader) umma_commit(&Bb.hb_empty);
                        SSD_TRACE_EV(3, u);
                    }
                    // the next block's CB runs while the mask warps finish this block's last head
                    if (kSt > 1 && j == KH - 1 && c + 1 < nblk) {
                        ok = issue_cb(c + 1);
                        if (!ok) break;
                    }
                    // Yd = Pm X, once the accumulator is free: the previous Yd read, or (shared
                    // with Yo) this unit's Yo read
                    ok = mbar_wait<kInlW>(&Bb.pm_full[pi], pph, abort) &&
                         mbar_wait<kInlW>(&Bb.x_full[xs], (u >> 1) & 1, abort) &&
                         (kSharedY ? mbar_wait<kInlW>(&Bb.yo_empty, u & 1, abort)
                                   : (u == 0 || mbar_wait<kInlW>(&Bb.yd_empty, (u - 1) & 1, abort)));
                    SSD_TRACE_EV(16, u);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t x0 = sdesc_sw128(smem_u32(S.x[xs]), 16384, 1024);
                    const bool ip = kInPlace && j == 1;
                    const uint32_t pm = ip ? tb + kColCB : tb + kColPm + 64 * pi;
#pragma unroll
                    for (int kk = 0; kk < kQ / 16; ++kk) {
                        const uint32_t acol = pm + kk * 8 + (ip && kk >= 4 ? 32u : 0u);
                        if (leader) umma_ts(tb + kColYd, acol, desc_adv(x0, kk * 2048), id_y, kk > 0);
                    }
                    if (leader) umma_commit(&Bb.pm_empty[pi]);
                    if (leader) umma_commit(&Bb.y_full);
                    if (leader) umma_commit(&Bb.x_empty[xs]);
                    SSD_TRACE_EV(5, u);
                }
                if (!kYoOnState && leader) umma_commit(&Bb.bc_empty[bs]);
            }
            // every UMMA issued so far has completed before TMEM is released
            if (leader) umma_commit(&Bb.drain_o);
            mbar_wait<kInlW>(&Bb.drain_o, 0, abort, 200000000ull);
        }
    } else if ((warp >= 4 && warp < 8) || warp == 10 || warp == 11) {
        // ------------------------------------------------------------- mask
        // Pm = CB o exp(cs_l - cs_s) delta_s (causal) + D on the diagonal, as
        // bf16 pairs in TMEM.  Warps 4-7: columns 0..63 for row quarters 0-3;
        // warps 10-11: columns 64..127 for row quarters 2-3 (quarters 0-1 are
        // zero there, written once by warps 8-9).
        if (!STATE_ONLY) {
            const int half = warp >= 8 ? 1 : 0;
            const int l = q * 32 + lane;               // row of this thread
            const int s_begin = half * 64;
            const int s_hi = min(s_begin + 64, q * 32 + 32);
            const int npairs = s_hi > s_begin ? (s_hi - s_begin + 31) / 32 : 0;
            float Dreg[KH];
#pragma unroll
            for (int j = 0; j < KH; ++j) Dreg[j] = prm.D ? prm.D[it.h0 + j] : 0.0f;
            bool ok = true;
            for (int c = 0; c < nblk && ok; ++c) {
                ok = mbar_wait<kInlW>(&Bb.cb_full, c & 1, abort);
                if (!ok) break;
                tc_fence_after();
                for (int j = 0; j < KH; ++j) {
                    const int u = c * KH + j, slot = u % kCsd;
                    const bool ip = kInPlace && j == 1;    // written over the CB columns just read
                    const int pi = kInPlace ? j : u % kPmB;
                    ok = mbar_wait<kInlW>(&Bb.cs_full[slot], (u / kCsd) & 1, abort);
                    if (kInPlace)
                        ok = ok && (ip || c == 0 || mbar_wait<kInlW>(&Bb.pm_empty[0], (c - 1) & 1, abort));
                    else
                        ok = ok && (u < kPmB || mbar_wait<kInlW>(&Bb.pm_empty[pi], ((u / kPmB) + 1) & 1, abort));
                    if (!ok) break;
                    tc_fence_after();
                    if (warp == 4 && lane == 0) SSD_TRACE_EV(7, u);
                    if (warp == 7 && lane == 0) SSD_TRACE_EV(18, u);
                    const float rowc = S.cs2[slot][l];
                    float Dh = Dreg[0];
#pragma unroll
                    for (int jj = 1; jj < KH; ++jj)
                        if (j == jj) Dh = Dreg[jj];
                    const uint32_t pm_col =
                        ip ? tb + lane_base + kColCB + half * 64 : tb + lane_base + kColPm + 64 * pi + half * 32;
                    const bool exact = S.exact[slot] != 0;
#pragma unroll 1
                    for (int pair = 0; pair < 2; ++pair) {      // 32 columns -> 16 TMEM columns
                        if (pair < npairs) {                    // warp-uniform
                            const int s0 = s_begin + pair * 32;
                            uint32_t r[32];
                            tmem_ld16(tb + lane_base + kColCB + s0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
                            tmem_ld16(tb + lane_base + kColCB + s0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
                            float cf[32];                       // column factors
                            const float R0 = S.cs2[slot][s0], R1 = S.cs2[slot][s0 + 16];
                            if (!exact) {
                                const float4 *uu = reinterpret_cast<const float4 *>(&S.u[slot][s0]);
#pragma unroll
                                for (int i4 = 0; i4 < 8; ++i4) {
                                    const float4 v4 = uu[i4];
                                    cf[4 * i4] = v4.x; cf[4 * i4 + 1] = v4.y;
                                    cf[4 * i4 + 2] = v4.z; cf[4 * i4 + 3] = v4.w;
                                }
                            }
                            tmem_ld_wait();
                            if (warp == 7 && lane == 0) SSD_TRACE_EV(19 + pair, u);
                            if (j == KH - 1 && pair == npairs - 1) {
                                tc_fence_before();
                                __syncwarp();
                                if (lane == 0) mbar_arrive(&Bb.cb_empty);
                            }
                            float m[32];
                            if (!exact) {
                                // exp2(cs2_l - cs2_s) delta_s = exp2(cs2_l - R) * [exp2(R - cs2_s) delta_s]:
                                // CB times the column factor, then the row factor of each 16-column chunk
                                const float v0 = ex2_approx(fminf(rowc - R0, 0.0f)), v1 = ex2_approx(fminf(rowc - R1, 0.0f));
#pragma unroll
                                for (int i = 0; i < 32; i += 2)
                                    mul_f32x2(m[i], m[i + 1], __uint_as_float(r[i]), __uint_as_float(r[i + 1]), cf[i],
                                              cf[i + 1]);
#pragma unroll
                                for (int i = 0; i < 32; i += 2) {
                                    const float v = i < 16 ? v0 : v1;
                                    mul_f32x2(m[i], m[i + 1], m[i], m[i + 1], v, v);
                                }
                            } else {
                                const float4 *cc = reinterpret_cast<const float4 *>(&S.cs2[slot][s0]);
                                const float4 *dd = reinterpret_cast<const float4 *>(&S.dl[slot][s0]);
#pragma unroll
                                for (int i4 = 0; i4 < 8; ++i4) {
                                    const float4 c4 = cc[i4], d4 = dd[i4];
                                    m[4 * i4 + 0] = __uint_as_float(r[4 * i4 + 0]) * (ex2_approx(fminf(rowc - c4.x, 0.0f)) * d4.x);
                                    m[4 * i4 + 1] = __uint_as_float(r[4 * i4 + 1]) * (ex2_approx(fminf(rowc - c4.y, 0.0f)) * d4.y);
                                    m[4 * i4 + 2] = __uint_as_float(r[4 * i4 + 2]) * (ex2_approx(fminf(rowc - c4.z, 0.0f)) * d4.z);
                                    m[4 * i4 + 3] = __uint_as_float(r[4 * i4 + 3]) * (ex2_approx(fminf(rowc - c4.w, 0.0f)) * d4.w);
                                }
                            }
                            // pairs are 32-aligned like the warp's rows: only the pair holding the
                            // warp's diagonal block needs the causal edge (s > l is zero, s == l gains D)
                            if (s0 + 31 >= q * 32) {            // warp-uniform
#pragma unroll
                                for (int i = 0; i < 32; ++i) {
                                    const int sa = s0 + i;
                                    m[i] = sa < l ? m[i] : (sa == l ? m[i] + Dh : 0.0f);
                                }
                            }
                            uint32_t packed[16];
#pragma unroll
                            for (int i2 = 0; i2 < 16; ++i2) packed[i2] = pack_bf16x2(m[2 * i2], m[2 * i2 + 1]);
                            tmem_st16(pm_col + pair * 16, packed);
                        } else {                                // above the diagonal for every row
                            uint32_t zeros[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) zeros[i] = 0u;
                            tmem_st16(pm_col + pair * 16, zeros);
                        }
                        if (warp == 7 && lane == 0) SSD_TRACE_EV(21 + pair, u);
                    }
                    if (j == KH - 1 && npairs == 0) {           // rows with no work still release CB
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&Bb.cb_empty);
                    }
                    if (ip && q < 2) {
                        // rows 0..63: K steps 4-7 (columns 64-95 in place) lie above the diagonal; nothing
                        // else touches these columns of these rows, which the CB UMMA filled
                        uint32_t zeros[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) zeros[i] = 0u;
                        tmem_st16(tb + lane_base + kColCB + 64, zeros);
                        tmem_st16(tb + lane_base + kColCB + 80, zeros);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&Bb.pm_full[pi]);
                        mbar_arrive(&Bb.cs_empty[slot]);
                        if (warp == 4) SSD_TRACE_EV(8, u);
                    }
                }
            }
        }
    } else if (warp == 8 || warp == 9) {
        // --------------------------------------------------- w o X (state input)
        if (!STATE_ONLY) {
            // the causal mask's columns 64..127 are zero for rows 0..63, in both Pm buffers
            uint32_t zeros[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) zeros[i] = 0u;
#pragma unroll
            for (int pi = 0; pi < kPmB; ++pi)
#pragma unroll
                for (int pair = 0; pair < 2; ++pair) tmem_st16(tb + lane_base + kColPm + 64 * pi + 32 + 16 * pair, zeros);
            tmem_st_wait();
            tc_fence_before();
        }
        bool ok = true;
        const int r0 = (warp - 8) * 64 + lane;          // rows r0 and r0 + 32
        for (int u = 0; u < nunits && ok; ++u) {
            const int slot = u % kCsd, xs = u % kXR, wi = u % kXwR;
            ok = mbar_wait<kInlW>(&Bb.cs_full[slot], (u / kCsd) & 1, abort) &&
                 mbar_wait<kInlW>(&x_full_b[xs], (u / kXR) & 1, abort) &&
                 (STATE_ONLY || u < kXwR || mbar_wait<kInlW>(&Bb.xw_empty[wi], ((u / kXwR) + 1) & 1, abort));
            if (!ok) break;
            if (warp == 8 && lane == 0) SSD_TRACE_EV(25, u);
            {
                // all 16 loads in flight before any math or store.  Step ch of lane i touches the
                // 16-byte chunk ch ^ (i & 7) of its row: the 8 lanes of each shared-memory phase
                // then cover 8 different bank groups (the same chunk of 8 rows would be 8-way
                // conflicted); each chunk is written back to where it was read.
                const uint32_t rot = (uint32_t)(lane & 7) * 16u;
                uint4 v[2][8];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch)
                        v[rr][ch] = *reinterpret_cast<const uint4 *>(x_tile(xs) + (r0 + 32 * rr) * 128 + ((ch * 16) ^ rot));
                __syncwarp();
                if (!STATE_ONLY && lane == 0) mbar_arrive(&Bb.x_empty[xs]);   // X no longer read by this warp
                // w o X: into its ring, or in place (this thread's own rows only)
                uint8_t *const dst_tile = STATE_ONLY ? x_tile(xs) : xw_tile(wi);
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int t = r0 + 32 * rr;
                    const __nv_bfloat162 ws2 = __float2bfloat162_rn(S.w[slot][t]);
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        __nv_bfloat162 *pv = reinterpret_cast<__nv_bfloat162 *>(&v[rr][ch]);
#pragma unroll
                        for (int i = 0; i < 4; ++i) pv[i] = __hmul2(pv[i], ws2);
                        *reinterpret_cast<uint4 *>(dst_tile + t * 128 + ((ch * 16) ^ rot)) = v[rr][ch];
                    }
                }
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(STATE_ONLY ? &Bb.xws_full[xs] : &Bb.xw_full[wi]);
                mbar_arrive(&Bb.cs_empty[slot]);
                if (warp == 8) SSD_TRACE_EV(11, u);
            }
        }
    } else if (warp >= 12) {
        // --------------------------------------------------- state + epilogue
        const int t = q * 32 + lane;                   // TMEM lane: state row n / output row l
        const int N = NST;
        const size_t PN = (size_t)kP * N;
        // initial state of every head: from the caller, from the segment scan, or zero.  Plain
        // loads: a segment state written by another CTA of this launch (the segmented walk) was
        // only ever read here through L2 (.cg) loads, so no stale line of it sits in L1
        for (int j = 0; j < KH; ++j) {
            const int h = it.h0 + j;
            // state-only mode measures each segment from a zero state
            const float *src = nullptr;
            if (!STATE_ONLY) {
                if (it.nseg > 1)
                    src = prm.segstate + (size_t)(srow + j) * PN;
                else if (prm.init)
                    src = prm.init + ((size_t)it.seq * prm.H + h) * PN;
            }
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
                const int n = kMT > 1 ? t + 128 * mt : t % N;   // N = 64: lanes 64..127 mirror 0..63
                // all 64 loads of the row in flight before the first tensor-memory store (the
                // stores are ordered after earlier loads, so a batch of 16 would wait 4 times)
                uint32_t r[kP];
#pragma unroll
                for (int p = 0; p < kP; ++p) r[p] = src ? __float_as_uint(src[(size_t)p * N + n]) : 0u;
#pragma unroll
                for (int p0 = 0; p0 < kP; p0 += 16)
                    tmem_st16(tb + lane_base + kColH + 64 * (j + KH * mt) + p0,
                              *reinterpret_cast<uint32_t(*)[16]>(&r[p0]));
            }
        }
        tmem_st_wait();
        if (kTmaY && lane == 0) tma_prefetch_desc(&mapY);
        bool ok = true;
        float ldec_sum[KH];
#pragma unroll
        for (int j = 0; j < KH; ++j) ldec_sum[j] = 0.0f;

        // epilogue of unit v: y = Yd + exp(cs_l) Yo for this thread's row
        auto epilogue = [&](int v) -> bool {
            const int c = v / KH, j = v % KH, slot = v % kCsd;
            // Yd and Yo in one accumulator: Yo is read first, then Pm X may write Yd
            if (!kSharedY && !mbar_wait<kInlW>(&Bb.y_full, v & 1, abort)) return false;
            if (kYoOnState && !mbar_wait<kInlW>(&Bb.yo_full, v & 1, abort)) return false;
            tc_fence_after();
            if (warp == 12 && lane == 0) SSD_TRACE_EV(12, v);
            const int valid = min(kQ, it.len - c * kQ);
            const int tok = it.tok0 + c * kQ + t;
            const float el = S.e[slot][t];
            // Yo first (scaled into registers), then Yo goes back to the MMA warp
            uint32_t yo[64];
#pragma unroll
            for (int p0 = 0; p0 < kP; p0 += 16)
                tmem_ld16(tb + lane_base + kColYo + p0, *reinterpret_cast<uint32_t(*)[16]>(&yo[p0]));
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&Bb.yo_empty);
            if (warp == 12 && lane == 0) SSD_TRACE_EV(26, v);
            if (kSharedY) {
                if (!mbar_wait<kInlW>(&Bb.y_full, v & 1, abort)) return false;
                tc_fence_after();
                if (warp == 12 && lane == 0) SSD_TRACE_EV(17, v);
            }
            __nv_bfloat16 *dst = prm.y + ((size_t)tok * prm.H + it.h0 + j) * kP;
            const int wi = v % kXwD;
            uint8_t *stage = S.xw[wi] + q * 32 * 128;     // this warp's 32 rows, 128-byte swizzled
            const bool via_tma = kTmaY && valid == kQ;
            // the slot's w o X tile is free once the state UMMA of unit v has completed
            if (kTmaY && !mbar_wait<kInlW>(&Bb.xw_free[wi], (v / kXwD) & 1, abort)) return false;
            if (GN) {
                // Mamba-2 block output (Sec. 7.1): g = y * silu(z), staged as bf16 while the
                // statistics accumulate (shifted by the row's first g), then normalised over the
                // head's 64 channels with the per-channel weight and bias
                const bool row_ok = via_tma || t < valid;
                const __nv_bfloat16 *zrow = gnp.z + ((size_t)tok * prm.H + it.h0 + j) * kP;
                float sh = 0.0f, s1 = 0.0f, s2 = 0.0f;
#pragma unroll
                for (int h0 = 0; h0 < kP; h0 += 32) {
                    uint32_t yd[32];
                    tmem_ld16(tb + lane_base + kColYd + h0, *reinterpret_cast<uint32_t(*)[16]>(&yd[0]));
                    tmem_ld16(tb + lane_base + kColYd + h0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&yd[16]));
                    tmem_ld_wait();
                    if (h0 == kP - 32) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&Bb.yd_empty);
                    }
                    if (row_ok) {
#pragma unroll
                        for (int q8 = 0; q8 < 32; q8 += 8) {
                            const uint4 zz = *reinterpret_cast<const uint4 *>(zrow + h0 + q8);
                            const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
                            uint32_t pk[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int pp = q8 + 2 * i;
                                float ya, yb;
                                fma_f32x2(ya, yb, el, el, __uint_as_float(yo[h0 + pp]), __uint_as_float(yo[h0 + pp + 1]),
                                          __uint_as_float(yd[pp]), __uint_as_float(yd[pp + 1]));
                                const float2 zf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&zw[i]));
                                const float ga = ya * __fdividef(zf.x, 1.0f + __expf(-zf.x));
                                const float gb = yb * __fdividef(zf.y, 1.0f + __expf(-zf.y));
                                if (h0 == 0 && pp == 0) sh = ga;
                                const float da = ga - sh, db = gb - sh;
                                s1 += da + db;
                                s2 = fmaf(da, da, fmaf(db, db, s2));
                                pk[i] = pack_bf16x2(ga, gb);
                            }
                            const uint4 v4 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                            if (via_tma)
                                *reinterpret_cast<uint4 *>(stage + sw128_offset(lane, h0 + q8)) = v4;
                            else
                                *reinterpret_cast<uint4 *>(dst + h0 + q8) = v4;
                        }
                    }
                }
                if (row_ok) {
                    const float mo = s1 * (1.0f / kP);
                    const float rstd = rsqrtf(fmaxf(s2 * (1.0f / kP) - mo * mo, 0.0f) + gnp.eps);
                    const float mean = sh + mo;
                    const float *wrow = gnp.w + (size_t)(it.h0 + j) * kP;
                    const float *brow = gnp.b ? gnp.b + (size_t)(it.h0 + j) * kP : nullptr;
#pragma unroll
                    for (int c8 = 0; c8 < kP; c8 += 8) {
                        uint4 *slot_ptr = via_tma ? reinterpret_cast<uint4 *>(stage + sw128_offset(lane, c8))
                                                  : reinterpret_cast<uint4 *>(dst + c8);
                        uint4 v4 = *slot_ptr;
                        uint32_t *vw = reinterpret_cast<uint32_t *>(&v4);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&vw[i]));
                            const int cc = c8 + 2 * i;
                            float oa = (g2.x - mean) * rstd * wrow[cc], ob = (g2.y - mean) * rstd * wrow[cc + 1];
                            if (brow) {
                                oa += brow[cc];
                                ob += brow[cc + 1];
                            }
                            vw[i] = pack_bf16x2(oa, ob);
                        }
                        *slot_ptr = v4;
                    }
                }
            } else {
#pragma unroll
            for (int h0 = 0; h0 < kP; h0 += 32) {
                uint32_t yd[32];
                tmem_ld16(tb + lane_base + kColYd + h0, *reinterpret_cast<uint32_t(*)[16]>(&yd[0]));
                tmem_ld16(tb + lane_base + kColYd + h0 + 16, *reinterpret_cast<uint32_t(*)[16]>(&yd[16]));
                tmem_ld_wait();
                if (h0 == kP - 32) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&Bb.yd_empty);
                }
                if (via_tma || t < valid) {
#pragma unroll
                    for (int q8 = 0; q8 < 32; q8 += 8) {
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int pp = q8 + 2 * i;
                            float ya, yb;
                            fma_f32x2(ya, yb, el, el, __uint_as_float(yo[h0 + pp]), __uint_as_float(yo[h0 + pp + 1]),
                                      __uint_as_float(yd[pp]), __uint_as_float(yd[pp + 1]));
                            pk[i] = pack_bf16x2(ya, yb);
                        }
                        const uint4 v4 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        if (via_tma)
                            *reinterpret_cast<uint4 *>(stage + sw128_offset(lane, h0 + q8)) = v4;
                        else
                            *reinterpret_cast<uint4 *>(dst + h0 + q8) = v4;
                    }
                }
            }
            }
            if (via_tma) fence_async_smem();
            __syncwarp();
            if (warp == 12 && lane == 0) SSD_TRACE_EV(23, v);
            if (lane == 0) {
                if (via_tma) {
                    tma_store_2d(&mapY, stage, (it.h0 + j) * kP, it.tok0 + c * kQ + q * 32);
                    bulk_commit();
                    bulk_wait_read_all();
                }
                if (warp == 12) SSD_TRACE_EV(24, v);
                if (kTmaY) mbar_arrive(&Bb.xw_empty[wi]);
                mbar_arrive(&Bb.cs_empty[slot]);
            }
            if (warp == 12 && lane == 0) SSD_TRACE_EV(13, v);
            return true;
        };

        for (int u = 0; u <= nunits && ok; ++u) {
            if (u == nunits) {
                if (!STATE_ONLY && u >= 1) ok = epilogue(u - 1);
                break;
            }
            const int c = u / KH, j = u % KH, slot = u % kCsd;
            if (STATE_ONLY) {
                // backward walk: the state is one accumulation from zero, never rescaled
                if (c == 0) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&Bb.hs_full[j]);   // the zeroed state is in place
                }
                ok = mbar_wait<kInlW>(&Bb.cs_full[slot], (u / kCsd) & 1, abort);
                if (!ok) break;
                const float ld = S.ldec[slot];
#pragma unroll
                for (int jj = 0; jj < KH; ++jj)
                    if (j == jj) ldec_sum[jj] += ld;
                __syncwarp();
                if (lane == 0) mbar_arrive(&Bb.cs_empty[slot]);
                continue;
            }
            ok = mbar_wait<kInlW>(&Bb.cs_full[slot], (u / kCsd) & 1, abort) &&
                 (c == 0 || mbar_wait<kInlW>(&Bb.h_ready[j], (c - 1) & 1, abort));
            if (!ok) break;
            if (!STATE_ONLY) ok = (u == 0 || mbar_wait<kInlW>(&Bb.hb_empty, (u - 1) & 1, abort));
            if (!ok) break;
            tc_fence_after();
            if (warp == 12 && lane == 0) SSD_TRACE_EV(9, u);
            const float alpha = S.alpha[slot];
            float ld = S.ldec[slot];
#pragma unroll
            for (int jj = 0; jj < KH; ++jj)
                if (j == jj) ldec_sum[jj] += ld;
            // H pass: Hbf = bf16(H) (rows n, MN-major), H <- alpha * H in place
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
                const uint32_t hcol = tb + lane_base + kColH + 64 * (j + KH * mt);
                const int n = t + 128 * mt;
                uint32_t r[64];
#pragma unroll
                for (int p0 = 0; p0 < kP; p0 += 16)
                    tmem_ld16(hcol + p0, *reinterpret_cast<uint32_t(*)[16]>(&r[p0]));
                tmem_ld_wait();
#pragma unroll
                for (int p0 = 0; p0 < kP; p0 += 16) {
                    if (!STATE_ONLY && n < N) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pk[i] = pack_bf16x2(__uint_as_float(r[p0 + 2 * i]), __uint_as_float(r[p0 + 2 * i + 1]));
                        *reinterpret_cast<uint4 *>(S.hbf + sw128_offset(n, p0)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        *reinterpret_cast<uint4 *>(S.hbf + sw128_offset(n, p0 + 8)) =
                            make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        float ha, hb;
                        mul_f32x2(ha, hb, alpha, alpha, __uint_as_float(r[p0 + i]), __uint_as_float(r[p0 + i + 1]));
                        r[p0 + i] = __float_as_uint(ha);
                        r[p0 + i + 1] = __float_as_uint(hb);
                    }
                    tmem_st16(hcol + p0, *reinterpret_cast<uint32_t(*)[16]>(&r[p0]));
                }
            }
            tmem_st_wait();
            if (!STATE_ONLY) fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (!STATE_ONLY) mbar_arrive(&Bb.hb_full);
                mbar_arrive(&Bb.hs_full[j]);
                if (STATE_ONLY) mbar_arrive(&Bb.cs_empty[slot]);
            }
            if (warp == 12 && lane == 0) SSD_TRACE_EV(10, u);
            if (!STATE_ONLY && u >= 1) ok = epilogue(u - 1);
        }
        // end of the segment: the state after the last token.  The full walk has waited for every
        // earlier phase of h_ready[j], so the last one is the next to complete; the state-only walk
        // has not (a parity wait more than one phase ahead would pass at once), so it waits for the
        // state issuer's drain commit instead, which completes once, after the last state UMMA
        if (ok) {
            for (int j = 0; j < KH; ++j) {
                ok = STATE_ONLY ? mbar_wait<kInlW>(&Bb.drain_s, 0, abort)
                                : mbar_wait<kInlW>(&Bb.h_ready[j], (nblk - 1) & 1, abort);
                if (!ok) break;
                tc_fence_after();
                const int h = it.h0 + j;
                float *dst = nullptr;
                if (STATE_ONLY)
                    dst = prm.segstate + (size_t)(srow + j) * PN;
                else if (it.seg == it.nseg - 1 && prm.final_states)
                    dst = prm.final_states + ((size_t)it.seq * prm.H + h) * PN;
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    const uint32_t hcol = tb + lane_base + kColH + 64 * (j + KH * mt);
                    const int n = t + 128 * mt;
#pragma unroll
                    for (int p0 = 0; p0 < kP; p0 += 16) {
                        uint32_t r[16];
                        tmem_ld16(hcol + p0, r);
                        tmem_ld_wait();
                        if (dst && n < N) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) dst[(size_t)(p0 + i) * N + n] = __uint_as_float(r[i]);
                        }
                    }
                }
                if (STATE_ONLY && t == 0)
                    prm.seglogdec[srow + j] = ldec_sum[j];
            }
        }
        if (kTmaY && lane == 0) bulk_wait_all();       // this warp's y stores have landed
    }

}

// Shared-memory carve-out and the 512-column TMEM allocation of a walk CTA;
// every kernel below starts with it and ends with walk_teardown.
template <int NST>
__device__ __forceinline__ TcSmem<NST> &walk_smem()
{
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment (128-byte swizzle atoms) computed as an offset from the
    // shared array itself, so every access below stays a shared-memory access
    const uint32_t smem_pad = ((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw);
    return *reinterpret_cast<TcSmem<NST> *>(smem_raw + smem_pad);
}

template <int NST>
__device__ __forceinline__ uint32_t walk_setup(TcSmem<NST> &S)
{
    if (threadIdx.x == 0) S.abort = 0;
    if (threadIdx.x / 32 == 3) {
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    __syncthreads();
    tc_fence_after();
    return S.tmem_base;
}

template <int NST>
__device__ __forceinline__ void walk_teardown(TcSmem<NST> &S, uint32_t tb, int *status)
{
    __syncthreads();
    if (S.abort && threadIdx.x == 0) record_timeout(status);
    if (threadIdx.x / 32 == 3) {
        tc_fence_after();
        tmem_dealloc(tb, 512);
    }
}

template <int NST, int KH, bool STATE_ONLY, bool GN = false>
__global__ void __launch_bounds__(kThreadsTc, 1)
ssd_tc_walk(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
            const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapY,
            const __grid_constant__ TcParams prm, const __grid_constant__ GnParams gnp)
{
    TcSmem<NST> &S = walk_smem<NST>();
    const int item_idx = blockIdx.x;
    TcItem it;
    if (prm.items) {
        if (item_idx >= *prm.count) return;
        it = prm.items[item_idx];
    } else {
        if (item_idx >= prm.n_items) return;
        const int g0 = prm.direct_base + item_idx * KH;
        const int row = g0 / prm.H;
        it.seq = row;
        it.tok0 = row * prm.seqlen;
        it.len = prm.seqlen;
        it.gseg = row;
        it.seg = 0;
        it.nseg = 1;
        it.h0 = g0 - row * prm.H;
        it.pad = 0;
    }
    // only non-final segments need end states (every sequence's, for a summary)
    if (STATE_ONLY && !prm.summary && it.seg >= it.nseg - 1) return;
    // a launch queued behind this one as a programmatic dependent (the one-head items left
    // after whole waves, which read nothing this launch writes) may start as SMs free up
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const uint32_t tb = walk_setup(S);
    const int srow = (prm.summary ? it.seq : it.gseg) * prm.H + it.h0;
    walk_body<NST, KH, STATE_ONLY, GN>(mapX, mapB, mapC, mapY, prm, gnp, S, S.bar[0], tb, it, item_idx, srow);
    walk_teardown(S, tb, prm.status);
    // launched as a programmatic dependent: do not finish before the launch ahead of this one,
    // so that work queued after this launch sees both complete (immediate otherwise)
    if (threadIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Wait (bounded, 2 s) until the counter at p reaches target; acquire ordering.
__device__ __noinline__ bool counter_wait(const int *p, int target, volatile int *abort)
{
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
        if (v >= target) return true;
        if ((it & 63u) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > 2000000000ull) {
                *abort = 1;
                return false;
            }
        }
        __nanosleep(100);
    }
}

// Segments of equal-length rows in one launch (Sec. 8.2, state passing
// between pieces of a sequence).  CTA (pair, seg) of a (row, head block) pair
// cut into fp.nseg segments: (1) a non-final segment measures its end state
// from zero (the state-only walk) and publishes it; (2) once every non-final
// segment of the pair has published, the pair's nseg CTAs each chain one slice
// of the states through the segments, replacing segment k's state by the state
// entering segment k (the caller's initial state for k = 0); (3) once every
// slice is chained, every CTA runs the full walk of its segment from its
// entering state.  The waits between CTAs need every CTA of the pair resident
// at once: the grid is at most one CTA per SM, launched cooperatively, and
// every wait is bounded.
struct FuseParams {
    int *ctr;        // [pairs][2] arrival counters, zero before the launch
    int pair_base;   // flattened (row, head block) index of the launch's first pair
    int nseg;        // segments per pair (>= 2)
    int seg_len;     // tokens of every segment but the last (the last takes the rest)
};

template <int NST, int KH, bool GN = false>
__global__ void __launch_bounds__(kThreadsTc, 1)
ssd_tc_fused(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapB,
             const __grid_constant__ CUtensorMap mapC, const __grid_constant__ CUtensorMap mapY,
             const __grid_constant__ TcParams prm, const __grid_constant__ GnParams gnp, const FuseParams fp)
{
    TcSmem<NST> &S = walk_smem<NST>();
    const int tid = threadIdx.x;
    const int pl = blockIdx.x / fp.nseg, seg = blockIdx.x - pl * fp.nseg;
    const int n_hb = prm.H / KH;
    const int pair = fp.pair_base + pl, row = pair / n_hb;
    TcItem it;
    it.seq = row;
    it.tok0 = row * prm.seqlen + seg * fp.seg_len;
    it.len = seg < fp.nseg - 1 ? fp.seg_len : prm.seqlen - (fp.nseg - 1) * fp.seg_len;
    it.gseg = pl * fp.nseg + seg;
    it.seg = seg;
    it.nseg = fp.nseg;
    it.h0 = (pair - row * n_hb) * KH;
    it.pad = 0;
    // segment states of the launch: [pair][segment][KH heads][P x N], decays [pair][segment][KH]
    const int srow = it.gseg * KH;
    const uint32_t tb = walk_setup(S);
    if (seg < fp.nseg - 1)
        walk_body<NST, KH, true, false>(mapX, mapB, mapC, mapY, prm, gnp, S, S.bar[0], tb, it, blockIdx.x, srow);
    tc_fence_before();      // the first walk's tensor-memory accesses come before the second walk's
    __syncthreads();

    constexpr int PN = kP * NST;
    int *const ctr = fp.ctr + 2 * pl;
    if (tid == 0 && !S.abort) {
        if (seg < fp.nseg - 1) {
            __threadfence();
            atomicAdd(ctr, 1);
        }
        counter_wait(ctr, fp.nseg - 1, &S.abort);
        __threadfence();
    }
    __syncthreads();
    if (!S.abort) {
        // this CTA's slice of the pair's KH x P x N state elements, in whole 128-byte lines
        // (float4 units), chained through the segments in place
        constexpr int kTot4 = KH * PN / 4;
        const int per4 = ((kTot4 + fp.nseg - 1) / fp.nseg + 7) / 8 * 8;
        const int b4 = seg * per4, e4 = min(kTot4, b4 + per4);
        const int srow0 = pl * fp.nseg * KH;
        for (int i4 = b4 + tid; i4 < e4; i4 += kThreadsTc) {
            const int e = i4 * 4, j = e / PN, idx = e - j * PN;
            float4 hv = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (prm.init) {
                // the caller's buffer: element loads (no alignment beyond 4 bytes assumed)
                const float *ip = prm.init + ((size_t)row * prm.H + it.h0 + j) * PN + idx;
                hv = make_float4(__ldcg(ip), __ldcg(ip + 1), __ldcg(ip + 2), __ldcg(ip + 3));
            }
            constexpr int kGroup = 8;
            for (int k0 = 0; k0 < fp.nseg; k0 += kGroup) {
                float4 sv[kGroup];
                float dk[kGroup];
#pragma unroll
                for (int i = 0; i < kGroup; ++i) {
                    const int k = k0 + i;
                    const bool has = k < fp.nseg - 1;
                    const int sr = srow0 + k * KH + j;
                    sv[i] = has ? __ldcg(reinterpret_cast<const float4 *>(prm.segstate + (size_t)sr * PN + idx))
                                : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    dk[i] = has ? __expf(__ldcg(prm.seglogdec + sr)) : 0.0f;
                }
#pragma unroll
                for (int i = 0; i < kGroup; ++i) {
                    const int k = k0 + i;
                    if (k < fp.nseg) {
                        const int sr = srow0 + k * KH + j;
                        __stcg(reinterpret_cast<float4 *>(prm.segstate + (size_t)sr * PN + idx), hv);
                        hv.x = fmaf(dk[i], hv.x, sv[i].x);
                        hv.y = fmaf(dk[i], hv.y, sv[i].y);
                        hv.z = fmaf(dk[i], hv.z, sv[i].z);
                        hv.w = fmaf(dk[i], hv.w, sv[i].w);
                    }
                }
            }
        }
    }
    __syncthreads();
    if (tid == 0 && !S.abort) {
        __threadfence();
        atomicAdd(ctr + 1, 1);
        counter_wait(ctr + 1, fp.nseg, &S.abort);
        __threadfence();
    }
    __syncthreads();
    tc_fence_after();
    if (!S.abort)
        walk_body<NST, KH, false, GN>(mapX, mapB, mapC, mapY, prm, gnp, S, S.bar[1], tb, it, blockIdx.x, srow);
    walk_teardown(S, tb, prm.status);
    // launched behind whole waves of the plain walk as a programmatic dependent: finish only
    // after that launch, so that work queued after this one sees both complete
    if (tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- planning
// Work items: (sequence, head block, segment), item index = global segment *
// n_hb + head block.  One block of 1024 threads: per chunk of 1024 sequences a
// block-wide scan places each sequence's segments, then every thread writes
// items (one per (segment, head block)); seqseg[s] = first global segment of a
// sequence cut into two or more segments (-1 otherwise) for the segment scan.
__global__ void __launch_bounds__(1024)
tc_plan_kernel(const int32_t *__restrict__ cu_seqlens, int nseq, int seqlen, int seg_len, int n_hb, int KH,
               TcItem *items, int *count, int max_items, int *status, const float *__restrict__ init,
               float *__restrict__ final_states, int H, int PN, int *seqseg)
{
    __shared__ int s_bad, s_carry;
    __shared__ int s_warp[32];
    __shared__ int s_incl[1024], s_tok0[1024], s_len[1024];
    const int tid = threadIdx.x;
    if (tid == 0) {
        *status = 0;
        s_bad = 0;
        s_carry = 0;
    }
    __syncthreads();
    if (cu_seqlens) {
        for (int i = tid; i < nseq; i += 1024) {
            const int a = cu_seqlens[i], b = cu_seqlens[i + 1];
            if (b < a || (i == 0 && a != 0) || (i == nseq - 1 && b != seqlen)) s_bad = 1;
        }
    }
    __syncthreads();
    if (s_bad) {
        // no work item and no segment chain: the later kernels of this call read
        // nothing from a previous call's tables
        if (tid == 0) {
            set_status(status, kDevBadSeqlens);
            *count = 0;
        }
        if (seqseg)
            for (int i = tid; i < nseq; i += 1024) seqseg[i] = -1;
        return;
    }
    for (int base = 0; base < nseq; base += 1024) {
        const int i = base + tid;
        const int cnt = min(1024, nseq - base);
        int tok0 = 0, len = 0, ns = 0;
        if (i < nseq) {
            tok0 = cu_seqlens ? cu_seqlens[i] : i * seqlen;
            len = cu_seqlens ? cu_seqlens[i + 1] - tok0 : seqlen;
            ns = (len + seg_len - 1) / seg_len;
        }
        int v = ns;
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, v, o);
            if ((tid & 31) >= o) v += t;
        }
        if ((tid & 31) == 31) s_warp[tid >> 5] = v;
        __syncthreads();
        if (tid < 32) {
            int w = s_warp[tid];
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, w, o);
                if (tid >= o) w += t;
            }
            s_warp[tid] = w;
        }
        __syncthreads();
        const int incl = v + ((tid >> 5) ? s_warp[(tid >> 5) - 1] : 0);   // segments up to i, in this chunk
        const int carry = s_carry;
        s_incl[tid] = incl;
        s_tok0[tid] = tok0;
        s_len[tid] = len;
        if (i < nseq && seqseg) seqseg[i] = ns >= 2 ? carry + incl - ns : -1;
        __syncthreads();
        const int chunk_segs = s_incl[cnt - 1];
        for (int idx = tid; idx < chunk_segs * n_hb; idx += 1024) {
            const int sl = idx / n_hb, hb = idx - sl * n_hb;
            // the sequence holding chunk segment sl: first k with incl[k] > sl
            int lo = 0, hi = cnt - 1;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (s_incl[mid] > sl) hi = mid; else lo = mid + 1;
            }
            const int first = lo ? s_incl[lo - 1] : 0;   // chunk segment where sequence lo starts
            const int segi = sl - first;
            const int gs = carry + sl;
            const int item = gs * n_hb + hb;
            if (item < max_items) {
                TcItem t;
                t.seq = base + lo;
                t.tok0 = s_tok0[lo] + segi * seg_len;
                t.len = min(seg_len, s_len[lo] - segi * seg_len);
                t.gseg = gs;
                t.seg = segi;
                t.nseg = s_incl[lo] - first;
                t.h0 = hb * KH;
                t.pad = 0;
                items[item] = t;
            }
        }
        // empty sequences: the final state is the initial state
        if (final_states) {
            for (int k2 = 0; k2 < cnt; ++k2) {
                if (s_len[k2] != 0) continue;
                const size_t o = (size_t)(base + k2) * H * PN;
                for (int e = tid; e < H * PN; e += 1024) final_states[o + e] = init ? init[o + e] : 0.0f;
            }
        }
        __syncthreads();
        if (tid == 0) s_carry = carry + chunk_segs;
        __syncthreads();
    }
    if (tid == 0) *count = min(s_carry * n_hb, max_items);
}

// Segment scan: entering state of every segment of every sequence,
// H_in(0) = initial state, H_in(k+1) = exp(ldec_k) H_in(k) + S_k; written in
// place over the pass-1 end states.
__global__ void __launch_bounds__(256)
tc_seg_scan_kernel(const TcItem *__restrict__ items, const int *__restrict__ seqseg, int n_hb, float *segstate,
                   const float *__restrict__ seglogdec, const float *__restrict__ init, int H, int PN,
                   const int *__restrict__ count, int max_segments)
{
    // grid: (sequences, H, ceil(PN / 256)); only sequences cut into two or more segments work
    const int gs = seqseg[blockIdx.x];
    // a plan the planner rejected (malformed cu_seqlens) has no items
    if (gs < 0 || gs >= max_segments || (long long)gs * n_hb >= *count) return;
    const TcItem it = items[(size_t)gs * n_hb];
    if (gs + it.nseg > max_segments) return;
    const int h = blockIdx.y;
    const int e = blockIdx.z * 256 + threadIdx.x;
    if (e >= PN) return;
    float hv = init ? init[((size_t)it.seq * H + h) * PN + e] : 0.0f;
    // segment k's slot holds the state measured over segment k from zero on entry and
    // the state entering segment k on exit; loads go out in groups so that the chain
    // waits on memory once per group, not once per segment
    constexpr int kGroup = 8;
    for (int k0 = 0; k0 < it.nseg; k0 += kGroup) {
        float sv[kGroup], dk[kGroup];
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            const int k = k0 + i;
            const bool has = k < it.nseg - 1;
            sv[i] = has ? segstate[((size_t)(gs + k) * H + h) * PN + e] : 0.0f;
            dk[i] = has ? __expf(seglogdec[(size_t)(gs + k) * H + h]) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < kGroup; ++i) {
            const int k = k0 + i;
            if (k < it.nseg) {
                segstate[((size_t)(gs + k) * H + h) * PN + e] = hv;
                hv = fmaf(dk[i], hv, sv[i]);
            }
        }
    }
}

// ------------------------------------------------------------------- host
// The driver's tensor-map encoder, looked up once (a function-local static is
// initialised exactly once even when several host threads call concurrently).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        return nullptr;
    }();
    return fn;
}

// 2-D bf16 view [rows][inner] with a {64, box_rows} box and 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint32_t box_rows = 128)
{
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcPlanShape {
    int KH, n_hb, seg_len, max_segments, max_items;
    bool segmented;
};

// The split of packed sequences is a pure function of the parameters, sized
// for the B200's 148 SMs.  The schedule of equal-length rows (uniform_plan)
// also takes min(148, SMs of the current device): its segmented launch needs
// every CTA resident at once.  So the workspace size is that of the device
// current when it is asked for; ssd_fwd recomputes it and rejects a smaller
// workspace.
constexpr int kPlanSMs = 148;

// Segment count (1 = no cut) with the smallest modelled makespan for `rows`
// equal rows of `nblk` 128-token blocks and `items_per_row` items per row, in
// block steps of one SM.  Pass 2 runs ceil(items * n / SMs) rounds of items of
// ceil(blocks / n) blocks; pass 1 (state only, about 0.65 of a pass-2 block)
// the same over n - 1 segments; each round costs about 1.5 blocks of fill and
// drain, the segment scan 2.
long long best_segment_count(long long items, long long nblk)
{
    const long long sms = kPlanSMs;
    long long best_n = 1;
    double best = 1e300;
    for (long long n = 1; n <= 64 && n <= nblk; ++n) {
        const long long bps = (nblk + n - 1) / n;
        const long long r2 = (items * n + sms - 1) / sms;
        const long long r1 = n > 1 ? (items * (n - 1) + sms - 1) / sms : 0;
        const double cost = (double)bps * ((double)r2 + 0.65 * (double)r1) + 1.5 * (double)(r1 + r2) +
                            (n > 1 ? 2.0 : 0.0);
        if (cost < best - 1e-9) {
            best = cost;
            best_n = n;
        }
    }
    return best_n;
}

TcPlanShape plan_shape(const ssd_fwd_params &p)
{
    TcPlanShape s;
    const int hpg = p.nheads / p.ngroups;
    // two heads per CTA share B/C tiles (at dstate 256 with one Yd/Yo accumulator)
    s.KH = hpg % 2 == 0 ? 2 : 1;
    s.n_hb = p.nheads / s.KH;
    const int nseq = p.num_seqs > 0 ? p.num_seqs : p.batch;
    const long long tokens = (long long)p.batch * p.seqlen;
    const long long items = (long long)nseq * s.n_hb;   // unsegmented work items
    long long seg;
    if (p.num_seqs > 0) {
        // packed: the lengths live on the device, so the model runs on rows of the
        // average length; when it asks for cuts, segments are bounded so that no
        // sequence dominates the makespan (about two items per SM, >= 1024 tokens)
        const long long avg_blk = (tokens / nseq + kQ - 1) / kQ;
        if (avg_blk < 1 || best_segment_count(items, avg_blk) == 1) {
            seg = tokens > 0 ? tokens : kQ;
        } else {
            const int target = 2 * kPlanSMs;
            seg = (tokens * s.n_hb + target - 1) / target;
            seg = seg < 1024 ? 1024 : seg;
        }
    } else {
        const long long nblk = (p.seqlen + kQ - 1) / kQ;
        const long long n = best_segment_count(items, nblk > 0 ? nblk : 1);
        seg = (nblk + n - 1) / n * kQ;
    }
    seg = (seg + kQ - 1) / kQ * kQ;
    if (seg < kQ) seg = kQ;
    s.seg_len = (int)seg;
    if (p.num_seqs > 0)
        s.max_segments = (int)((tokens + seg - 1) / seg) + nseq;
    else
        s.max_segments = p.batch * (int)((p.seqlen + seg - 1) / seg);
    s.max_items = s.max_segments * s.n_hb;
    s.segmented = s.seg_len < p.seqlen;
    return s;
}

template <int NST, int KH, bool SO, bool GN>
cudaError_t launch_walk(int grid, const CUtensorMap &mX, const CUtensorMap &mB, const CUtensorMap &mC,
                        const CUtensorMap &mY,
                        const TcParams &prm, cudaStream_t st, const GnParams &gnp = GnParams{}, bool overlap = false)
{
    const size_t smem = tc_smem_bytes<NST>();
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_walk<NST, KH, SO, GN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    if (!overlap) {
        ssd_tc_walk<NST, KH, SO, GN><<<grid, kThreadsTc, smem, st>>>(mX, mB, mC, mY, prm, gnp);
        return cudaGetLastError();
    }
    // programmatic dependent launch: may begin before the previous kernel on the stream has
    // finished; only for work that reads nothing that kernel writes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ssd_tc_walk<NST, KH, SO, GN>, mX, mB, mC, mY, prm, gnp);
}

template <int NST, bool SO, bool GN>
cudaError_t launch_walk_kh(int KH, int grid, const CUtensorMap &mX, const CUtensorMap &mB, const CUtensorMap &mC,
                           const CUtensorMap &mY,
                           const TcParams &prm, cudaStream_t st, const GnParams &gnp = GnParams{}, bool overlap = false)
{
    return KH == 2 ? launch_walk<NST, 2, SO, GN>(grid, mX, mB, mC, mY, prm, st, gnp, overlap)
                   : launch_walk<NST, 1, SO, GN>(grid, mX, mB, mC, mY, prm, st, gnp, overlap);
}

template <bool SO, bool GN = false>
cudaError_t launch_walk_any(int N, int KH, int grid, const CUtensorMap &mX, const CUtensorMap &mB,
                            const CUtensorMap &mC, const CUtensorMap &mY, const TcParams &prm, cudaStream_t st,
                            const GnParams &gnp = GnParams{}, bool overlap = false)
{
    if (N == 256) return launch_walk_kh<256, SO, GN>(KH, grid, mX, mB, mC, mY, prm, st, gnp, overlap);
    return N == 128 ? launch_walk_kh<128, SO, GN>(KH, grid, mX, mB, mC, mY, prm, st, gnp, overlap)
                    : launch_walk_kh<64, SO, GN>(KH, grid, mX, mB, mC, mY, prm, st, gnp, overlap);
}

// the output pass, with or without the gated norm epilogue
cudaError_t launch_out(const GnParams &gnp, int N, int KH, int grid, const CUtensorMap &mX, const CUtensorMap &mB,
                       const CUtensorMap &mC, const CUtensorMap &mY, const TcParams &prm, cudaStream_t st,
                       bool overlap = false)
{
    return gnp.z ? launch_walk_any<false, true>(N, KH, grid, mX, mB, mC, mY, prm, st, gnp, overlap)
                 : launch_walk_any<false, false>(N, KH, grid, mX, mB, mC, mY, prm, st, GnParams{}, overlap);
}

template <int NST, int KH, bool GN>
cudaError_t launch_fused_t(int grid, const CUtensorMap &mX, const CUtensorMap &mB, const CUtensorMap &mC,
                           const CUtensorMap &mY, const TcParams &prm, const GnParams &gnp, const FuseParams &fp,
                           bool after_walk, cudaStream_t st)
{
    const size_t smem = tc_smem_bytes<NST>();
    cudaError_t e = cudaFuncSetAttribute(ssd_tc_fused<NST, KH, GN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreadsTc);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (after_walk) {
        // behind whole waves of the plain walk, which writes nothing this launch reads: start as
        // SMs free up (the grid is at most one CTA per SM, so every CTA becomes resident)
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    } else {
        // the CTAs of a pair wait for one another: all resident at once
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, ssd_tc_fused<NST, KH, GN>, mX, mB, mC, mY, prm, gnp, fp);
}

template <int NST, bool GN>
cudaError_t launch_fused_kh(int KH, int grid, const CUtensorMap &mX, const CUtensorMap &mB, const CUtensorMap &mC,
                            const CUtensorMap &mY, const TcParams &prm, const GnParams &gnp, const FuseParams &fp,
                            bool after_walk, cudaStream_t st)
{
    return KH == 2 ? launch_fused_t<NST, 2, GN>(grid, mX, mB, mC, mY, prm, gnp, fp, after_walk, st)
                   : launch_fused_t<NST, 1, GN>(grid, mX, mB, mC, mY, prm, gnp, fp, after_walk, st);
}

template <bool GN>
cudaError_t launch_fused_n(int N, int KH, int grid, const CUtensorMap &mX, const CUtensorMap &mB,
                           const CUtensorMap &mC, const CUtensorMap &mY, const TcParams &prm, const GnParams &gnp,
                           const FuseParams &fp, bool after_walk, cudaStream_t st)
{
    if (N == 256) return launch_fused_kh<256, GN>(KH, grid, mX, mB, mC, mY, prm, gnp, fp, after_walk, st);
    return N == 128 ? launch_fused_kh<128, GN>(KH, grid, mX, mB, mC, mY, prm, gnp, fp, after_walk, st)
                    : launch_fused_kh<64, GN>(KH, grid, mX, mB, mC, mY, prm, gnp, fp, after_walk, st);
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// SMs of the current device, looked up once per device.
int device_sms()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kPlanSMs;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = kPlanSMs;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Schedule of equal-length rows (no cu_seqlens): work item = (row, block of KH
// heads), taken from the block index.  Whole waves of the SMs walk whole rows in
// one launch; the pairs left over either join that launch (a last partial
// wave), or run as one-head items in a second launch, or are cut into nseg
// segments each and run by the single-launch segmented walk (ssd_tc_fused),
// whichever a cost model in block steps of one SM prefers: a whole row costs
// nblk, a one-head row about 0.6 nblk (started as SMs free up), a row cut into
// segments of L blocks (the last one the rest) (1 + r) L + 6: every segment's
// full walk starts after the slowest state-only walk (r: its cost per block
// relative to the full walk; measured 0.4 at dstate 256, taken 0.5 below),
// plus about 6 blocks for the second pipeline fill, the exchange and the drains
// (measured on one B200: 6 to 8).
struct UniformPlan {
    int full;      // items of the whole-row launch (from item 0)
    int tail1;     // one-head items of the second launch (the pairs after `full`), 0 = none
    int pairs;     // pairs of the segmented launch (the pairs after `full`), 0 = none
    int nseg, seg_len;
};

UniformPlan uniform_plan(const ssd_fwd_params &p, const TcPlanShape &s)
{
    UniformPlan u{};
    const long long items = (long long)p.batch * s.n_hb;
    const long long sms = std::min(kPlanSMs, device_sms());
    const long long nblk = (p.seqlen + kQ - 1) / kQ;
    const long long full = items / sms * sms, left = items - full;
    u.full = (int)items;
    if (left == 0 || nblk < 2) return u;
    double best = (double)nblk;
    int mode = 0;
    if (s.KH == 2 && full > 0 && 0.6 * (double)nblk < best) {
        best = 0.6 * (double)nblk;
        mode = 1;
    }
    const double r = p.dstate >= 256 ? 0.4 : 0.5;
    const long long nmax = std::min<long long>(std::min<long long>(sms / left, nblk), 64);
    long long bn = 0, bl = 0;
    for (long long n = 2; n <= nmax; ++n) {
        const long long L = (nblk + n - 1) / n;
        if (nblk - (n - 1) * L < 1) continue;     // the last segment would be empty
        const double c = (1.0 + r) * (double)L + 6.0;
        if (c < best - 1e-9) {
            best = c;
            mode = 2;
            bn = n;
            bl = L;
        }
    }
    if (mode == 1) {
        u.full = (int)full;
        u.tail1 = (int)(2 * left);
    } else if (mode == 2) {
        u.full = (int)full;
        u.pairs = (int)left;
        u.nseg = (int)bn;
        u.seg_len = (int)(bl * kQ);
    }
    return u;
}

size_t fused_state_bytes(const ssd_fwd_params &p, const TcPlanShape &s, const UniformPlan &u)
{
    const size_t rows = (size_t)u.pairs * u.nseg * s.KH;
    return align256(rows * kP * p.dstate * sizeof(float)) + align256(rows * sizeof(float));
}

}  // namespace

bool tc_supported(const ssd_fwd_params &p)
{
    return p.io_dtype == SSD_DTYPE_BF16 && p.headdim == kP &&
           (p.dstate == 64 || p.dstate == 128 || p.dstate == 256) &&
           p.dt_softplus == 1 && p.chunk_len >= 128 && (long long)p.batch * p.seqlen >= kQ;
}

size_t tc_workspace_bytes(const ssd_fwd_params &p)
{
    const TcPlanShape s = plan_shape(p);
    if (p.num_seqs == 0) return fused_state_bytes(p, s, uniform_plan(p, s));
    size_t b = align256(sizeof(TcItem) * (size_t)s.max_items);
    if (s.segmented) {
        b += align256((size_t)s.max_segments * p.nheads * kP * p.dstate * sizeof(float));
        b += align256((size_t)s.max_segments * p.nheads * sizeof(float));
        const int nseq = p.num_seqs > 0 ? p.num_seqs : p.batch;
        b += align256((size_t)nseq * sizeof(int));
    }
    return b;
}

int tc_launch_count(const ssd_fwd_params &p)
{
    const TcPlanShape s = plan_shape(p);
    if (p.num_seqs == 0) {
        const UniformPlan u = uniform_plan(p, s);
        return (u.full > 0 ? 1 : 0) + (u.tail1 > 0 || u.pairs > 0 ? 1 : 0);
    }
    return s.segmented ? 4 : 2;
}

namespace {
// Equal-length rows: see uniform_plan.
cudaError_t launch_tc_uniform(const ssd_fwd_params &p, const Plan &plan, const TcArgs &a, const TcPlanShape &s,
                              TcParams prm, const GnParams &gnp, cudaStream_t stream, const Instr &ins)
{
    const UniformPlan u = uniform_plan(p, s);
    const long long tokens = (long long)p.batch * p.seqlen;
    // the status word, and the segmented launch's counters (two per pair, in the status region)
    if (2 * (size_t)u.pairs > kStatusRegion / sizeof(int) - kSyncOffsetInts) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(plan.status, 0, sizeof(int) * (kSyncOffsetInts + 2 * (size_t)u.pairs), stream);
    if (e != cudaSuccess || tokens == 0) return e;
    CUtensorMap mX, mB, mC, mY;
    // y has x's layout; its map moves 32-row slabs (one per epilogue warp)
    if (!make_map(&mX, a.x, (uint64_t)p.nheads * kP, (uint64_t)tokens) ||
        !make_map(&mY, a.y, (uint64_t)p.nheads * kP, (uint64_t)tokens, 32) ||
        !make_map(&mB, a.B, (uint64_t)p.ngroups * p.dstate, (uint64_t)tokens) ||
        !make_map(&mC, a.C, (uint64_t)p.ngroups * p.dstate, (uint64_t)tokens))
        return cudaErrorInvalidValue;
    prm.items = nullptr;
    prm.direct_base = 0;
    if (u.pairs > 0) {
        char *ws = static_cast<char *>(a.scratch);
        const size_t rows = (size_t)u.pairs * u.nseg * s.KH;
        prm.segstate = reinterpret_cast<float *>(ws);
        prm.seglogdec = reinterpret_cast<float *>(ws + align256(rows * kP * p.dstate * sizeof(float)));
    }
    // one launch holds every phase of the work, so the output pass is the whole forward
    if (ins.begin) cudaEventRecord(ins.begin, stream);
    if (ins.main) cudaEventRecord(ins.main, stream);
    if (u.full > 0) {
        prm.n_items = u.full;
        e = launch_out(gnp, p.dstate, s.KH, u.full, mX, mB, mC, mY, prm, stream);
    }
    if (e == cudaSuccess && u.tail1 > 0) {
        TcParams tail = prm;
        tail.direct_base = u.full * 2;
        tail.n_items = u.tail1;
        e = launch_out(gnp, p.dstate, 1, u.tail1, mX, mB, mC, mY, tail, stream, /*overlap=*/true);
    }
    if (e == cudaSuccess && u.pairs > 0) {
        FuseParams fp;
        fp.ctr = plan.status + kSyncOffsetInts;
        fp.pair_base = u.full;
        fp.nseg = u.nseg;
        fp.seg_len = u.seg_len;
        const int grid = u.pairs * u.nseg;
        e = gnp.z ? launch_fused_n<true>(p.dstate, s.KH, grid, mX, mB, mC, mY, prm, gnp, fp, u.full > 0, stream)
                  : launch_fused_n<false>(p.dstate, s.KH, grid, mX, mB, mC, mY, prm, gnp, fp, u.full > 0, stream);
    }
    if (ins.end) cudaEventRecord(ins.end, stream);
    return e;
}
}  // namespace

cudaError_t launch_tc(const ssd_fwd_params &p, const Plan &plan, const Dims &d, const TcArgs &a,
                      cudaStream_t stream, const Instr &ins)
{
    const TcPlanShape s = plan_shape(p);
    TcParams prm;
    prm.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    prm.A_log = a.A_log;
    prm.D = a.D;
    prm.init = a.init;
    prm.y = static_cast<__nv_bfloat16 *>(a.y);
    prm.final_states = a.final_states;
    prm.segstate = nullptr;
    prm.seglogdec = nullptr;
    prm.items = nullptr;
    prm.count = plan.count;
    prm.n_items = 0;
    prm.direct_base = 0;
    prm.seqlen = p.seqlen;
    prm.status = plan.status;
    prm.H = p.nheads;
    prm.G = p.ngroups;
    prm.N = p.dstate;
    prm.heads_per_group = d.heads_per_group;
    prm.dt_softplus = p.dt_softplus;
    prm.withhold_x0 = ins.withhold_first_tile != 0;
    prm.summary = 0;
    GnParams gnp{static_cast<const __nv_bfloat16 *>(a.z), a.gn_w, a.gn_b, a.gn_eps};
    if (p.num_seqs == 0) return launch_tc_uniform(p, plan, a, s, prm, gnp, stream, ins);

    // packed sequences (cu_seqlens): the planner builds the work items on the device
    char *ws = static_cast<char *>(a.scratch);
    TcItem *items = reinterpret_cast<TcItem *>(ws);
    size_t off = align256(sizeof(TcItem) * (size_t)s.max_items);
    float *segstate = nullptr, *seglogdec = nullptr;
    int *seqseg = nullptr;
    if (s.segmented) {
        segstate = reinterpret_cast<float *>(ws + off);
        off += align256((size_t)s.max_segments * p.nheads * kP * p.dstate * sizeof(float));
        seglogdec = reinterpret_cast<float *>(ws + off);
        off += align256((size_t)s.max_segments * p.nheads * sizeof(float));
        seqseg = reinterpret_cast<int *>(ws + off);
    }
    const long long tokens = (long long)p.batch * p.seqlen;
    const int PN = kP * p.dstate;
    const int nseq = plan.nseq;
    tc_plan_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, nseq, p.seqlen, s.seg_len, s.n_hb, s.KH, items, plan.count,
                                           s.max_items, plan.status, a.init, a.final_states, p.nheads, PN, seqseg);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || tokens == 0) return e;

    CUtensorMap mX, mB, mC, mY;
    // y has x's layout; its map moves 32-row slabs (one per epilogue warp)
    if (!make_map(&mX, a.x, (uint64_t)p.nheads * kP, (uint64_t)tokens) ||
        !make_map(&mY, a.y, (uint64_t)p.nheads * kP, (uint64_t)tokens, 32) ||
        !make_map(&mB, a.B, (uint64_t)p.ngroups * p.dstate, (uint64_t)tokens) ||
        !make_map(&mC, a.C, (uint64_t)p.ngroups * p.dstate, (uint64_t)tokens))
        return cudaErrorInvalidValue;

    prm.segstate = segstate;
    prm.seglogdec = seglogdec;
    prm.items = items;
    prm.n_items = s.max_items;

    if (ins.begin) cudaEventRecord(ins.begin, stream);
    if (s.segmented) {
        e = launch_walk_any<true>(p.dstate, s.KH, s.max_items, mX, mB, mC, mY, prm, stream);
        if (e != cudaSuccess) return e;
        const dim3 gs(nseq, p.nheads, (PN + 255) / 256);
        tc_seg_scan_kernel<<<gs, 256, 0, stream>>>(items, seqseg, s.n_hb, segstate, seglogdec, a.init, p.nheads, PN,
                                                   plan.count, s.max_segments);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (ins.main) cudaEventRecord(ins.main, stream);
    e = launch_out(gnp, p.dstate, s.KH, s.max_items, mX, mB, mC, mY, prm, stream);
    if (ins.end) cudaEventRecord(ins.end, stream);
    return e;
}

// State summary on the tensor-core path: every sequence's end state from a
// zero state and its total log decay, by the state-only walk over whole
// sequences (one segment each).
cudaError_t launch_tc_summary(const ssd_fwd_params &p, const Plan &plan, const TcArgs &a, float *end_states,
                              float *logdecay, cudaStream_t stream)
{
    TcPlanShape s = plan_shape(p);
    const long long tokens = (long long)p.batch * p.seqlen;
    const int nseq = plan.nseq;
    s.seg_len = (int)(p.num_seqs > 0 ? (tokens > 0 ? tokens : 1) : (p.seqlen > 0 ? p.seqlen : 1));
    s.max_segments = nseq;
    s.max_items = nseq * s.n_hb;
    s.segmented = false;
    TcItem *items = reinterpret_cast<TcItem *>(a.scratch);
    const int PN = kP * p.dstate;
    cudaError_t e = cudaMemsetAsync(logdecay, 0, sizeof(float) * (size_t)nseq * p.nheads, stream);
    if (e != cudaSuccess) return e;
    const bool direct = p.num_seqs == 0;
    if (direct) {
        e = cudaMemsetAsync(plan.status, 0, sizeof(int), stream);
    } else {
        // empty sequences get a zero end state here (no initial state); the others get items
        tc_plan_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, nseq, p.seqlen, s.seg_len, s.n_hb, s.KH, items,
                                               plan.count, s.max_items, plan.status, nullptr, end_states,
                                               p.nheads, PN, nullptr);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess || tokens == 0) return e;
    CUtensorMap mX, mB;
    if (!make_map(&mX, a.x, (uint64_t)p.nheads * kP, (uint64_t)tokens) ||
        !make_map(&mB, a.B, (uint64_t)p.ngroups * p.dstate, (uint64_t)tokens))
        return cudaErrorInvalidValue;
    TcParams prm{};
    prm.dt = static_cast<const __nv_bfloat16 *>(a.dt);
    prm.A_log = a.A_log;
    prm.segstate = end_states;
    prm.seglogdec = logdecay;
    prm.items = direct ? nullptr : items;
    prm.count = plan.count;
    prm.n_items = s.max_items;
    prm.direct_base = 0;
    prm.seqlen = p.seqlen;
    prm.status = plan.status;
    prm.H = p.nheads;
    prm.G = p.ngroups;
    prm.N = p.dstate;
    prm.heads_per_group = p.nheads / p.ngroups;
    prm.dt_softplus = p.dt_softplus;
    prm.summary = 1;
    // C and y maps are not read in state-only mode
    return launch_walk_any<true>(p.dstate, s.KH, s.max_items, mX, mB, mB, mX, prm, stream);
}

size_t tc_summary_workspace_bytes(const ssd_fwd_params &p)
{
    const TcPlanShape s = plan_shape(p);
    const int nseq = p.num_seqs > 0 ? p.num_seqs : p.batch;
    return align256(sizeof(TcItem) * (size_t)nseq * s.n_hb);
}

}  // namespace ssd

#ifdef SSD_TRACE
extern "C" SSD_API int ssd_trace_enable(long long *buf)
{
    return (int)cudaMemcpyToSymbol(ssd::g_trace, &buf, sizeof(buf));
}
#endif
