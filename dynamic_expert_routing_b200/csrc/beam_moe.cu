// beam_moe.cu -- C ABI and host orchestration of the BEAM masked MoE-layer forward (sm_100a).
//
// One handle owns the repacked weights and every workspace buffer, sized at create time for
// max_tokens, so the forward allocates nothing and never synchronises with the host: the
// per-expert token counts are produced and consumed on the device.  Kernels are chained with
// programmatic dependent launch (each waits on griddepcontrol before reading its producer's
// output), so a kernel's launch overlaps the tail of the one before it.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/beam_moe.h"
#include "common.cuh"
#include "router.cuh"
#include "compact.cuh"
#include "stream_experts.cuh"
#include "tc_experts.cuh"
#include "tc_down_astat.cuh"
#include "decode_fused.cuh"
#include "route_grad.cuh"
#include "softtopk.cuh"

using namespace beam;

// ---------------------------------------------------------------- errors
static thread_local char g_err[512] = "";

static beam_status_t fail(beam_status_t st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return st;
}

#define BEAM_CUDA(call)                                                                   \
    do {                                                                                  \
        cudaError_t e_ = (call);                                                          \
        if (e_ != cudaSuccess)                                                            \
            return fail(BEAM_ERR_CUDA, "%s failed: %s (%s:%d)", #call,                    \
                        cudaGetErrorString(e_), __FILE__, __LINE__);                      \
    } while (0)

// ---------------------------------------------------------------- repack kernels
// Wrm [n_pad][D] for nL layers (W_r, W_m [nL][D][E]): row 2lE + j (j < E) is column j of layer
// l's W_r, row 2lE + E + j column j of its W_m; rows from 2E*nL on are zero.  One layer: the
// layer's router; nL layers: the cross-layer mask generator.
template <typename T>
__global__ void repack_router_kernel(const T* __restrict__ wr, const T* __restrict__ wm, int D,
                                     int E, int nL, int n_pad, T* __restrict__ out)
{
    const size_t n = (size_t)n_pad * D;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
         i += (size_t)gridDim.x * blockDim.x) {
        const int j = (int)(i / D), d = (int)(i % D);
        const int l = j / (2 * E), c = j % (2 * E);
        T v = from_float<T>(0.f);
        if (l < nL) {
            const size_t base = ((size_t)l * D + d) * E;
            v = c < E ? wr[base + c] : wm[base + (c - E)];
        }
        out[i] = v;
    }
}

// Gate/up interleaving in blocks of 128 rows: out[e][b][0][r][:] = wg[e][128b + r][:],
// out[e][b][1][r][:] = wu[e][128b + r][:].  One block of 128 threads per output row.
template <typename T>
__global__ void repack_gateup_kernel(const T* __restrict__ wg, const T* __restrict__ wu, int nE,
                                     int F, int D, T* __restrict__ out)
{
    const long long row = blockIdx.x;  // output row in [nE][F/128][2][128]
    const long long nrows = (long long)nE * 2 * F;
    if (row >= nrows) return;
    const int r = (int)(row % 128);
    const int half = (int)((row / 128) % 2);
    const long long b = row / 256;       // global 128-row block index (e * F/128 + block)
    const long long src_row = b * 128 + r;  // row of [nE*F][D]
    const uint4* s = reinterpret_cast<const uint4*>((half ? wu : wg) + src_row * D);
    uint4* d = reinterpret_cast<uint4*>(out + row * D);
    const int nv = D * (int)sizeof(T) / 16;
    for (int v = threadIdx.x; v < nv; v += blockDim.x) d[v] = s[v];
}

// Down projection into the type of H (fp16 for bf16 layers: exact for every bf16 value of
// magnitude >= 2^-14, within 2^-25 absolute below it; a magnitude >= 65504 sets *bad).
// Routed: out[e][j][f] = w[e][j][f] (S = 1, Fs = F, n = E*D*F).  Shared concatenation:
// out[j][s*Fs + f] = w[s][j][f].
template <typename TI, typename TO>
__global__ void repack_down_kernel(const TI* __restrict__ w, long long n, int S, int D, int Fs,
                                   int concat, TO* __restrict__ out, int* __restrict__ bad)
{
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const float v = to_float(w[i]);
        if (!(fabsf(v) < 65504.f) && sizeof(TO) == 2) atomicOr(bad, 1);
        long long o = i;
        if (concat) {
            const long long f = i % Fs;
            const long long j = (i / Fs) % D;
            const long long s = i / ((long long)Fs * D);
            o = j * S * Fs + s * Fs + f;
        }
        out[o] = from_float<TO>(v);
    }
}

// ---------------------------------------------------------------- the handle
// Routing given by the caller (beam_moe_forward_routed): the forward then starts at the
// compaction.  gate and mlogit are optional (only beam_moe_get_routing reads them).
struct RouteIn {
    const int* topk_id = nullptr;
    const uint8_t* keep = nullptr;
    const float* ghat = nullptr;
    const int* nkeep = nullptr;
    const float* lreg = nullptr;
    const float* gate = nullptr;
    const float* mlogit = nullptr;
    bool operator==(const RouteIn& o) const {
        return topk_id == o.topk_id && keep == o.keep && ghat == o.ghat && nkeep == o.nkeep &&
               lreg == o.lreg && gate == o.gate && mlogit == o.mlogit;
    }
};

struct beam_moe;
static RouteIn own_routing(const beam_moe* h);

// Where a forward left the routed experts' outputs Y_perm: `splits` slices `stride` elements
// apart (added in slice order), fp16 or fp32.
struct YOut {
    const void* base = nullptr;
    int splits = 1;
    long long stride = 0;
    bool f16 = false;
};

struct beam_moe {
    beam_moe_config_t cfg;
    int E, K, D, F, Fsh, Tmax, S;
    int Ew = 0;          // routed experts whose weights the handle holds: E, or 0 for the
                         // routing-only handle of expert parallelism (beam_moe_create_ep)
    int n2E;             // 2E: router + mask logit columns
    int ldL;             // leading dimension of the logits and rows of the repacked router
    size_t esz;
    int num_sms;
    int max_nch;
    // repacked weights
    void *wrm = nullptr, *wgu = nullptr, *wd = nullptr, *wsgu = nullptr, *wsd = nullptr;
    // routing workspace
    float* L = nullptr;
    int* topk_id = nullptr;
    float *gate = nullptr, *mlogit = nullptr, *ghat = nullptr;
    uint8_t* keep = nullptr;
    int* nkeep_tok = nullptr;
    float* lreg_tok = nullptr;
    uint32_t* bits = nullptr;
    int *chunk_base = nullptr, *counts = nullptr, *offsets = nullptr, *perm = nullptr, *inv = nullptr;
    ScanPart* scan_part = nullptr;  // compact_scan's per-CTA statistics
    Group* groups = nullptr;
    int* n_groups = nullptr;     // [0]: kept groups, [1]: their 128-row tiles
    Group* tile_group = nullptr; // 128-row tile (numbered across the groups) -> its group
    DevStats* dstats = nullptr;
    // expert workspace
    void *xperm = nullptr, *hbuf = nullptr, *hsh = nullptr;
    float *yperm = nullptr, *ysh = nullptr;
    // host-call staging
    void* x_stage = nullptr;
    float* y_stage = nullptr;
    __nv_bfloat16* y16_stage = nullptr;   // bf16 y of a BEAM_HOST_Y_BF16 host call
    // pipelined host calls (BEAM_HOST_PIPELINE): copy streams, per-chunk events, statistics
    // accumulated over the chunks
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    cudaEvent_t ev_in[4] = {}, ev_out[4] = {};
    cudaEvent_t ev_copied = nullptr;
    // asynchronous host calls (BEAM_HOST_ASYNC): a second staging set, allocated on the first
    // such call; call k uses set k % 2.  ev_ax_free[b]: the forward that read x set b and
    // wrote y set b is done; ev_ay_free[b]: the copy out of y set b is done; ev_async_last: the
    // last asynchronous call's copy out.
    void* x_stage2 = nullptr;
    float* y_stage2 = nullptr;
    __nv_bfloat16* y16_stage2 = nullptr;
    cudaEvent_t ev_ax_ready[2] = {}, ev_ax_free[2] = {}, ev_ay_free[2] = {}, ev_async_last = nullptr;
    bool async_used[2] = {false, false};
    int async_next = 0;
    bool async_pending = false;
    DevStats* acc_stats = nullptr;
    int* acc_counts = nullptr;
    bool last_pipelined = false;
    size_t hsz;          // bytes per element of H and of the stored down projections
    bool tc_ok = false;  // tensor-core expert path available (bf16, D % 256 == 0)
    bool fused_ok = false;  // fused decode launch available (tc_ok and cooperative launches)
    PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    tc::TcParams p0;      // router GEMM (one dense problem; its x map is set per forward)
    tc::TcParams p1, p2;  // GEMM1 / GEMM2 parameters (the x map of GEMM1 is set per forward)
    tc::TcParams p1s;     // GEMM1 in split-K mode: f32 partials into g1part
    int split_rows = 0;   // token rows (routed: x K) the split-K workspaces hold
    float* g1part = nullptr;     // [kMaxSplits][split_rows*K][2F]
    float* g1part_sh = nullptr;  // [kMaxSplits][split_rows][2Fsh]
    float* ypart = nullptr;      // [kMaxSplits][split_rows*K][D]
    float* ysh_part = nullptr;   // [kMaxSplits][split_rows][D]
    // tail split of the routed problem's whole-K launches: partial workspace and arrival
    // counters (cleared by the compaction scan of every forward)
    float* tail_ws = nullptr;
    int* tail_cnt = nullptr;     // [kTailCntRegions][num_sms][kEpiWarps]
    int* fold_cnt = nullptr;     // split-K gate/up with SwiGLU folded in: arrival counters
                                 // [E * 2F/256 + 2Fsh/256][4], zero between launches
    int* zero_int = nullptr;     // two zeros: an empty group table
    int* range_flag = nullptr;
    unsigned* rcnt = nullptr;    // arrival counters of the small-batch router, one per block of
                                 // 8 logit columns; zero between calls
    cudaEvent_t done = nullptr;
    // side stream for the shared experts (they depend on x only, so they overlap routing)
    cudaStream_t side = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    int last_T = -1;
    // training: the last forward's mode and where it left Y_perm (read by the routing
    // gradient), the per-pair logit gradients and the dW partial columns
    bool last_train = false;
    YOut last_yr;
    float2* pair_grad = nullptr;  // [Tmax*K] (d_gate_logit, d_mask_logit) of routed rows, at
                                  // each pair's position in perm
    int dw_chunks = 0;            // column chunks of the dW pass (32 vectors of x each)
    float* dw_part = nullptr;     // [16*num_sms/dw_chunks + E + 1][2][D] partial columns
    int* dw_cnt = nullptr;        // [E][dw_chunks] arrival counters, zero between calls
    std::vector<void*> allocs;
    // replay cache: the last forward captured as a CUDA graph, keyed by its arguments
    cudaGraphExec_t graph_exec = nullptr;
    const void* g_x = nullptr;
    float* g_y = nullptr;
    int g_T = -1;
    uint32_t g_flags = 0;
    bool g_tc = false;
    RouteIn cur;         // the routing arrays the last forward read (beam_moe_get_routing)
    int g_kernels = 0;   // kernels in the captured graph
    bool g_routed = false;
    RouteIn g_rin;       // routing pointers of a captured routed forward
    // expert parallelism: the last beam_moe_ep_dispatch (token count, where the shared experts'
    // output is, whether they ran on the side stream), read by beam_moe_ep_combine
    int ep_T = -1;
    YOut ep_ysh;
    bool ep_fork = false;
    YOut g_yr;           // Y_perm of the captured forward
    // launch accounting and optional per-stage timing
    long long launches = 0;
    bool prof = false;
    int prof_max = 0, prof_forwards = 0;
    std::vector<cudaEvent_t> prof_pool;   // free events
    struct ProfRec { int stage; cudaEvent_t a, b; };
    std::vector<ProfRec> prof_recs;
};

enum Stage {
    ST_ROUTER_LOGITS = 0, ST_ROUTE_SELECT, ST_COMPACT_BITS, ST_COMPACT_SCAN, ST_SCATTER_GATHER,
    ST_STREAM_GATEUP, ST_STREAM_DOWN, ST_COMBINE, ST_TC_GATEUP, ST_TC_DOWN, ST_TC_ROUTER,
    ST_TC_SH_GATEUP, ST_TC_SH_DOWN, ST_FUSED_DECODE,
    ST_ROUTE_GRAD, ST_ROUTE_DW, ST_CHUNK_STATS, ST_COUNT
};
static_assert(ST_COUNT == BEAM_N_STAGES, "stage table out of sync with the header");
static const char* kStageNames[ST_COUNT] = {
    "router_logits", "route_select", "compact_bits", "compact_scan", "scatter_gather",
    "stream_gateup", "stream_down", "combine", "tc_gateup", "tc_down", "tc_router",
    "tc_shared_gateup", "tc_shared_down",
    "fused_decode", "route_grad", "route_dw", "chunk_stats"};

static void prof_release(beam_moe* h)
{
    for (auto& r : h->prof_recs) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
    h->prof_recs.clear();
    for (cudaEvent_t e : h->prof_pool) cudaEventDestroy(e);
    h->prof_pool.clear();
    h->prof = false;
}

static void drop_graph(beam_moe* h)
{
    if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
    h->graph_exec = nullptr;
    h->g_T = -1;
}

static void free_all(beam_moe* h)
{
    drop_graph(h);
    prof_release(h);
    for (void* p : h->allocs) cudaFree(p);
    h->allocs.clear();
    if (h->done) cudaEventDestroy(h->done);
    h->done = nullptr;
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->side) cudaStreamDestroy(h->side);
    h->ev_fork = h->ev_join = nullptr;
    h->side = nullptr;
    for (int i = 0; i < 4; ++i) {
        if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
        if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
        h->ev_in[i] = h->ev_out[i] = nullptr;
    }
    if (h->ev_copied) cudaEventDestroy(h->ev_copied);
    for (int b = 0; b < 2; ++b) {
        if (h->ev_ax_ready[b]) cudaEventDestroy(h->ev_ax_ready[b]);
        if (h->ev_ax_free[b]) cudaEventDestroy(h->ev_ax_free[b]);
        if (h->ev_ay_free[b]) cudaEventDestroy(h->ev_ay_free[b]);
        h->ev_ax_ready[b] = h->ev_ax_free[b] = h->ev_ay_free[b] = nullptr;
    }
    if (h->ev_async_last) cudaEventDestroy(h->ev_async_last);
    h->ev_async_last = nullptr;
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
    h->ev_copied = nullptr;
    h->copy_in = h->copy_out = nullptr;
}

// Test hook: BEAM_TEST_FAIL_ALLOC=n makes the n-th device allocation of a create fail as if
// the device were out of memory (n = 1 is the first), so the error path can be exercised.
static int fail_alloc_at()
{
    const char* v = getenv("BEAM_TEST_FAIL_ALLOC");
    return v ? atoi(v) : 0;
}

template <typename P>
static beam_status_t dalloc(beam_moe* h, P** out, size_t bytes)
{
    void* p = nullptr;
    if (bytes == 0) bytes = 16;
    const int fail_at = fail_alloc_at();
    if (fail_at > 0 && (int)h->allocs.size() + 1 == fail_at)
        return fail(BEAM_ERR_OOM, "device allocation %d failed (BEAM_TEST_FAIL_ALLOC)", fail_at);
    cudaError_t e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(BEAM_ERR_OOM, "cudaMalloc of %zu bytes failed: %s", bytes, cudaGetErrorString(e));
    }
    h->allocs.push_back(p);
    *out = static_cast<P*>(p);
    return BEAM_OK;
}

#define BEAM_TRY(x)                              \
    do {                                         \
        beam_status_t s_ = (x);                  \
        if (s_ != BEAM_OK) return s_;            \
    } while (0)

static beam_status_t validate(const beam_moe_config_t* c)
{
    if (!c) return fail(BEAM_ERR_INVALID_ARG, "cfg is NULL");
    if (c->dtype != BEAM_DTYPE_F32 && c->dtype != BEAM_DTYPE_BF16)
        return fail(BEAM_ERR_INVALID_ARG, "dtype must be BEAM_DTYPE_F32 or BEAM_DTYPE_BF16");
    const int dmul = c->dtype == BEAM_DTYPE_BF16 ? 64 : 4;
    const int dmax = c->dtype == BEAM_DTYPE_BF16 ? 8192 : 4096;
    if (c->d_model <= 0 || c->d_model % dmul || c->d_model > dmax)
        return fail(BEAM_ERR_INVALID_ARG, "d_model=%d must be a positive multiple of %d, <= %d",
                    c->d_model, dmul, dmax);
    if (c->n_experts < 1 || c->n_experts > kMaxE)
        return fail(BEAM_ERR_INVALID_ARG, "n_experts=%d must be in [1, %d]", c->n_experts, kMaxE);
    if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > 32)
        return fail(BEAM_ERR_INVALID_ARG, "top_k=%d must be in [1, min(n_experts, 32)]", c->top_k);
    if (c->d_ff <= 0 || c->d_ff % 128 || c->d_ff > 65536)
        return fail(BEAM_ERR_INVALID_ARG, "d_ff=%d must be a positive multiple of 128", c->d_ff);
    if (c->n_shared < 0 || c->n_shared > 16)
        return fail(BEAM_ERR_INVALID_ARG, "n_shared=%d must be in [0, 16]", c->n_shared);
    if (c->n_shared > 0 && (c->d_ff_shared <= 0 || c->d_ff_shared % 128))
        return fail(BEAM_ERR_INVALID_ARG, "d_ff_shared=%d must be a positive multiple of 128",
                    c->d_ff_shared);
    if (c->segment_len < 0 || c->segment_len > 65536)
        return fail(BEAM_ERR_INVALID_ARG, "segment_len=%d out of range", c->segment_len);
    if (c->max_tokens < 1 || c->max_tokens > 65536)
        return fail(BEAM_ERR_INVALID_ARG, "max_tokens=%d must be in [1, 65536]", c->max_tokens);
    return BEAM_OK;
}

static int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// Automatic path choice for bf16 layers: from this many tokens up the experts run on the
// tensor cores (measured on B200 to stream weights faster than the CUDA-core GEMV from one
// token up, once small batches split K); the GEMV path serves fp32 layers and the
// BEAM_PATH_STREAM flag.
constexpr int kTcMinTokens = 1;
// Router logits run on the tensor cores from this many routed rows up (bf16 layers).
constexpr int kTcRouterMinRows = 64;
// Counter regions of the tail split: routed gate/up, routed down.  (The shared problem runs
// concurrently with the routing on a second stream, so its last wave has no idle SMs to fill.)
constexpr int kTailCntRegions = 2;
// The handle's own routing arrays (written by its router and Top-K/mask kernels).
static RouteIn own_routing(const beam_moe* h)
{
    RouteIn r;
    r.topk_id = h->topk_id; r.keep = h->keep; r.ghat = h->ghat; r.nkeep = h->nkeep_tok;
    r.lreg = h->lreg_tok; r.gate = h->gate; r.mlogit = h->mlogit;
    return r;
}

static int tail_cnt_ints(int num_sms) { return kTailCntRegions * num_sms * tc::kEpiWarps; }

// Small batches gather their kept rows inside the fused routing kernel up to this many bytes.
constexpr long long kInlineGatherBytes = 256 * 1024;
// Split-K for small batches on the tensor-core path: up to kMaxSplits K slices per tile, for
// forwards of at most kSplitMaxTokens tokens (the partial-sum workspaces are sized for that).
constexpr int kMaxSplits = 16;
constexpr int kSplitMaxTokens = 64;
constexpr int kMinStepsPerSplit = 4;

// K-split factor that spreads `tiles` output tiles over the SMs, keeping at least
// kMinStepsPerSplit k steps per slice and no empty slice.
// Split count s in [1, kMaxSplits] that minimises the wave makespan of `tiles` tiles split
// s ways on num_sms SMs, ceil(tiles*s/num_sms)/s (in units of one unsplit tile), inflated by
// 4 % per extra split for the per-tile fixed costs and the partial sums written and re-read.
static int choose_splits(int num_sms, long long tiles)
{
    if (tiles <= 0) return 1;
    int best = 1;
    double best_cost = 1e30;
    for (int s = 1; s <= kMaxSplits; ++s) {
        const double waves = (double)((tiles * s + num_sms - 1) / num_sms);
        const double cost = waves / s * (1.0 + 0.04 * (s - 1));
        if (cost < best_cost - 1e-9) { best_cost = cost; best = s; }
    }
    return best;
}

// The split count actually used for a problem with `ksteps` k steps: at least
// kMinStepsPerSplit steps per slice, and slices of equal length except the last, which is
// never empty (every slice writes its partial sums).
static int normalise_splits(int s, int ksteps)
{
    s = std::max(1, std::min(s, std::max(1, ksteps / kMinStepsPerSplit)));
    const int per = (ksteps + s - 1) / s;
    return (ksteps + per - 1) / per;
}

template <typename T>
static beam_status_t repack(beam_moe* h, const beam_moe_weights_t* w, cudaStream_t st)
{
    using TH = typename HType<T>::type;
    const int D = h->D, E = h->E, F = h->F, Ew = h->Ew;
    repack_router_kernel<T><<<1024, 256, 0, st>>>(static_cast<const T*>(w->w_router),
                                                  static_cast<const T*>(w->w_mask), D, E, 1,
                                                  h->ldL, static_cast<T*>(h->wrm));
    BEAM_CUDA(cudaGetLastError());
    if (Ew > 0) {
        repack_gateup_kernel<T><<<(unsigned)((long long)Ew * 2 * F), 128, 0, st>>>(
            static_cast<const T*>(w->w_gate), static_cast<const T*>(w->w_up), Ew, F, D,
            static_cast<T*>(h->wgu));
        BEAM_CUDA(cudaGetLastError());
        repack_down_kernel<T, TH><<<2048, 256, 0, st>>>(static_cast<const T*>(w->w_down),
                                                        (long long)Ew * D * F, 1, D, F, 0,
                                                        static_cast<TH*>(h->wd), h->range_flag);
        BEAM_CUDA(cudaGetLastError());
    }
    if (h->Fsh > 0) {
        repack_gateup_kernel<T><<<(unsigned)(2LL * h->Fsh), 128, 0, st>>>(
            static_cast<const T*>(w->ws_gate), static_cast<const T*>(w->ws_up), 1, h->Fsh, D,
            static_cast<T*>(h->wsgu));
        BEAM_CUDA(cudaGetLastError());
        repack_down_kernel<T, TH><<<1024, 256, 0, st>>>(
            static_cast<const T*>(w->ws_down), (long long)h->cfg.n_shared * D * h->cfg.d_ff_shared,
            h->cfg.n_shared, D, h->cfg.d_ff_shared, 1, static_cast<TH*>(h->wsd), h->range_flag);
        BEAM_CUDA(cudaGetLastError());
    }
    return BEAM_OK;
}

// ---------------------------------------------------------------- tensor-core path set-up
static beam_status_t encode_map(beam_moe* h, CUtensorMap* m, CUtensorMapDataType dt,
                                const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                                uint64_t row_stride_elems = 0)
{
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {(row_stride_elems ? row_stride_elems : cols) * 2};
    cuuint32_t box[2] = {(cuuint32_t)tc::BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = h->encode(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(BEAM_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a %llu x %llu tensor",
                    (int)r, (unsigned long long)rows, (unsigned long long)cols);
    return BEAM_OK;
}

static beam_status_t setup_tc(beam_moe* h)
{
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    BEAM_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
    if (!fn || q != cudaDriverEntryPointSuccess)
        return fail(BEAM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    h->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    const uint64_t D = h->D, E = h->E, F = h->F, Fsh = h->Fsh, Tm = h->Tmax;
    const uint64_t rows = Tm * h->K;
    const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, HF = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    tc::TcParams& a = h->p1;
    tc::TcParams& b = h->p2;
    memset(&a, 0, sizeof a);
    memset(&b, 0, sizeof b);
    // GEMM1: X_perm [rows][D] x W_gu [E*2F][D] -> H (fp16) [rows][F]
    BEAM_TRY(encode_map(h, &a.a_routed, BF, h->xperm, rows, D, tc::BM));
    if (h->Ew > 0) BEAM_TRY(encode_map(h, &a.b_routed, BF, h->wgu, E * 2 * F, D, tc::BN));
    // GEMM2: H [rows][F] x W_d [E*D][F] -> Y_perm (f32) [rows][D]
    BEAM_TRY(encode_map(h, &b.a_routed, HF, h->hbuf, rows, F, tc::BM));
    if (h->Ew > 0) BEAM_TRY(encode_map(h, &b.b_routed, HF, h->wd, E * D, F, tc::BN));
    // the same activations in boxes of kSwapBox rows, for the swapped small groups
    BEAM_TRY(encode_map(h, &a.a_routed_tail, BF, h->xperm, rows, D, tc::kSwapBox));
    BEAM_TRY(encode_map(h, &b.a_routed_tail, HF, h->hbuf, rows, F, tc::kSwapBox));
    if (h->Ew == 0) {
        // a routing-only handle holds no routed expert weights: its launches carry no routed
        // group, so these maps are never read; they point at the router matrix so that every
        // map a kernel is given (and prefetches) is a valid one
        BEAM_TRY(encode_map(h, &a.b_routed, BF, h->wrm, (uint64_t)h->ldL, D, tc::BN));
        BEAM_TRY(encode_map(h, &b.b_routed, BF, h->wrm, (uint64_t)h->ldL, D, tc::BN));
    }
    if (Fsh) {
        BEAM_TRY(encode_map(h, &a.b_shared, BF, h->wsgu, 2 * Fsh, D, tc::BN));
        BEAM_TRY(encode_map(h, &b.a_shared, HF, h->hsh, Tm, Fsh, tc::BM));
        BEAM_TRY(encode_map(h, &b.b_shared, HF, h->wsd, D, Fsh, tc::BN));
    } else {
        a.b_shared = a.b_routed;
        b.a_shared = b.a_routed;
        b.b_shared = b.b_routed;
    }
    a.a_shared = a.a_routed;  // replaced by the map of x in every forward
    a.groups = b.groups = h->groups;
    a.n_groups = b.n_groups = h->n_groups;
    a.tile_group = b.tile_group = h->tile_group;
    a.out_routed = h->hbuf; a.ld_routed = (int)F;
    a.out_shared = h->hsh;  a.ld_shared = (int)Fsh;
    b.out_routed = h->yperm; b.ld_routed = (int)D;
    b.out_shared = h->ysh;   b.ld_shared = (int)D;
    a.b_rows_per_expert = (int)(2 * F);
    b.b_rows_per_expert = (int)D;
    a.n_tiles_routed = (int)(2 * F / tc::BN);
    a.n_tiles_shared = (int)(2 * Fsh / tc::BN);
    b.n_tiles_routed = b.n_tiles_shared = (int)(D / tc::BN);
    a.k_steps_routed = a.k_steps_shared = (int)(D / tc::BK);
    b.k_steps_routed = (int)(F / tc::BK);
    b.k_steps_shared = (int)(Fsh / tc::BK);
    a.err = b.err = &h->dstats->err;
    a.k_splits_routed = a.k_splits_shared = 1;
    b.k_splits_routed = b.k_splits_shared = 1;
    // split-K variant of GEMM1: raw f32 gate/up accumulators, one slice per K split
    {
        const size_t sr = (size_t)std::min(h->Tmax, kSplitMaxTokens);
        h->split_rows = (int)sr;
        BEAM_TRY(dalloc(h, &h->g1part, kMaxSplits * sr * h->K * 2 * F * sizeof(float)));
        BEAM_TRY(dalloc(h, &h->ypart, kMaxSplits * sr * h->K * D * sizeof(float)));
        if (Fsh) {
            BEAM_TRY(dalloc(h, &h->g1part_sh, kMaxSplits * sr * 2 * Fsh * sizeof(float)));
            BEAM_TRY(dalloc(h, &h->ysh_part, kMaxSplits * sr * D * sizeof(float)));
        }
        tc::TcParams& c = h->p1s;
        c = a;
        c.out_routed = h->g1part; c.ld_routed = (int)(2 * F);
        c.out_shared = h->g1part_sh; c.ld_shared = (int)(2 * Fsh);
        c.split_stride_routed = (long long)sr * h->K * 2 * F;
        c.split_stride_shared = (long long)sr * 2 * Fsh;
    }
    // split-K gate/up launches finish SwiGLU in the epilogue: one counter per (tile, lane
    // quadrant); a split launch has at most one 128-row tile per group (<= 64 rows each)
    {
        const size_t n = ((size_t)E * (2 * F / tc::BN) + (Fsh ? 2 * Fsh / tc::BN : 0)) * 4;
        BEAM_TRY(dalloc(h, &h->fold_cnt, n * sizeof(int)));
        BEAM_CUDA(cudaMemset(h->fold_cnt, 0, n * sizeof(int)));
    }
    // tail split: at most kTailMaxSubWaves * num_sms piece slots per launch
    {
        const size_t slots = (size_t)tc::kTailMaxSubWaves * h->num_sms * tc::kEpiWarps;
        BEAM_TRY(dalloc(h, &h->tail_ws, slots * tc::kTailSlotFloats * sizeof(float)));
    }
    // router: logits L [Tr][ldL] = x_rows [Tr][D] . Wrm [ldL][D]^T as one dense problem
    tc::TcParams& r = h->p0;
    memset(&r, 0, sizeof r);
    BEAM_TRY(encode_map(h, &r.b_shared, BF, h->wrm, (uint64_t)h->ldL, D, tc::BN));
    r.b_routed = r.b_shared;
    r.a_routed = r.a_shared = a.a_routed;  // the x map is set in every forward
    r.groups = h->groups;
    r.n_groups = h->zero_int;              // no routed groups
    r.out_routed = r.out_shared = h->L;
    r.ld_routed = r.ld_shared = h->ldL;
    r.b_rows_per_expert = 0;
    r.n_tiles_routed = r.n_tiles_shared = h->ldL / tc::BN;
    r.k_steps_routed = r.k_steps_shared = (int)(D / tc::BK);
    r.k_splits_routed = r.k_splits_shared = 1;
    r.store_cols = 2 * E;                  // columns past 2E are padding nobody reads
    r.err = &h->dstats->err;
    {
        const void* kernels[] = {
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 1, tc::MODE_PLAIN>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_SWIGLU, 1, tc::MODE_PLAIN>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_SWIGLU, 1, tc::MODE_TAIL>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_SWIGLU, 1, tc::MODE_SWAP>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 0, tc::MODE_PLAIN>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F16, 0, tc::MODE_PLAIN>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F16, 0, tc::MODE_TAIL>,
            (const void*)tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F16, 0, tc::MODE_SWAP>};
        for (const void* k : kernels)
            BEAM_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES));
        BEAM_CUDA(cudaFuncSetAttribute((const void*)tc::tc_down_astat_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, tc::AS_SMEM_BYTES));
    }
    // the fused decode kernel: one resident block per SM is required for its grid barriers
    {
        const void* fk[] = {(const void*)fused_decode_kernel<1>, (const void*)fused_decode_kernel<2>,
                            (const void*)fused_decode_kernel<3>, (const void*)fused_decode_kernel<4>,
                            (const void*)fused_decode_kernel<5>, (const void*)fused_decode_kernel<6>,
                            (const void*)fused_decode_kernel<7>, (const void*)fused_decode_kernel<8>};
        for (const void* k : fk)
            BEAM_CUDA(cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES));
        int dev = 0, coop = 0, per_sm = 0;
        BEAM_CUDA(cudaGetDevice(&dev));
        BEAM_CUDA(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
        BEAM_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_decode_kernel<8>,
                                                                tc::kThreads, tc::SMEM_BYTES));
        h->fused_ok = coop != 0 && per_sm >= 1;
    }
    h->tc_ok = true;
    return BEAM_OK;
}

static beam_status_t create_impl(const beam_moe_config_t* cfg, const beam_moe_weights_t* w,
                                 cudaStream_t st, beam_moe* h, bool routing_only = false)
{
    h->cfg = *cfg;
    h->E = cfg->n_experts; h->K = cfg->top_k; h->D = cfg->d_model; h->F = cfg->d_ff;
    h->Ew = routing_only ? 0 : h->E;
    h->Fsh = cfg->n_shared * cfg->d_ff_shared;
    h->Tmax = cfg->max_tokens;
    h->S = cfg->segment_len > 1 ? cfg->segment_len : 1;
    h->n2E = 2 * h->E;
    // bf16 layers pad the router rows to the tensor-core tile width (extra rows are zero)
    h->ldL = (cfg->dtype == BEAM_DTYPE_BF16) ? ((h->n2E + tc::BN - 1) / tc::BN) * tc::BN : h->n2E;
    h->esz = cfg->dtype == BEAM_DTYPE_BF16 ? 2 : 4;
    h->hsz = cfg->dtype == BEAM_DTYPE_BF16 ? 2 : 4;
    h->max_nch = ceil_div(h->Tmax, 32);
    int dev = 0;
    BEAM_CUDA(cudaGetDevice(&dev));
    BEAM_CUDA(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));

    const size_t D = h->D, E = h->E, K = h->K, F = h->F, Fsh = h->Fsh, Tm = h->Tmax;
    const size_t es = h->esz, hs = h->hsz;
    const size_t rows = Tm * K;  // upper bound on kept pairs
    BEAM_TRY(dalloc(h, &h->wrm, (size_t)h->ldL * D * es));
    BEAM_TRY(dalloc(h, &h->zero_int, 2 * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->wgu, (size_t)h->Ew * 2 * F * D * es));
    BEAM_TRY(dalloc(h, &h->wd, (size_t)h->Ew * D * F * hs));
    BEAM_TRY(dalloc(h, &h->range_flag, sizeof(int)));
    if (Fsh) {
        BEAM_TRY(dalloc(h, &h->wsgu, 2 * Fsh * D * es));
        BEAM_TRY(dalloc(h, &h->wsd, D * Fsh * hs));
        BEAM_TRY(dalloc(h, &h->hsh, Tm * Fsh * hs));
        BEAM_TRY(dalloc(h, &h->ysh, Tm * D * sizeof(float)));
    }
    // logits; bf16 layers keep room for K-split slices of the tensor-core router
    // logits; room for K-split slices of the tensor-core router (bf16) and for the D-chunk
    // slices of the small-batch router (at most 16 chunks of kRouterChunkBytes)
    static_assert(8192 * 2 / kRouterChunkBytes <= kMaxSplits && 4096 * 4 / kRouterChunkBytes <= kMaxSplits,
                  "the logit slices of the small-batch router must fit the L buffer");
    BEAM_TRY(dalloc(h, &h->L, (size_t)kMaxSplits * Tm * h->ldL * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->rcnt, (size_t)ceil_div(h->ldL, 8) * sizeof(unsigned)));
    BEAM_CUDA(cudaMemsetAsync(h->rcnt, 0, (size_t)ceil_div(h->ldL, 8) * sizeof(unsigned), st));
    BEAM_TRY(dalloc(h, &h->topk_id, rows * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->gate, rows * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->mlogit, rows * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->ghat, rows * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->keep, rows));
    BEAM_TRY(dalloc(h, &h->nkeep_tok, Tm * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->lreg_tok, Tm * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->bits, E * h->max_nch * sizeof(uint32_t)));
    BEAM_TRY(dalloc(h, &h->chunk_base, E * h->max_nch * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->scan_part, kScanMaxCtas * sizeof(ScanPart)));
    BEAM_TRY(dalloc(h, &h->counts, E * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->offsets, (E + 1) * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->perm, rows * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->inv, rows * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->groups, E * sizeof(Group)));
    BEAM_TRY(dalloc(h, &h->n_groups, 2 * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->tile_group, (ceil_div((long long)rows, kGroupTileRows) + E) * sizeof(Group)));
    BEAM_TRY(dalloc(h, &h->dstats, sizeof(DevStats)));
    BEAM_TRY(dalloc(h, &h->tail_cnt, tail_cnt_ints(h->num_sms) * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->xperm, rows * D * es));
    BEAM_TRY(dalloc(h, &h->hbuf, rows * F * hs));
    BEAM_TRY(dalloc(h, &h->yperm, rows * D * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->x_stage, Tm * D * es));
    BEAM_TRY(dalloc(h, &h->y_stage, Tm * D * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->y16_stage, Tm * D * sizeof(__nv_bfloat16)));
    BEAM_TRY(dalloc(h, &h->acc_stats, sizeof(DevStats)));
    BEAM_TRY(dalloc(h, &h->acc_counts, E * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->pair_grad, rows * sizeof(float2)));
    h->dw_chunks = ceil_div((long long)D, cfg->dtype == BEAM_DTYPE_BF16 ? dw_chunk_cols<__nv_bfloat16>()
                                                                       : dw_chunk_cols<float>());
    BEAM_TRY(dalloc(h, &h->dw_part, (16 * (size_t)h->num_sms / h->dw_chunks + E + 1) * 2 * D * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->dw_cnt, E * (size_t)h->dw_chunks * sizeof(int)));
    BEAM_CUDA(cudaMemsetAsync(h->dstats, 0, sizeof(DevStats), st));
    BEAM_CUDA(cudaMemsetAsync(h->tail_cnt, 0, tail_cnt_ints(h->num_sms) * sizeof(int), st));
    BEAM_CUDA(cudaMemsetAsync(h->range_flag, 0, sizeof(int), st));
    BEAM_CUDA(cudaMemsetAsync(h->dw_cnt, 0, E * (size_t)h->dw_chunks * sizeof(int), st));
    BEAM_CUDA(cudaMemsetAsync(h->zero_int, 0, 2 * sizeof(int), st));
    BEAM_CUDA(cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming));
    BEAM_CUDA(cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking));
    BEAM_CUDA(cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking));
    for (int i = 0; i < 4; ++i) {
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming));
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming));
    }
    BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_copied, cudaEventDisableTiming));
    if (h->Fsh > 0) {
        BEAM_CUDA(cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking));
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming));
    }

    if (cfg->dtype == BEAM_DTYPE_BF16) BEAM_TRY(repack<__nv_bfloat16>(h, w, st));
    else BEAM_TRY(repack<float>(h, w, st));

    if (cfg->dtype == BEAM_DTYPE_BF16) {
        BEAM_CUDA(cudaFuncSetAttribute(stream_gateup_kernel<__nv_bfloat16, __half>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       stream_gateup_smem()));
        BEAM_CUDA(cudaFuncSetAttribute(stream_down_kernel<__half>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       stream_down_smem()));
    } else {
        BEAM_CUDA(cudaFuncSetAttribute(stream_gateup_kernel<float, float>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       stream_gateup_smem()));
        BEAM_CUDA(cudaFuncSetAttribute(stream_down_kernel<float>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       stream_down_smem()));
    }
    BEAM_CUDA(cudaStreamSynchronize(st));
    int bad = 0;
    BEAM_CUDA(cudaMemcpy(&bad, h->range_flag, sizeof bad, cudaMemcpyDeviceToHost));
    if (bad)
        return fail(BEAM_ERR_UNSUPPORTED, "a down-projection weight has magnitude >= 65504, "
                    "outside the fp16 range of the intermediate");
    if (cfg->dtype == BEAM_DTYPE_BF16 && h->D % tc::BN == 0) BEAM_TRY(setup_tc(h));
    return BEAM_OK;
}

// ---------------------------------------------------------------- launch helper (PDL)
// Every forward kernel goes through here: it is counted, launched with programmatic stream
// serialisation, and (while profiling) bracketed by an event pair of its stage.  h == nullptr
// launches the kernel the same way without touching any handle state (no count, no events):
// the allocation-free routing call uses that, so it never writes to the handle.
// BEAM_TRACE=1 in the environment prints every launch (stage, grid, block, shared memory) to
// stderr before it is made, and its launch status after: a host-side fault can then be placed.
static bool trace_on()
{
    static const bool on = getenv("BEAM_TRACE") != nullptr;
    return on;
}

static void trace(const char* fmt, ...)
{
    if (!trace_on()) return;
    va_list ap;
    va_start(ap, fmt);
    fputs("[beam] ", stderr);
    vfprintf(stderr, fmt, ap);
    fputc('\n', stderr);
    fflush(stderr);
    va_end(ap);
}

template <typename... KArgs, typename... Args>
static cudaError_t launch_ex(beam_moe* h, int stage, bool coop, void (*kernel)(KArgs...), dim3 grid,
                             dim3 block, size_t smem, cudaStream_t st, Args&&... args)
{
    trace("launch stage %d grid (%u,%u,%u) block %u smem %zu stream %p", stage, grid.x, grid.y,
          grid.z, block.x, smem, (void*)st);
    cudaEvent_t ea = nullptr, eb = nullptr;
    if (h && h->prof && h->prof_pool.size() >= 2) {
        ea = h->prof_pool.back(); h->prof_pool.pop_back();
        eb = h->prof_pool.back(); h->prof_pool.pop_back();
        cudaError_t e = cudaEventRecord(ea, st);
        if (e != cudaSuccess) return e;
    }
    if (h) ++h->launches;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    if (coop) {
        // a cooperative launch: every block resident at once (the kernel has grid barriers)
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    }
    lc.attrs = attr;
    lc.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
    trace("  -> %s", cudaGetErrorString(e));
    if (e == cudaSuccess && ea) {
        e = cudaEventRecord(eb, st);
        h->prof_recs.push_back({stage, ea, eb});
    }
    return e;
}

template <typename... KArgs, typename... Args>
static cudaError_t launch(beam_moe* h, int stage, void (*kernel)(KArgs...), dim3 grid,
                          dim3 block, size_t smem, cudaStream_t st, Args&&... args)
{
    return launch_ex(h, stage, false, kernel, grid, block, smem, st, std::forward<Args>(args)...);
}

// Router logits on the CUDA cores, L[r][j] (leading dimension ld) for ncols columns of the
// repacked matrix w [ncols][D]: one CTA per column, or one warp per column from
// kGemvWarpCols columns on (the choice depends on the column count alone, so a one-layer
// generator and the layer with the same matrices compute the same bits).
constexpr int kGemvWarpCols = 2048;
// Up to this many routed rows the one-CTA-per-column GEMV is faster than the small-batch router
// (measured on B200: 4.8 against 7.1 us for one token of the Mixtral-like layer): with so few
// rows the shared-memory staging and the cross-chunk sum do not pay.
constexpr int kRouterGemvMaxRows = 4;

template <typename T>
static cudaError_t launch_router_gemv(beam_moe* h, const T* x, int S, int Tr, int D, const T* w,
                                      int ncols, int ld, float* L, cudaStream_t st)
{
    if (ncols >= kGemvWarpCols) {
        const dim3 grid1(ceil_div(ncols, 8), Tr);
        if (Tr == 1)
            return launch(h, ST_ROUTER_LOGITS, router_gemv_warp_kernel<T, 1>, grid1, dim3(256), 0,
                          st, x, S, Tr, D, w, ncols, ld, L);
        if (Tr <= 4)
            return launch(h, ST_ROUTER_LOGITS, router_gemv_warp_kernel<T, 4>,
                          dim3(ceil_div(ncols, 8), 1), dim3(256), 0, st, x, S, Tr, D, w, ncols, ld, L);
        return launch(h, ST_ROUTER_LOGITS, router_gemv_warp_kernel<T, kGemvRows>,
                      dim3(ceil_div(ncols, 8), ceil_div(Tr, kGemvRows)), dim3(256), 0, st, x, S,
                      Tr, D, w, ncols, ld, L);
    }
    return launch(h, ST_ROUTER_LOGITS, router_gemv_kernel<T>, dim3(ncols, ceil_div(Tr, kGemvRows)),
                  dim3(256), 0, st, x, S, Tr, D, w, ncols, ld, L);
}

template <int EPL>
static cudaError_t launch_select(beam_moe* h, int Tr, int T, int mask_off, int splits,
                                 long long split_stride, cudaStream_t st)
{
    return launch(h, ST_ROUTE_SELECT, route_select_kernel<EPL>, dim3(ceil_div(Tr, 8)), dim3(256), 0, st,
                  (const float*)h->L, h->ldL, splits, split_stride, Tr, T, h->E, h->K, h->S,
                  mask_off, h->topk_id, h->gate, h->mlogit, h->keep, h->ghat, h->nkeep_tok,
                  h->lreg_tok, 0LL, 0LL, (uint32_t*)nullptr);
}

template <int EPL, typename T>
static cudaError_t launch_small(beam_moe* h, const T* x, int Tr, int T_, int mask_off, int splits,
                                long long split_stride, int gather, cudaStream_t st)
{
    return launch(h, ST_ROUTE_SELECT, route_compact_small_kernel<EPL, T>, dim3(1), dim3(1024), 0, st,
                  (const float*)h->L, h->ldL, splits, split_stride, Tr, T_, h->E, h->K, h->S,
                  mask_off, h->topk_id, h->gate, h->mlogit, h->keep, h->ghat, h->nkeep_tok,
                  h->lreg_tok, h->counts, h->offsets, h->groups, h->n_groups, h->dstats, h->perm,
                  h->inv, x, (T*)h->xperm, h->D, gather, h->tail_cnt, tail_cnt_ints(h->num_sms),
                  h->tile_group);
}

// Output of one expert problem for the combine: `splits` slices `stride` elements apart,
// fp16 (unsplit tensor-core output) or fp32 (split-K partials, GEMV path).
// GEMM1 (+ SwiGLU finish when split) and GEMM2 on the tensor cores, on stream `st`, for the
// routed groups (PROB_ROUTED), the always-on shared group (PROB_SHARED), or both in the same
// launches (PROB_BOTH: the shared tiles first, then the routed ones; used for small batches,
// where one set of launches costs less than two overlapping ones).
enum { PROB_ROUTED = 1, PROB_SHARED = 2, PROB_BOTH = 3 };

template <typename T>
static beam_status_t tc_problem(beam_moe* h, const T* x, int T_, int which, cudaStream_t st,
                                YOut& out_r, YOut& out_s)
{
    const int D = h->D, F = h->F, Fsh = h->Fsh, K = h->K, E = h->E;
    const bool routed = (which & PROB_ROUTED) != 0, shared = (which & PROB_SHARED) != 0;
    int s1 = 1, s2 = 1;
    if (T_ <= kSplitMaxTokens) {
        // a small batch has few tiles: split K so the launch covers every SM
        const long long mts = ceil_div(T_, tc::BM);
        const long long groups = std::min<long long>(E, std::max(1LL, ((long long)T_ * K + 1) / 2));
        const long long t1 = (routed ? mts * groups * (2LL * F / tc::BN) : 0) +
                             (shared ? mts * (2LL * Fsh / tc::BN) : 0);
        const long long t2 = (routed ? mts * groups * (D / tc::BN) : 0) +
                             (shared ? mts * ((long long)D / tc::BN) : 0);
        s1 = choose_splits(h->num_sms, t1);
        s2 = choose_splits(h->num_sms, t2);
        // a gate/up whose tiles alone cover three quarters of the SMs runs whole-K: its SwiGLU
        // epilogue writes H directly, and the split's partial stores and fold cost more than
        // the SMs left idle (Mixtral-like layer, one token: 112 tiles, 53.6 -> 49.7 us)
        if (t1 * 4 >= 3LL * h->num_sms) s1 = 1;
    }
    // per-problem split counts (gate/up: both K = D; down: K = F routed, Fsh shared)
    const int s1n = normalise_splits(s1, D / tc::BK);
    const int s2r = normalise_splits(s2, F / tc::BK);
    const int s2s = shared ? normalise_splits(s2, Fsh / tc::BK) : 1;
    const bool split1 = s1n > 1;
    const bool split2 = (routed && s2r > 1) || (shared && s2s > 1);
    const int rows_sh = shared ? T_ : 0;
    // a shared-only launch is timed under stages of its own
    const bool sh_only = which == PROB_SHARED;
    const int st_gu = sh_only ? ST_TC_SH_GATEUP : ST_TC_GATEUP;
    const int st_dn = sh_only ? ST_TC_SH_DOWN : ST_TC_DOWN;
    const int* ngroups = routed ? h->n_groups : h->zero_int;

    // GEMM1: gate/up, SwiGLU in the epilogue, or f32 partials + the finishing kernel
    tc::TcParams p = split1 ? h->p1s : h->p1;
    if (shared)
        BEAM_TRY(encode_map(h, &p.a_shared, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)T_,
                            (uint64_t)D, tc::BM));
    p.n_groups = ngroups;
    p.shared_rows = rows_sh;
    p.k_splits_routed = p.k_splits_shared = s1n;
    // Kernel form of a whole-K launch.  Routed groups averaging at most 2 * kSwapBox rows
    // (T*K <= 64 E): the swap form, which runs groups of <= 64 rows with the weights as the M
    // operand.  Otherwise, for the routed problem alone and deep enough in K: the tail form,
    // which may cut the tiles of the last, partial wave into K pieces (decided on the device).
    const size_t creg = (size_t)h->num_sms * tc::kEpiWarps;
    const bool small_groups = routed && (long long)T_ * K <= 2LL * tc::kSwapBox * E;
    const bool swap1 = small_groups && !split1;
    const bool swap2 = small_groups && !split2;
    const bool tail1 = which == PROB_ROUTED && !small_groups && !split1 && D / tc::BK >= tc::kTailMinKSteps;
    const bool tail2 = which == PROB_ROUTED && !small_groups && !split2 && F / tc::BK >= tc::kTailMinKSteps;
    p.tail_cnt = tail1 ? h->tail_cnt : nullptr;
    p.tail_ws = tail1 ? h->tail_ws : nullptr;
    if (split1) {
        // f32 partial slices; the warp that completes a tile quadrant's slices adds them in
        // slice order and writes H (SwiGLU), so no finishing launch follows
        p.fold_cnt = h->fold_cnt;
        p.fold_h_routed = static_cast<__half*>(h->hbuf);
        p.fold_h_shared = static_cast<__half*>(h->hsh);
        p.fold_f_routed = F;
        p.fold_f_shared = Fsh;
        BEAM_CUDA(launch(h, st_gu, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 1, tc::MODE_PLAIN>,
                         dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, p));
    } else if (swap1) {
        BEAM_CUDA(launch(h, st_gu, tc::tc_grouped_gemm_kernel<tc::EPI_SWIGLU, 1, tc::MODE_SWAP>,
                         dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, p));
    } else if (tail1) {
        BEAM_CUDA(launch(h, st_gu, tc::tc_grouped_gemm_kernel<tc::EPI_SWIGLU, 1, tc::MODE_TAIL>,
                         dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, p));
    } else {
        BEAM_CUDA(launch(h, st_gu, tc::tc_grouped_gemm_kernel<tc::EPI_SWIGLU, 1, tc::MODE_PLAIN>,
                         dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, p));
    }

    // GEMM2: down projection, fp16 output, or f32 partials added by the combine
    tc::TcParams q = h->p2;
    q.n_groups = ngroups;
    q.shared_rows = rows_sh;
    q.k_splits_routed = s2r;
    q.k_splits_shared = s2s;
    q.tail_cnt = tail2 ? h->tail_cnt + creg : nullptr;
    q.tail_ws = tail2 ? h->tail_ws : nullptr;
    if (split2) {
        q.out_routed = h->ypart;
        q.split_stride_routed = (long long)h->split_rows * K * D;
        q.out_shared = h->ysh_part;
        q.split_stride_shared = (long long)h->split_rows * D;
        if (routed) { out_r.base = h->ypart; out_r.splits = s2r; out_r.stride = q.split_stride_routed; out_r.f16 = false; }
        if (shared) { out_s.base = h->ysh_part; out_s.splits = s2s; out_s.stride = q.split_stride_shared; out_s.f16 = false; }
        BEAM_CUDA(launch(h, st_dn, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 0, tc::MODE_PLAIN>,
                         dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, q));
    } else {
        q.out_routed = h->yperm;
        q.out_shared = h->ysh;
        q.split_stride_routed = q.split_stride_shared = 0;
        if (routed) { out_r.base = h->yperm; out_r.splits = 1; out_r.stride = 0; out_r.f16 = true; }
        if (shared) { out_s.base = h->ysh; out_s.splits = 1; out_s.stride = 0; out_s.f16 = true; }
        if (swap2)
            BEAM_CUDA(launch(h, st_dn, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F16, 0, tc::MODE_SWAP>,
                             dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, q));
        else if (which == PROB_ROUTED && F / tc::BK <= tc::AS_MAX_KSTEPS)
            // short K: the unit's H rows stay in shared memory for all of its N-tiles
            BEAM_CUDA(launch(h, st_dn, tc::tc_down_astat_kernel, dim3(h->num_sms), dim3(tc::kThreads),
                             (size_t)tc::AS_SMEM_BYTES, st, q));
        else if (tail2)
            BEAM_CUDA(launch(h, st_dn, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F16, 0, tc::MODE_TAIL>,
                             dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, q));
        else
            BEAM_CUDA(launch(h, st_dn, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F16, 0, tc::MODE_PLAIN>,
                             dim3(h->num_sms), dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, q));
    }
    return BEAM_OK;
}

template <typename TR, typename TS, typename TO>
static cudaError_t launch_combine_to(beam_moe* h, const YOut& r, const YOut& sh, const float* ghat,
                                     int T_, TO* y, cudaStream_t st)
{
    // few tokens: split each token's columns over several CTAs so the combine spans the SMs;
    // otherwise one CTA per token whose threads take the row's float4 columns in equal passes
    // (D/4 = 384: 192 threads x 2 rather than 256 + 128)
    const int d4 = h->D / 4;
    if (T_ < h->num_sms && (r.splits > 1 || sh.splits > 1) && h->K <= 32 &&
        r.splits <= kCombineMaxSplits && sh.splits <= kCombineMaxSplits) {
        // a small batch with split-K slices: slots and slices read in parallel
        return launch(h, ST_COMBINE, combine_small_kernel<TR, TS, TO>,
                      dim3(T_, ceil_div(d4, kCombineSmallCols)),
                      dim3(kCombineSmallCols, h->K + 1), 0, st,
                      (const TR*)r.base, r.splits, r.stride, (const TS*)sh.base, sh.splits, sh.stride,
                      (const int*)h->inv, ghat, T_, h->K, h->D, y);
    }
    const bool split_cols = T_ < h->num_sms;
    const int passes = ceil_div(d4, 256);
    const int nthr = split_cols ? 256 : std::min(256, ceil_div(ceil_div(d4, passes), 32) * 32);
    const dim3 cgrid(T_, split_cols ? ceil_div(d4, 256) : 1);
    return launch(h, ST_COMBINE, combine_kernel<TR, TS, TO>, cgrid, dim3(nthr), 0, st,
                  (const TR*)r.base, r.splits, r.stride, (const TS*)sh.base, sh.splits, sh.stride,
                  (const int*)h->inv, ghat, T_, h->K, h->D, y);
}

// y: float32 [T][D], or bf16 [T][D] (the same pointer, BEAM_Y_BF16) when y16 is set
template <typename TR, typename TS>
static cudaError_t launch_combine(beam_moe* h, const YOut& r, const YOut& sh, const float* ghat,
                                  int T_, float* y, cudaStream_t st, bool y16 = false)
{
    if (y16)
        return launch_combine_to<TR, TS>(h, r, sh, ghat, T_, reinterpret_cast<__nv_bfloat16*>(y), st);
    return launch_combine_to<TR, TS>(h, r, sh, ghat, T_, y, st);
}

// ep_dispatch: stop after the compaction (expert parallelism, beam_moe_ep_dispatch): the kept
// rows stay in X_perm for the caller's exchange, and the shared experts run on their own (on
// the side stream on the tensor path), their output kept for beam_moe_ep_combine.
template <typename T>
static beam_status_t forward_impl(beam_moe* h, const T* x, int T_, float* y, uint32_t flags,
                                  bool use_tc, cudaStream_t st, const RouteIn* rin = nullptr,
                                  bool ep_dispatch = false)
{
    const int E = h->E, K = h->K, D = h->D;
    const int S = h->S;
    const int Tr = ceil_div(T_, S);
    const int nch = ceil_div(T_, 32);
    const int mask_off = (flags & BEAM_TRAIN) ? 2 : (flags & BEAM_MASK_OFF) ? 1 : 0;

    // 0. shared experts: they need only x, so for larger batches on the tensor path they run on
    // a side stream, concurrently with the router and the compaction, and join before the
    // combine.  Small batches (split K) run them in the routed launches instead: their GEMMs
    // are short, and two streams of them would only add launches that wait for each other.
    BEAM_CUDA(cudaMemsetAsync(&h->dstats->err, 0, 2 * sizeof(int), st));  // err, grid_bar
    YOut ysh_out;
    const bool fork = use_tc && h->Fsh > 0 && (T_ > kSplitMaxTokens || ep_dispatch);
    const bool joint = use_tc && h->Fsh > 0 && !fork;
    if (fork) {
        YOut unused;
        BEAM_CUDA(cudaEventRecord(h->ev_fork, st));
        BEAM_CUDA(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
        BEAM_TRY(tc_problem(h, x, T_, PROB_SHARED, h->side, unused, ysh_out));
        BEAM_CUDA(cudaEventRecord(h->ev_join, h->side));
    }

    // the routing this forward reads: computed below, or given by the caller
    const RouteIn rt = rin ? *rin : own_routing(h);
    h->cur = rt;

    // 1. router logits L = x [W_r | W_m]  (routed rows only: segment leaders when S > 1)
    int lsplits = 1;
    long long lstride = 0;
    if (rin) {
        // the routing is given: no router
    } else if (h->tc_ok && Tr >= kTcRouterMinRows) {
        tc::TcParams& p0 = h->p0;
        BEAM_TRY(encode_map(h, &p0.a_shared, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)Tr,
                            (uint64_t)D, tc::BM, (uint64_t)S * D));
        p0.a_routed = p0.a_shared;
        p0.shared_rows = Tr;
        // few M tiles: split K so the router covers the SMs; route_select adds the slices
        const long long tiles = (long long)ceil_div(Tr, tc::BM) * p0.n_tiles_shared;
        lsplits = normalise_splits(choose_splits(h->num_sms, tiles), D / tc::BK);
        lstride = (long long)Tr * h->ldL;
        p0.k_splits_routed = p0.k_splits_shared = lsplits;
        p0.split_stride_routed = p0.split_stride_shared = lstride;
        BEAM_CUDA(launch(h, ST_TC_ROUTER, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 1, tc::MODE_PLAIN>,
                         dim3((unsigned)std::min<long long>(h->num_sms, tiles * lsplits)),
                         dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, h->p0));
    } else if (Tr > kRouterGemvMaxRows && Tr <= kRouterSmallRows) {
        // a few routed rows: per-chunk slices of D, added in chunk order inside the kernel
        constexpr int DC = kRouterChunkBytes / (int)sizeof(T);
        BEAM_CUDA(launch(h, ST_ROUTER_LOGITS, router_small_kernel<T>,
                         dim3(ceil_div(h->n2E, 8), ceil_div(D, DC)), dim3(256), 0, st, x, S, Tr, D,
                         (const T*)h->wrm, h->n2E, h->ldL, (long long)Tr * h->ldL, h->L, h->rcnt));
    } else {
        BEAM_CUDA(launch_router_gemv<T>(h, x, S, Tr, D, (const T*)h->wrm, h->n2E, h->ldL, h->L, st));
    }
    // 2-3. routing decision and compaction.  Small batches (one 32-token chunk) run them as one
    // single-CTA kernel; larger ones as select -> bit planes -> scan -> scatter + gather.
    cudaError_t e;
    if (!rin && T_ <= kSmallT) {
        const int gather_inline = (long long)T_ * K * D * (long long)sizeof(T) <= kInlineGatherBytes;
        switch ((E + 31) / 32) {
            case 1: e = launch_small<1>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            case 2: e = launch_small<2>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            case 3: e = launch_small<3>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            case 4: e = launch_small<4>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            case 5: e = launch_small<5>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            case 6: e = launch_small<6>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            case 7: e = launch_small<7>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
            default: e = launch_small<8>(h, x, Tr, T_, mask_off, lsplits, lstride, gather_inline, st); break;
        }
        BEAM_CUDA(e);
        if (!gather_inline)
            BEAM_CUDA(launch(h, ST_SCATTER_GATHER, gather_rows_kernel<T>, dim3(h->num_sms * 2),
                             dim3(256), 0, st, (const int*)h->perm, (const int*)(h->offsets + E),
                             K, D, x, (T*)h->xperm));
    } else {
        if (!rin) {
            switch ((E + 31) / 32) {
                case 1: e = launch_select<1>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                case 2: e = launch_select<2>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                case 3: e = launch_select<3>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                case 4: e = launch_select<4>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                case 5: e = launch_select<5>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                case 6: e = launch_select<6>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                case 7: e = launch_select<7>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
                default: e = launch_select<8>(h, Tr, T_, mask_off, lsplits, lstride, st); break;
            }
            BEAM_CUDA(e);
        }
        BEAM_CUDA(launch(h, ST_COMPACT_BITS, compact_bits_kernel, dim3(ceil_div(nch, 8)), dim3(256), 0, st,
                         rt.topk_id, rt.keep, T_, K, E, nch, h->bits));
        BEAM_CUDA(launch(h, ST_COMPACT_SCAN, compact_scan_kernel, dim3(scan_ctas(E, T_)),
                         dim3(32 * kScanWarps), 0, st,
                         (const uint32_t*)h->bits, nch, E, T_, rt.nkeep,
                         rt.lreg, h->counts, h->offsets, h->chunk_base, h->groups,
                         h->n_groups, h->dstats, h->tail_cnt, tail_cnt_ints(h->num_sms), h->tile_group,
                         h->scan_part, &h->dstats->grid_bar));
        BEAM_CUDA(launch(h, ST_SCATTER_GATHER, compact_scatter_gather_kernel<T>,
                         dim3(ceil_div((long long)T_ * K, 8)), dim3(256), 0, st,
                         rt.topk_id, rt.keep, T_, K, D, nch,
                         (const uint32_t*)h->bits, (const int*)h->offsets,
                         (const int*)h->chunk_base, x, h->perm, h->inv, (T*)h->xperm, 1));
    }
    using TH = typename HType<T>::type;
    if (ep_dispatch) {
        // the routed experts run on the ranks that hold them; only the shared ones run here
        if (!use_tc && h->Fsh > 0) {
            StreamArgs a;
            a.xperm = h->xperm; a.x = x; a.wgu = h->wgu; a.wsgu = h->wsgu; a.wd = h->wd; a.wsd = h->wsd;
            a.h = h->hbuf; a.hsh = h->hsh; a.yperm = h->yperm; a.ysh = h->ysh;
            a.groups = h->groups; a.n_groups = h->zero_int; a.err = &h->dstats->err;
            a.D = D; a.F = h->F; a.Fsh = h->Fsh; a.T = T_;
            BEAM_CUDA(launch(h, ST_STREAM_GATEUP, stream_gateup_kernel<T, TH>, dim3(h->num_sms), dim3(kStreamThreads),
                             (size_t)stream_gateup_smem(), st, a));
            BEAM_CUDA(launch(h, ST_STREAM_DOWN, stream_down_kernel<TH>, dim3(h->num_sms), dim3(kStreamThreads),
                             (size_t)stream_down_smem(), st, a));
            ysh_out.base = h->ysh; ysh_out.f16 = false;
        }
        h->ep_T = T_;
        h->ep_ysh = ysh_out;
        h->ep_fork = fork;
        return BEAM_OK;
    }
    // 4. experts: kept groups only (plus the shared group when it is not on the side stream)
    YOut yr;
    if (use_tc) {
        BEAM_TRY(tc_problem(h, x, T_, joint ? PROB_BOTH : PROB_ROUTED, st, yr, ysh_out));
    } else {
        StreamArgs a;
        a.xperm = h->xperm; a.x = x; a.wgu = h->wgu; a.wsgu = h->wsgu; a.wd = h->wd; a.wsd = h->wsd;
        a.h = h->hbuf; a.hsh = h->hsh; a.yperm = h->yperm; a.ysh = h->ysh;
        a.groups = h->groups; a.n_groups = h->n_groups; a.err = &h->dstats->err;
        a.D = D; a.F = h->F; a.Fsh = h->Fsh; a.T = T_;
        const int grid = h->num_sms;  // one CTA per SM (shared-memory rings)
        BEAM_CUDA(launch(h, ST_STREAM_GATEUP, stream_gateup_kernel<T, TH>, dim3(grid), dim3(kStreamThreads),
                         (size_t)stream_gateup_smem(), st, a));
        BEAM_CUDA(launch(h, ST_STREAM_DOWN, stream_down_kernel<TH>, dim3(grid), dim3(kStreamThreads),
                         (size_t)stream_down_smem(), st, a));
        yr.base = h->yperm; yr.f16 = false;
        if (h->Fsh) { ysh_out.base = h->ysh; ysh_out.f16 = false; }
    }
    h->last_yr = yr;
    // 5. fixed-order combine (after the side stream joins)
    if (fork) BEAM_CUDA(cudaStreamWaitEvent(st, h->ev_join, 0));
    if (!h->Fsh) ysh_out.f16 = yr.f16;  // no shared term: only its (unused) type must match
    cudaError_t ce;
    const bool y16 = (flags & BEAM_Y_BF16) != 0;
    if (yr.f16 && ysh_out.f16) ce = launch_combine<__half, __half>(h, yr, ysh_out, rt.ghat, T_, y, st, y16);
    else if (yr.f16) ce = launch_combine<__half, float>(h, yr, ysh_out, rt.ghat, T_, y, st, y16);
    else if (ysh_out.f16) ce = launch_combine<float, __half>(h, yr, ysh_out, rt.ghat, T_, y, st, y16);
    else ce = launch_combine<float, float>(h, yr, ysh_out, rt.ghat, T_, y, st, y16);
    BEAM_CUDA(ce);
    return BEAM_OK;
}

// ---------------------------------------------------------------- pipelined host calls
// Statistics of a host call run as several chunks: after each chunk's forward, mode 0 (the
// first chunk) copies its statistics and per-expert counts into the accumulator, mode 1 adds
// them (integer sums, the L_reg sum in chunk order; error bits OR-ed); mode 2 writes the
// accumulated values back as the statistics of the whole call (the active experts recounted
// from the summed counts).  One block.
__global__ void __launch_bounds__(256)
stats_accumulate_kernel(DevStats* __restrict__ st, const int* __restrict__ counts,
                        DevStats* __restrict__ acc, int* __restrict__ acc_counts, int E, int mode)
{
    pdl_wait();
    __shared__ int s_act;
    if (threadIdx.x == 0) s_act = 0;
    __syncthreads();
    int act = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        if (mode == 0) acc_counts[e] = counts[e];
        else if (mode == 1) acc_counts[e] += counts[e];
        else { const_cast<int*>(counts)[e] = acc_counts[e]; act += acc_counts[e] > 0; }
    }
    if (mode == 2) atomicAdd(&s_act, act);   // an integer count: order-free
    __syncthreads();
    if (threadIdx.x == 0) {
        if (mode == 0) {
            *acc = *st;
        } else if (mode == 1) {
            acc->keep_sum += st->keep_sum;
            acc->lreg_sum += st->lreg_sum;
            acc->n_all_masked += st->n_all_masked;
            acc->n_kept += st->n_kept;
            acc->tokens += st->tokens;
            acc->err |= st->err;
        } else {
            st->keep_sum = acc->keep_sum;
            st->lreg_sum = acc->lreg_sum;
            st->n_all_masked = acc->n_all_masked;
            st->n_kept = acc->n_kept;
            st->tokens = acc->tokens;
            st->err |= acc->err;
            st->n_active = s_act;
        }
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- fused decode
// Whether a forward runs as the single fused decode launch.
static bool fused_eligible(const beam_moe* h, int T, uint32_t flags, bool use_tc)
{
    return h->fused_ok && use_tc && T >= 1 && T <= kSmallT && (flags & BEAM_FUSED_DECODE) &&
           h->cfg.dtype == BEAM_DTYPE_BF16;
}

// The whole forward of a batch of 1..kSmallT tokens as one cooperative launch (see
// decode_fused.cuh).  The split counts are the ones the separate launches would use, with the
// shared experts in the same GEMMs; both GEMMs always store f32 partial slices.
static beam_status_t forward_fused(beam_moe* h, const __nv_bfloat16* x, int T_, float* y,
                                   uint32_t flags, cudaStream_t st)
{
    const int D = h->D, F = h->F, Fsh = h->Fsh, K = h->K, E = h->E, S = h->S;
    const int Tr = ceil_div(T_, S);
    h->cur = own_routing(h);
    BEAM_CUDA(cudaMemsetAsync(&h->dstats->err, 0, 2 * sizeof(int), st));  // err, grid_bar
    const long long mts = ceil_div(T_, tc::BM);
    const long long groups = std::min<long long>(E, std::max(1LL, ((long long)T_ * K + 1) / 2));
    const long long t1 = mts * groups * (2LL * F / tc::BN) + (Fsh ? mts * (2LL * Fsh / tc::BN) : 0);
    const long long t2 = mts * groups * (D / tc::BN) + (Fsh ? mts * ((long long)D / tc::BN) : 0);
    const int s1 = normalise_splits(choose_splits(h->num_sms, t1), D / tc::BK);
    const int s2c = choose_splits(h->num_sms, t2);
    const int s2r = normalise_splits(s2c, F / tc::BK);
    const int s2s = Fsh ? normalise_splits(s2c, Fsh / tc::BK) : 1;

    FusedDecodeParams P;
    memset(&P, 0, sizeof P);
    P.g1 = h->p1s;
    if (Fsh)
        BEAM_TRY(encode_map(h, &P.g1.a_shared, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)T_,
                            (uint64_t)D, tc::BM));
    P.g1.n_groups = h->n_groups;
    P.g1.shared_rows = Fsh ? T_ : 0;
    P.g1.k_splits_routed = P.g1.k_splits_shared = s1;
    P.g1.tail_cnt = nullptr;
    P.g1.tail_ws = nullptr;
    P.g2 = h->p2;
    P.g2.n_groups = h->n_groups;
    P.g2.shared_rows = Fsh ? T_ : 0;
    P.g2.k_splits_routed = s2r;
    P.g2.k_splits_shared = s2s;
    P.g2.tail_cnt = nullptr;
    P.g2.tail_ws = nullptr;
    P.g2.out_routed = h->ypart;
    P.g2.split_stride_routed = (long long)h->split_rows * K * D;
    P.g2.out_shared = h->ysh_part;
    P.g2.split_stride_shared = (long long)h->split_rows * D;
    P.x = x;
    P.wrm = static_cast<const __nv_bfloat16*>(h->wrm);
    P.L = h->L;
    P.lchunk = 256 * ceil_div(D, 256 * kMaxSplits);   // at most kMaxSplits slices of D
    P.lchunks = ceil_div(D, P.lchunk);
    P.T = T_; P.Tr = Tr; P.seg = S; P.D = D; P.E = E; P.K = K; P.n2E = h->n2E;
    P.mask_off = (flags & BEAM_MASK_OFF) ? 1 : 0;
    P.topk_id = h->topk_id; P.gate = h->gate; P.mlogit = h->mlogit; P.keep = h->keep;
    P.ghat = h->ghat; P.nkeep_tok = h->nkeep_tok; P.lreg_tok = h->lreg_tok;
    P.counts = h->counts; P.offsets = h->offsets; P.groups = h->groups; P.n_groups = h->n_groups;
    P.stats = h->dstats; P.perm = h->perm; P.inv = h->inv; P.tile_group = h->tile_group;
    P.xperm = static_cast<__nv_bfloat16*>(h->xperm);
    P.F = F; P.Fsh = Fsh;
    P.h = static_cast<__half*>(h->hbuf); P.hsh = static_cast<__half*>(h->hsh);
    P.y = y;
    P.grid_bar = &h->dstats->grid_bar;
    P.err = &h->dstats->err;
    const dim3 grid(h->num_sms), block(tc::kThreads);
    const size_t smem = tc::SMEM_BYTES;
    cudaError_t e;
    switch ((E + 31) / 32) {
        case 1: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<1>, grid, block, smem, st, P); break;
        case 2: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<2>, grid, block, smem, st, P); break;
        case 3: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<3>, grid, block, smem, st, P); break;
        case 4: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<4>, grid, block, smem, st, P); break;
        case 5: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<5>, grid, block, smem, st, P); break;
        case 6: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<6>, grid, block, smem, st, P); break;
        case 7: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<7>, grid, block, smem, st, P); break;
        default: e = launch_ex(h, ST_FUSED_DECODE, true, fused_decode_kernel<8>, grid, block, smem, st, P); break;
    }
    BEAM_CUDA(e);
    return BEAM_OK;
}

// ---------------------------------------------------------------- routing without allocation
// Scratch of beam_moe_route_noalloc: a fixed array in the library's own device memory, so the
// call needs no cudaMalloc.  Every GPU that loads the library holds it until the process
// exits.  Layout per call: logits [Tr][2E] f32 (256-byte aligned), then per-token kept counts
// [T] i32 and L_reg terms [T] f32.  Nothing in it has to start at zero: each element the
// kernels read is written earlier in the same call.  Calls share it, so calls whose work
// overlaps on the GPU (other streams, other threads) race on it.
static __device__ __align__(256) unsigned char g_route_scratch[BEAM_ROUTE_NOALLOC_SCRATCH_BYTES];

static std::mutex g_route_scratch_mu;
static void* g_route_scratch_dev[256] = {};  // device address of the array, per device

// Device address of the scratch array on the current device (the host-side name of a
// __device__ array is not a device address).  It is looked up with cudaGetSymbolAddress on the
// first call on each device, and again on every later call made while `st` is not capturing,
// so a context that was reset and reloaded the module gets the new address; during a stream
// capture (where the lookup could have to load the module) the cached address is used.
static beam_status_t route_scratch_address(void** out, cudaStream_t st)
{
    int dev = -1;
    BEAM_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 256) return fail(BEAM_ERR_UNSUPPORTED, "device index %d out of range", dev);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    BEAM_CUDA(cudaStreamIsCapturing(st, &cs));
    std::lock_guard<std::mutex> lock(g_route_scratch_mu);
    if (!g_route_scratch_dev[dev] || cs == cudaStreamCaptureStatusNone) {
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess || !p)
            return fail(BEAM_ERR_CUDA, "cudaGetSymbolAddress of the routing scratch failed: %s",
                        cudaGetErrorString(e));
        g_route_scratch_dev[dev] = p;
    }
    *out = g_route_scratch_dev[dev];
    return BEAM_OK;
}

template <int EPL>
static cudaError_t launch_select_into(beam_moe* h, const float* L, int Tr, int T, int mask_off,
                                      int* topk_id, float* gate, float* mlogit, uint8_t* keep,
                                      float* ghat, int* nkeep_tok, float* lreg_tok,
                                      cudaStream_t st)
{
    // launched without the handle (nullptr): the call leaves its launch count and profile alone
    return launch(nullptr, ST_ROUTE_SELECT, route_select_kernel<EPL>, dim3(ceil_div(Tr, 8)), dim3(256),
                  0, st, L, h->n2E, 1, 0LL, Tr, T, h->E, h->K, h->S, mask_off, topk_id, gate,
                  mlogit, keep, ghat, nkeep_tok, lreg_tok, 0LL, 0LL, (uint32_t*)nullptr);
}

template <typename T>
static beam_status_t route_noalloc_impl(beam_moe* h, const T* x, int T_, int32_t* topk_id,
                                        float* gate, float* mlogit, uint8_t* keep, float* ghat,
                                        int mask_off, unsigned char* scratch, cudaStream_t st)
{
    const int S = h->S;
    const int Tr = ceil_div(T_, S);
    const size_t l_bytes = ((size_t)Tr * h->n2E * sizeof(float) + 255) & ~(size_t)255;
    float* L = reinterpret_cast<float*>(scratch);
    int* nkeep = reinterpret_cast<int*>(scratch + l_bytes);
    float* lreg = reinterpret_cast<float*>(scratch + l_bytes + (size_t)T_ * sizeof(int));
    BEAM_CUDA(launch_router_gemv<T>(nullptr, x, S, Tr, h->D, (const T*)h->wrm, h->n2E, h->n2E, L, st));
    cudaError_t e;
    switch ((h->E + 31) / 32) {
        case 1: e = launch_select_into<1>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        case 2: e = launch_select_into<2>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        case 3: e = launch_select_into<3>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        case 4: e = launch_select_into<4>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        case 5: e = launch_select_into<5>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        case 6: e = launch_select_into<6>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        case 7: e = launch_select_into<7>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
        default: e = launch_select_into<8>(h, L, Tr, T_, mask_off, topk_id, gate, mlogit, keep, ghat, nkeep, lreg, st); break;
    }
    BEAM_CUDA(e);
    return BEAM_OK;
}

// ---------------------------------------------------------------- cross-layer routing
// The mask generator ("Stepped MoE: Segment-Level Routing with Configurable Inference
// Complexity", core method): the logits of every layer from one GEMM over the segment
// leaders' rows of z, G = z_lead [W_r^(1) | W_m^(1) | ... | W_r^(L) | W_m^(L)], then one warp per
// (segment, layer) takes BEAM's Top-K / softmax / mask decision (route_select_kernel with a
// layer grid dimension) and marks the layer's kept experts.
struct beam_gen {
    beam_moe core;          // device plumbing shared with the layer handle (allocations, tensor
                            // maps, launches, error word); its expert fields stay unused
    int L = 0;
    int nlog = 0;           // L * 2E logit columns
    int ldG = 0;            // row pitch of G: nlog, padded to the tile width on the tensor path
    void* wgen = nullptr;   // [ldG][D] repacked generator weights
    float* G = nullptr;     // logits [splits][Tr][ldG] (K-split slices when the GEMM splits)
};

static beam_status_t gen_validate(const beam_gen_config_t* c)
{
    if (!c) return fail(BEAM_ERR_INVALID_ARG, "cfg is NULL");
    if (c->dtype != BEAM_DTYPE_F32 && c->dtype != BEAM_DTYPE_BF16)
        return fail(BEAM_ERR_INVALID_ARG, "dtype must be BEAM_DTYPE_F32 or BEAM_DTYPE_BF16");
    const int dmul = c->dtype == BEAM_DTYPE_BF16 ? 64 : 4;
    const int dmax = c->dtype == BEAM_DTYPE_BF16 ? 8192 : 4096;
    if (c->d_model <= 0 || c->d_model % dmul || c->d_model > dmax)
        return fail(BEAM_ERR_INVALID_ARG, "d_model=%d must be a positive multiple of %d, <= %d",
                    c->d_model, dmul, dmax);
    if (c->n_layers < 1 || c->n_layers > 512)
        return fail(BEAM_ERR_INVALID_ARG, "n_layers=%d must be in [1, 512]", c->n_layers);
    if (c->n_experts < 1 || c->n_experts > kMaxE)
        return fail(BEAM_ERR_INVALID_ARG, "n_experts=%d must be in [1, %d]", c->n_experts, kMaxE);
    if (c->top_k < 1 || c->top_k > std::min(c->n_experts, 32))
        return fail(BEAM_ERR_INVALID_ARG, "top_k=%d must be in [1, min(E, 32)]", c->top_k);
    if (c->segment_len < 0 || c->segment_len > 65536)
        return fail(BEAM_ERR_INVALID_ARG, "segment_len=%d out of range", c->segment_len);
    if (c->max_tokens < 1 || c->max_tokens > 65536)
        return fail(BEAM_ERR_INVALID_ARG, "max_tokens=%d must be in [1, 65536]", c->max_tokens);
    return BEAM_OK;
}

static beam_status_t gen_create_impl(const beam_gen_config_t* c, const void* wr, const void* wm,
                                     cudaStream_t st, beam_gen* g)
{
    beam_moe* h = &g->core;
    memset(&h->cfg, 0, sizeof h->cfg);
    h->cfg.d_model = c->d_model; h->cfg.n_experts = c->n_experts; h->cfg.top_k = c->top_k;
    h->cfg.dtype = c->dtype; h->cfg.segment_len = c->segment_len; h->cfg.max_tokens = c->max_tokens;
    h->D = c->d_model; h->E = c->n_experts; h->K = c->top_k; h->F = h->Fsh = 0;
    h->Tmax = c->max_tokens;
    h->S = c->segment_len > 1 ? c->segment_len : 1;
    h->n2E = 2 * h->E;
    h->esz = h->hsz = c->dtype == BEAM_DTYPE_BF16 ? 2 : 4;
    int dev = 0;
    BEAM_CUDA(cudaGetDevice(&dev));
    BEAM_CUDA(cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev));
    g->L = c->n_layers;
    g->nlog = g->L * h->n2E;
    // the tensor-core GEMM under the same condition as a layer's router
    const bool tc = c->dtype == BEAM_DTYPE_BF16 && h->D % tc::BN == 0;
    g->ldG = tc ? ceil_div(g->nlog, tc::BN) * tc::BN : g->nlog;
    const int Trmax = ceil_div(h->Tmax, h->S);
    // room for the largest K-split the GEMM takes: the split count depends on the 128-row
    // tile count, so the largest row count of each tile count bounds it
    size_t gfloats = (size_t)Trmax * g->ldG;
    if (tc) {
        for (int mt = 1; mt <= ceil_div(Trmax, tc::BM); ++mt) {
            const int rows = std::min(mt * tc::BM, Trmax);
            if (rows < kTcRouterMinRows) continue;
            const int s = normalise_splits(choose_splits(h->num_sms, (long long)mt * (g->ldG / tc::BN)),
                                           h->D / tc::BK);
            gfloats = std::max(gfloats, (size_t)s * rows * g->ldG);
        }
    }
    // and for the D-chunk slices of the small-batch router (at most kRouterSmallRows rows)
    {
        const int rows = std::min(Trmax, kRouterSmallRows);
        const int chunks = ceil_div((long long)h->D * h->esz, kRouterChunkBytes);
        gfloats = std::max(gfloats, (size_t)chunks * rows * g->ldG);
    }
    BEAM_TRY(dalloc(h, &g->wgen, (size_t)g->ldG * h->D * h->esz));
    BEAM_TRY(dalloc(h, &g->G, gfloats * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->rcnt, (size_t)ceil_div(g->ldG, 8) * sizeof(unsigned)));
    BEAM_CUDA(cudaMemsetAsync(h->rcnt, 0, (size_t)ceil_div(g->ldG, 8) * sizeof(unsigned), st));
    BEAM_TRY(dalloc(h, &h->zero_int, 2 * sizeof(int)));
    BEAM_TRY(dalloc(h, &h->groups, sizeof(Group)));
    BEAM_TRY(dalloc(h, &h->dstats, sizeof(DevStats)));
    BEAM_CUDA(cudaMemsetAsync(h->dstats, 0, sizeof(DevStats), st));
    BEAM_CUDA(cudaMemsetAsync(h->zero_int, 0, 2 * sizeof(int), st));
    BEAM_CUDA(cudaEventCreateWithFlags(&h->done, cudaEventDisableTiming));
    if (c->dtype == BEAM_DTYPE_BF16)
        repack_router_kernel<__nv_bfloat16><<<2048, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(wr), static_cast<const __nv_bfloat16*>(wm), h->D,
            h->E, g->L, g->ldG, static_cast<__nv_bfloat16*>(g->wgen));
    else
        repack_router_kernel<float><<<2048, 256, 0, st>>>(
            static_cast<const float*>(wr), static_cast<const float*>(wm), h->D, h->E, g->L,
            g->ldG, static_cast<float*>(g->wgen));
    BEAM_CUDA(cudaGetLastError());
    if (tc) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        BEAM_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
        if (!fn || q != cudaDriverEntryPointSuccess)
            return fail(BEAM_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        h->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        BEAM_CUDA(cudaFuncSetAttribute(tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 1, tc::MODE_PLAIN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES));
        // one dense problem: G [Tr][ldG] = z_lead [Tr][D] . Wgen [ldG][D]^T
        tc::TcParams& r = h->p0;
        memset(&r, 0, sizeof r);
        BEAM_TRY(encode_map(h, &r.b_shared, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g->wgen,
                            (uint64_t)g->ldG, (uint64_t)h->D, tc::BN));
        r.b_routed = r.b_shared;
        r.groups = h->groups;
        r.n_groups = h->zero_int;          // no routed groups
        r.out_routed = r.out_shared = g->G;
        r.ld_routed = r.ld_shared = g->ldG;
        r.n_tiles_routed = r.n_tiles_shared = g->ldG / tc::BN;
        r.k_steps_routed = r.k_steps_shared = h->D / tc::BK;
        r.k_splits_routed = r.k_splits_shared = 1;
        r.store_cols = g->nlog;            // columns past L*2E are padding nobody reads
        r.err = &h->dstats->err;
        h->tc_ok = true;
    }
    BEAM_CUDA(cudaStreamSynchronize(st));
    return BEAM_OK;
}

template <int EPL>
static cudaError_t launch_select_layers(beam_gen* g, const float* G, int splits, long long sstride,
                                        int Tr, int T, int mask_off, const beam_routing_t* o,
                                        cudaStream_t st)
{
    beam_moe* h = &g->core;
    return launch(h, ST_ROUTE_SELECT, route_select_kernel<EPL>, dim3(ceil_div(Tr, 8), g->L),
                  dim3(256), 0, st, G, g->ldG, splits, sstride, Tr, T, h->E, h->K, h->S, mask_off,
                  o->topk_id, o->gate, o->mask_logit, o->keep, o->ghat, o->n_keep, o->lreg,
                  (long long)T * h->K, (long long)T, o->active);
}

template <typename T>
static beam_status_t gen_route_impl(beam_gen* g, const T* z, int T_, const beam_routing_t* o,
                                    int mask_off, cudaStream_t st)
{
    beam_moe* h = &g->core;
    const int S = h->S, Tr = ceil_div(T_, S), E = h->E, D = h->D;
    BEAM_CUDA(cudaMemsetAsync(&h->dstats->err, 0, 2 * sizeof(int), st));
    if (o->active)
        BEAM_CUDA(cudaMemsetAsync(o->active, 0, (size_t)g->L * ((E + 31) / 32) * sizeof(uint32_t), st));
    int splits = 1;
    long long sstride = 0;
    if (h->tc_ok && Tr >= kTcRouterMinRows) {
        tc::TcParams& p = h->p0;
        BEAM_TRY(encode_map(h, &p.a_shared, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, z, (uint64_t)Tr,
                            (uint64_t)D, tc::BM, (uint64_t)S * D));
        p.a_routed = p.a_shared;
        p.shared_rows = Tr;
        const long long tiles = (long long)ceil_div(Tr, tc::BM) * p.n_tiles_shared;
        splits = normalise_splits(choose_splits(h->num_sms, tiles), D / tc::BK);
        sstride = (long long)Tr * g->ldG;
        p.k_splits_routed = p.k_splits_shared = splits;
        p.split_stride_routed = p.split_stride_shared = sstride;
        BEAM_CUDA(launch(h, ST_TC_ROUTER, tc::tc_grouped_gemm_kernel<tc::EPI_STORE_F32, 1, tc::MODE_PLAIN>,
                         dim3((unsigned)std::min<long long>(h->num_sms, tiles * splits)),
                         dim3(tc::kThreads), (size_t)tc::SMEM_BYTES, st, h->p0));
    } else if (Tr > kRouterGemvMaxRows && Tr <= kRouterSmallRows) {
        // the layer's small-batch router, so that a one-layer generator and its layer compute
        // the same bits
        constexpr int DC = kRouterChunkBytes / (int)sizeof(T);
        BEAM_CUDA(launch(h, ST_ROUTER_LOGITS, router_small_kernel<T>,
                         dim3(ceil_div(g->nlog, 8), ceil_div(D, DC)), dim3(256), 0, st, z, S, Tr, D,
                         (const T*)g->wgen, g->nlog, g->ldG, (long long)Tr * g->ldG, g->G, h->rcnt));
    } else {
        BEAM_CUDA(launch_router_gemv<T>(h, z, S, Tr, D, (const T*)g->wgen, g->nlog, g->ldG, g->G, st));
    }
    cudaError_t e;
    switch ((E + 31) / 32) {
        case 1: e = launch_select_layers<1>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        case 2: e = launch_select_layers<2>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        case 3: e = launch_select_layers<3>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        case 4: e = launch_select_layers<4>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        case 5: e = launch_select_layers<5>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        case 6: e = launch_select_layers<6>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        case 7: e = launch_select_layers<7>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
        default: e = launch_select_layers<8>(g, g->G, splits, sstride, Tr, T_, mask_off, o, st); break;
    }
    BEAM_CUDA(e);
    return BEAM_OK;
}

// ---------------------------------------------------------------- C ABI
// ---------------------------------------------------------------- training: routing gradient
// Pairs per unit of the dW pass: about 16 warps per SM over all column chunks, at least 32.
// Then ceil(pairs / R) <= 16 * num_sms / chunks, so the units (at most that plus one partial
// unit per expert) fit the handle's 16 * num_sms / chunks + E + 1 partial column pairs.
static int dw_rows_per_unit(const beam_moe* h, int T_)
{
    const long long pairs = (long long)T_ * h->K;
    const long long warps = 16LL * h->num_sms;
    long long r = (pairs * h->dw_chunks + warps - 1) / warps;
    r = ((r + 31) / 32) * 32;
    return (int)std::max<long long>(32, r);
}

template <typename TY, typename TX>
static cudaError_t launch_route_grad(beam_moe* h, const float* dy, int T_, float reg, float* dx,
                                     float* dgl, float* dml, float* dgh, cudaStream_t st)
{
    const YOut& yr = h->last_yr;
    const int S = h->S, K = h->K;
    // one CTA per routed row (a token, or a segment)
    const unsigned grid = (unsigned)ceil_div(T_, S);
#define BEAM_RG(KM)                                                                              \
    launch(h, ST_ROUTE_GRAD, route_grad_kernel<TY, TX, KM>, dim3(grid), dim3(kGradThreads), 0, st, \
           (const TY*)yr.base, yr.splits, yr.stride, (const int*)h->inv, (const int*)h->topk_id, \
           (const float*)h->gate, (const float*)h->mlogit, dy, (const TX*)h->wrm, T_, K, h->E,  \
           h->D, S, reg, dgh, dgl, dml, h->pair_grad, dx)
    if (K <= 2) return BEAM_RG(2);
    if (K <= 4) return BEAM_RG(4);
    if (K <= 8) return BEAM_RG(8);
    if (K <= 16) return BEAM_RG(16);
    return BEAM_RG(32);
#undef BEAM_RG
}

template <typename TX>
static beam_status_t backward_impl(beam_moe* h, const TX* x, const float* dy, int T_,
                                   float reg_scale, float* dwr, float* dwm, float* dx, float* dgl,
                                   float* dml, float* dgh, cudaStream_t st)
{
    const int K = h->K, E = h->E, D = h->D;
    // dL/dm_hat of every (token, slot) from L_reg = mean over tokens of (1/K) sum_TK m_hat
    const float reg = (float)((double)reg_scale / ((double)T_ * (double)K));
    // 1. per routed row: the K dots with dy, the logit gradients, dx
    const cudaError_t e1 = h->last_yr.f16
        ? launch_route_grad<__half, TX>(h, dy, T_, reg, dx, dgl, dml, dgh, st)
        : launch_route_grad<float, TX>(h, dy, T_, reg, dx, dgl, dml, dgh, st);
    BEAM_CUDA(e1);
    // 2. dW: one warp per (unit of one expert's pairs, column chunk), then the expert's
    // partials in unit order
    const int R = dw_rows_per_unit(h, T_);
    const long long items = ((long long)ceil_div((long long)T_ * K, R) + E) * h->dw_chunks;
    BEAM_CUDA(launch(h, ST_ROUTE_DW, route_dw_kernel<TX>, dim3((unsigned)ceil_div(items, 8)),
                     dim3(256), 0, st, (const int*)h->offsets, (const int*)h->perm,
                     (const float2*)h->pair_grad, x, K, E, D, h->S, R, h->dw_chunks, h->dw_part,
                     h->dw_cnt, dwr, dwm));
    return BEAM_OK;
}

// ---------------------------------------------------------------- expert parallelism
// Routing of the rows an expert rank received: source s sent recv_counts[s][e] rows of its local
// expert e, source-major and expert-minor (the order of the sender's X_perm), so row j belongs
// to the (s, e) block whose range holds j.  Each row becomes a one-slot "token" routed to that
// expert with gate 1 (topk_id = e, keep = 1, g_hat = 1, n_keep = 1, lreg = 0), which a routed
// forward of the expert handle (K = 1) turns into the expert's output row: the compaction groups
// the rows by expert, the grouped GEMMs run, and the combine writes 1 * Y row back in place.
// Every block scans the nblk <= kEpMaxBlocks counts into shared memory (256 threads, each a run
// of consecutive counts, then a scan of the 256 run totals), then finds each row's block by a
// binary search.
constexpr int kEpMaxBlocks = 4096;

__global__ void __launch_bounds__(256)
ep_recv_routing_kernel(const int* __restrict__ recv_counts, int nblk, int El, int n_rows,
                       int* __restrict__ topk_id, uint8_t* __restrict__ keep,
                       float* __restrict__ ghat, int* __restrict__ nkeep, float* __restrict__ lreg)
{
    __shared__ int s_off[kEpMaxBlocks + 1];
    __shared__ int s_run[256];
    pdl_wait();
    const int tid = threadIdx.x;
    const int per = (nblk + 255) / 256;
    const int b0 = tid * per, b1 = min(nblk, b0 + per);
    int run = 0;
    for (int b = b0; b < b1; ++b) run += recv_counts[b];
    s_run[tid] = run;
    __syncthreads();
    if (tid < 32) {
        // exclusive scan of the 256 run totals by one warp, 8 per lane
        int v[8], sum = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { v[i] = s_run[tid * 8 + i]; sum += v[i]; }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (tid >= o) incl += n;
        }
        int ex = incl - sum;
#pragma unroll
        for (int i = 0; i < 8; ++i) { s_run[tid * 8 + i] = ex; ex += v[i]; }
    }
    __syncthreads();
    int off = s_run[tid];
    for (int b = b0; b < b1; ++b) { s_off[b] = off; off += recv_counts[b]; }
    if (b1 == nblk && b0 < b1) s_off[nblk] = off;
    if (nblk == 0 && tid == 0) s_off[0] = 0;
    __syncthreads();
    for (int j = blockIdx.x * blockDim.x + tid; j < n_rows; j += gridDim.x * blockDim.x) {
        int lo = 0, hi = nblk;   // s_off[lo] <= j < s_off[hi] for every j below the total
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_off[mid] <= j) lo = mid; else hi = mid;
        }
        topk_id[j] = lo % El;
        keep[j] = 1;
        ghat[j] = 1.f;
        nkeep[j] = 1;
        lreg[j] = 0.f;
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- SoftTopK
template <int EPL>
static cudaError_t launch_softtopk_fwd(const float* r, int T, int E, int K, float tau, float* y,
                                       uint8_t* mask, float* nu, cudaStream_t st)
{
    return launch(nullptr, 0, softtopk_fwd_kernel<EPL>, dim3(ceil_div(T, 8)), dim3(256), 0, st,
                  r, T, E, K, tau, y, mask, nu);
}

template <int EPL>
static cudaError_t launch_softtopk_bwd(const float* y, const float* dy, int T, int E, float tau,
                                       float* dr, cudaStream_t st)
{
    return launch(nullptr, 0, softtopk_bwd_kernel<EPL>, dim3(ceil_div(T, 8)), dim3(256), 0, st,
                  y, dy, T, E, tau, dr);
}

static beam_status_t softtopk_check(int32_t T, int32_t E, float tau, const void* a, const void* b,
                                    const void* c)
{
    if (T < 0) return fail(BEAM_ERR_INVALID_ARG, "T=%d is negative", T);
    if (E < 1 || E > kSoftTopkMaxE)
        return fail(BEAM_ERR_INVALID_ARG, "E=%d must be in [1, %d]", E, kSoftTopkMaxE);
    if (!(tau > 0.f) || !std::isfinite(tau))
        return fail(BEAM_ERR_INVALID_ARG, "tau must be a positive finite number");
    if ((long long)T * E > (1LL << 31) - 1)
        return fail(BEAM_ERR_INVALID_ARG, "T*E=%lld is too large", (long long)T * E);
    if (T > 0 && (!a || !b || !c)) return fail(BEAM_ERR_INVALID_ARG, "a required pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) |
         reinterpret_cast<uintptr_t>(c)) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "the float arrays must be 4-byte aligned");
    return BEAM_OK;
}

// A pipelined host call: the batch as C chunks of whole segments.  Chunk c's x copy runs on
// copy_in, its forward on `st` once the copy has landed, and its y copy on copy_out once the
// forward is done, so the copies of one chunk overlap the forwards of its neighbours.  The
// routing arrays of chunk c are written at the chunk's offset (the handle's pointers are
// shifted for the call), so the routing of every token is kept; the statistics are added up
// over the chunks on the device.
constexpr int kHostMaxChunks = 4;
constexpr int kHostPipelineMinTokens = 1024;   // smaller batches are copied and run whole
// Chunk plan of a pipelined host call, in quarters of the batch: the first chunk's copy in
// and the last chunk's copy out are the only copies nothing overlaps, so those two chunks are
// small; the middle is one chunk, because every chunk reads all the kept experts' weights.
// (Relative sizes; batches below 2048 tokens run as two halves.)
constexpr int kHostPlan[] = {1, 2, 1};
static_assert(sizeof(kHostPlan) / sizeof(kHostPlan[0]) <= kHostMaxChunks, "one event pair per chunk");

// Token counts of the chunks of a pipelined host call (whole segments of `align` tokens,
// none empty).
static int host_chunk_plan(int T_, int align, int* sizes)
{
    const int units = ceil_div(T_, align);
    int n = 0;
    if (T_ < 2048 || units < 4) {
        const int a = ceil_div(units, 2) * align;
        sizes[n++] = std::min(a, T_);
        if (T_ > a) sizes[n++] = T_ - a;
        return n;
    }
    int q = 0;
    for (int w : kHostPlan) q += w;
    int done = 0, acc = 0;
    for (size_t i = 0; i < sizeof(kHostPlan) / sizeof(kHostPlan[0]); ++i) {
        acc += kHostPlan[i];
        const int end = (i + 1 == sizeof(kHostPlan) / sizeof(kHostPlan[0]))
                            ? T_ : std::min(T_, (int)((long long)units * acc / q) * align);
        if (end > done) sizes[n++] = end - done;
        done = std::max(done, end);
    }
    return n;
}

// Host copy of n rows of y at row offset `off` from the device staging buffer: float32, or
// (y16) the bf16 rows the combine wrote under BEAM_Y_BF16.
static cudaError_t copy_y_out(beam_moe* h, void* y_host, long long off, int n, bool y16,
                              cudaStream_t copy_st)
{
    const size_t e0 = (size_t)off * h->D, ne = (size_t)n * h->D;
    if (!y16)
        return cudaMemcpyAsync(static_cast<float*>(y_host) + e0, h->y_stage + e0, ne * sizeof(float),
                               cudaMemcpyDeviceToHost, copy_st);
    return cudaMemcpyAsync(static_cast<__nv_bfloat16*>(y_host) + e0, h->y16_stage + e0,
                           ne * sizeof(__nv_bfloat16), cudaMemcpyDeviceToHost, copy_st);
}

// The device y of a host call: the float32 staging rows, or the bf16 ones (written through the
// same float* argument with BEAM_Y_BF16 set).
static float* host_y_dev(beam_moe* h, float* y32, __nv_bfloat16* y16, bool bf16)
{
    return bf16 ? reinterpret_cast<float*>(y16) : y32;
}

template <typename T>
static beam_status_t forward_host_pipelined(beam_moe* h, const T* x_host, int T_, void* y_host,
                                            uint32_t flags, cudaStream_t st)
{
    const int D = h->D, K = h->K, E = h->E;
    const int align = h->S > 1 ? h->S : 32;
    int sizes[kHostMaxChunks];
    const int C = host_chunk_plan(T_, align, sizes);
    const bool use_tc = (flags & BEAM_PATH_TENSOR) ? true : (flags & BEAM_PATH_STREAM) ? false
                                                                                        : h->tc_ok;
    const bool y16 = (flags & BEAM_HOST_Y_BF16) != 0;
    const uint32_t fflags = (flags & ~(BEAM_HOST_PIPELINE | BEAM_NO_GRAPH | BEAM_HOST_Y_BF16)) |
                            (y16 ? BEAM_Y_BF16 : 0u);
    // the copy streams start after the work already on `st` (x_stage / y_stage are free)
    BEAM_CUDA(cudaEventRecord(h->ev_copied, st));
    BEAM_CUDA(cudaStreamWaitEvent(h->copy_in, h->ev_copied, 0));
    BEAM_CUDA(cudaStreamWaitEvent(h->copy_out, h->ev_copied, 0));
    const RouteIn base = own_routing(h);
    int nchunks = 0;
    for (int c = 0, off = 0; c < C; off += sizes[c], ++c) {
        const int n = sizes[c];
        const size_t xo = (size_t)off * D;
        BEAM_CUDA(cudaMemcpyAsync(static_cast<T*>(h->x_stage) + xo, x_host + xo, (size_t)n * D * sizeof(T),
                                  cudaMemcpyHostToDevice, h->copy_in));
        BEAM_CUDA(cudaEventRecord(h->ev_in[c], h->copy_in));
        BEAM_CUDA(cudaStreamWaitEvent(st, h->ev_in[c], 0));
        // the chunk's routing lands at its offset of the handle's routing arrays
        h->topk_id = const_cast<int*>(base.topk_id) + (size_t)off * K;
        h->gate = const_cast<float*>(base.gate) + (size_t)off * K;
        h->mlogit = const_cast<float*>(base.mlogit) + (size_t)off * K;
        h->keep = const_cast<uint8_t*>(base.keep) + (size_t)off * K;
        h->ghat = const_cast<float*>(base.ghat) + (size_t)off * K;
        h->nkeep_tok = const_cast<int*>(base.nkeep) + off;
        h->lreg_tok = const_cast<float*>(base.lreg) + off;
        beam_status_t r = forward_impl<T>(h, static_cast<const T*>(h->x_stage) + xo, n,
                                          host_y_dev(h, h->y_stage + xo, h->y16_stage + xo, y16),
                                          fflags, use_tc, st);
        h->topk_id = const_cast<int*>(base.topk_id); h->gate = const_cast<float*>(base.gate);
        h->mlogit = const_cast<float*>(base.mlogit); h->keep = const_cast<uint8_t*>(base.keep);
        h->ghat = const_cast<float*>(base.ghat); h->nkeep_tok = const_cast<int*>(base.nkeep);
        h->lreg_tok = const_cast<float*>(base.lreg);
        BEAM_TRY(r);
        BEAM_CUDA(launch(h, ST_CHUNK_STATS, stats_accumulate_kernel, dim3(1), dim3(256), 0, st,
                         h->dstats, (const int*)h->counts, h->acc_stats, h->acc_counts, E, c == 0 ? 0 : 1));
        BEAM_CUDA(cudaEventRecord(h->ev_out[c], st));
        BEAM_CUDA(cudaStreamWaitEvent(h->copy_out, h->ev_out[c], 0));
        BEAM_CUDA(copy_y_out(h, y_host, off, n, y16, h->copy_out));
        ++nchunks;
    }
    BEAM_CUDA(launch(h, ST_CHUNK_STATS, stats_accumulate_kernel, dim3(1), dim3(256), 0, st,
                     h->dstats, (const int*)h->counts, h->acc_stats, h->acc_counts, E, 2));
    BEAM_CUDA(cudaEventRecord(h->ev_copied, h->copy_out));
    BEAM_CUDA(cudaStreamWaitEvent(st, h->ev_copied, 0));
    (void)nchunks;
    return BEAM_OK;
}

// beam_moe_forward_host with BEAM_HOST_ASYNC: one whole-batch forward per call, on staging
// set b = the call's parity, and no wait at the end.  The input copy (copy_in) waits for the
// forward that last read set b; the forward (on `st`) waits for its input copy and for the copy
// out that last read y set b; the output copy (copy_out) waits for the forward.  So call k+1's
// input copy and call k-1's output copy run during call k's forward.
static beam_status_t async_setup(beam_moe* h)
{
    if (h->x_stage2) return BEAM_OK;
    const size_t n = (size_t)h->Tmax * h->D;
    BEAM_TRY(dalloc(h, &h->x_stage2, n * h->esz));
    BEAM_TRY(dalloc(h, &h->y_stage2, n * sizeof(float)));
    BEAM_TRY(dalloc(h, &h->y16_stage2, n * sizeof(__nv_bfloat16)));
    for (int b = 0; b < 2; ++b) {
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_ax_ready[b], cudaEventDisableTiming));
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_ax_free[b], cudaEventDisableTiming));
        BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_ay_free[b], cudaEventDisableTiming));
    }
    BEAM_CUDA(cudaEventCreateWithFlags(&h->ev_async_last, cudaEventDisableTiming));
    return BEAM_OK;
}

template <typename T>
static beam_status_t forward_host_async(beam_moe* h, const T* x_host, int T_, void* y_host,
                                        uint32_t flags, cudaStream_t st)
{
    BEAM_TRY(async_setup(h));
    const int b = h->async_next;
    T* xs = static_cast<T*>(b ? h->x_stage2 : h->x_stage);
    float* ys = b ? h->y_stage2 : h->y_stage;
    __nv_bfloat16* y16 = b ? h->y16_stage2 : h->y16_stage;
    const size_t n = (size_t)T_ * h->D;
    const bool y16_out = (flags & BEAM_HOST_Y_BF16) != 0;
    const bool use_tc = (flags & BEAM_PATH_TENSOR) ? true : (flags & BEAM_PATH_STREAM) ? false : h->tc_ok;
    const uint32_t fflags = (flags & ~(BEAM_HOST_ASYNC | BEAM_NO_GRAPH | BEAM_HOST_Y_BF16)) |
                            (y16_out ? BEAM_Y_BF16 : 0u);
    if (!h->async_used[b]) {
        // first use of this set: after everything already on `st`
        BEAM_CUDA(cudaEventRecord(h->ev_ax_free[b], st));
    }
    BEAM_CUDA(cudaStreamWaitEvent(h->copy_in, h->ev_ax_free[b], 0));
    BEAM_CUDA(cudaMemcpyAsync(xs, x_host, n * sizeof(T), cudaMemcpyHostToDevice, h->copy_in));
    BEAM_CUDA(cudaEventRecord(h->ev_ax_ready[b], h->copy_in));
    BEAM_CUDA(cudaStreamWaitEvent(st, h->ev_ax_ready[b], 0));
    if (h->async_used[b]) BEAM_CUDA(cudaStreamWaitEvent(st, h->ev_ay_free[b], 0));
    BEAM_TRY(forward_impl<T>(h, xs, T_, host_y_dev(h, ys, y16, y16_out), fflags, use_tc, st));
    BEAM_CUDA(cudaEventRecord(h->ev_ax_free[b], st));
    BEAM_CUDA(cudaStreamWaitEvent(h->copy_out, h->ev_ax_free[b], 0));
    if (y16_out)
        BEAM_CUDA(cudaMemcpyAsync(y_host, y16, n * sizeof(__nv_bfloat16), cudaMemcpyDeviceToHost, h->copy_out));
    else
        BEAM_CUDA(cudaMemcpyAsync(y_host, ys, n * sizeof(float), cudaMemcpyDeviceToHost, h->copy_out));
    BEAM_CUDA(cudaEventRecord(h->ev_ay_free[b], h->copy_out));
    BEAM_CUDA(cudaEventRecord(h->ev_async_last, h->copy_out));
    h->async_used[b] = true;
    h->async_next = b ^ 1;
    h->async_pending = true;
    return BEAM_OK;
}

// Before a synchronous host call reuses staging set 0: the asynchronous calls' copies are done.
static cudaError_t join_async(beam_moe* h, cudaStream_t st)
{
    if (!h->async_pending) return cudaSuccess;
    h->async_pending = false;
    cudaError_t e = cudaStreamWaitEvent(st, h->ev_async_last, 0);
    if (e != cudaSuccess) return e;
    // and the next input copy of set 0 or 1 starts after this call's forward (copy_in waits
    // on ev_ax_free, which that call records again)
    return cudaSuccess;
}

extern "C" {

beam_status_t beam_moe_route_noalloc(beam_moe_t* h, const void* x, int32_t T, int32_t* topk_id,
                                     float* gate, float* mask_logit, uint8_t* keep, float* ghat,
                                     uint32_t flags, void* stream)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return fail(BEAM_ERR_INVALID_ARG, "T=%d is negative", T);
    if (flags & ~BEAM_MASK_OFF)
        return fail(BEAM_ERR_INVALID_ARG, "only BEAM_MASK_OFF is accepted, got flags 0x%x", flags);
    if (T == 0) return BEAM_OK;
    if (!x || !topk_id || !gate || !mask_logit || !keep || !ghat)
        return fail(BEAM_ERR_INVALID_ARG, "x and every output pointer must be non-NULL");
    if ((reinterpret_cast<uintptr_t>(topk_id) | reinterpret_cast<uintptr_t>(gate) |
         reinterpret_cast<uintptr_t>(mask_logit) | reinterpret_cast<uintptr_t>(ghat)) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "topk_id, gate, mask_logit and ghat must be 4-byte aligned");
    if (reinterpret_cast<uintptr_t>(x) & 15)
        return fail(BEAM_ERR_INVALID_ARG, "x must be 16-byte aligned");
    const long long Tr = (T + h->S - 1) / h->S;
    const long long need = ((Tr * h->n2E * 4 + 255) & ~255LL) + 8LL * T;
    if (need > (long long)BEAM_ROUTE_NOALLOC_SCRATCH_BYTES)
        return fail(BEAM_ERR_INVALID_ARG,
                    "T=%d needs %lld bytes of routing scratch; the static buffer holds %u bytes",
                    T, need, (unsigned)BEAM_ROUTE_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    BEAM_TRY(route_scratch_address(&scratch, st));
    const int mask_off = (flags & BEAM_MASK_OFF) ? 1 : 0;
    unsigned char* sc = static_cast<unsigned char*>(scratch);
    if (h->cfg.dtype == BEAM_DTYPE_BF16)
        return route_noalloc_impl<__nv_bfloat16>(h, static_cast<const __nv_bfloat16*>(x), T,
                                                 topk_id, gate, mask_logit, keep, ghat, mask_off,
                                                 sc, st);
    return route_noalloc_impl<float>(h, static_cast<const float*>(x), T, topk_id, gate,
                                     mask_logit, keep, ghat, mask_off, sc, st);
}

beam_status_t beam_gen_create(const beam_gen_config_t* cfg, const void* w_router,
                              const void* w_mask, void* stream, beam_gen_t** out)
{
    g_err[0] = 0;
    BEAM_TRY(gen_validate(cfg));
    if (!w_router || !w_mask || !out) return fail(BEAM_ERR_INVALID_ARG, "weights or out is NULL");
    beam_gen* g = new (std::nothrow) beam_gen();
    if (!g) return fail(BEAM_ERR_OOM, "host allocation failed");
    beam_status_t s = gen_create_impl(cfg, w_router, w_mask, static_cast<cudaStream_t>(stream), g);
    if (s != BEAM_OK) {
        cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        free_all(&g->core);
        delete g;
        return s;
    }
    *out = g;
    return BEAM_OK;
}

beam_status_t beam_gen_route(beam_gen_t* g, const void* z, int32_t T, const beam_routing_t* out,
                             uint32_t flags, void* stream)
{
    g_err[0] = 0;
    if (!g || !out) return fail(BEAM_ERR_INVALID_ARG, "generator or out is NULL");
    beam_moe* h = &g->core;
    if (T < 0 || T > h->Tmax) return fail(BEAM_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, h->Tmax);
    if (flags & ~BEAM_MASK_OFF)
        return fail(BEAM_ERR_INVALID_ARG, "only BEAM_MASK_OFF is accepted, got flags 0x%x", flags);
    if (T == 0) return BEAM_OK;
    if (!z || !out->topk_id || !out->gate || !out->mask_logit || !out->keep || !out->ghat ||
        !out->n_keep || !out->lreg)
        return fail(BEAM_ERR_INVALID_ARG, "z and every routing array except active must be non-NULL");
    if (reinterpret_cast<uintptr_t>(z) & 15) return fail(BEAM_ERR_INVALID_ARG, "z must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(out->topk_id) | reinterpret_cast<uintptr_t>(out->gate) |
         reinterpret_cast<uintptr_t>(out->mask_logit) | reinterpret_cast<uintptr_t>(out->ghat) |
         reinterpret_cast<uintptr_t>(out->n_keep) | reinterpret_cast<uintptr_t>(out->lreg) |
         reinterpret_cast<uintptr_t>(out->active)) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "the 32-bit routing arrays must be 4-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int mask_off = (flags & BEAM_MASK_OFF) ? 1 : 0;
    if (h->cfg.dtype == BEAM_DTYPE_BF16)
        BEAM_TRY(gen_route_impl<__nv_bfloat16>(g, static_cast<const __nv_bfloat16*>(z), T, out, mask_off, st));
    else
        BEAM_TRY(gen_route_impl<float>(g, static_cast<const float*>(z), T, out, mask_off, st));
    BEAM_CUDA(cudaEventRecord(h->done, st));
    return BEAM_OK;
}

beam_status_t beam_gen_sync(beam_gen_t* g)
{
    g_err[0] = 0;
    if (!g) return fail(BEAM_ERR_INVALID_ARG, "generator is NULL");
    BEAM_CUDA(cudaEventSynchronize(g->core.done));
    DevStats ds;
    BEAM_CUDA(cudaMemcpy(&ds, g->core.dstats, sizeof ds, cudaMemcpyDeviceToHost));
    if (ds.err & ~ERR_FP16_RANGE)
        return fail(BEAM_ERR_TIMEOUT, "a bounded device wait ran out (code %d)", ds.err);
    if (ds.err & ERR_FP16_RANGE)
        return fail(BEAM_ERR_RANGE, "an fp16 intermediate of the last forward (H = silu(gate) * up, "
                    "or an expert output) was outside the fp16 range; y holds infinities");
    return BEAM_OK;
}

void beam_gen_destroy(beam_gen_t* g)
{
    if (!g) return;
    if (g->core.done) cudaEventSynchronize(g->core.done);
    free_all(&g->core);
    delete g;
}

beam_status_t beam_moe_create(const beam_moe_config_t* cfg, const beam_moe_weights_t* w,
                              void* stream, beam_moe_t** out)
{
    g_err[0] = 0;
    BEAM_TRY(validate(cfg));
    if (!w || !out) return fail(BEAM_ERR_INVALID_ARG, "weights or out is NULL");
    if (!w->w_router || !w->w_mask || !w->w_gate || !w->w_up || !w->w_down)
        return fail(BEAM_ERR_INVALID_ARG, "a routed weight pointer is NULL");
    if (cfg->n_shared > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down))
        return fail(BEAM_ERR_INVALID_ARG, "a shared-expert weight pointer is NULL");
    beam_moe* h = new (std::nothrow) beam_moe();
    if (!h) return fail(BEAM_ERR_OOM, "host allocation failed");
    beam_status_t s = create_impl(cfg, w, static_cast<cudaStream_t>(stream), h);
    if (s != BEAM_OK) {
        cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        free_all(h);
        delete h;
        return s;
    }
    *out = h;
    return BEAM_OK;
}

beam_status_t beam_moe_create_ep(const beam_moe_config_t* cfg, const beam_moe_weights_t* w,
                                 void* stream, beam_moe_t** out)
{
    g_err[0] = 0;
    BEAM_TRY(validate(cfg));
    if (!w || !out) return fail(BEAM_ERR_INVALID_ARG, "weights or out is NULL");
    if (!w->w_router || !w->w_mask)
        return fail(BEAM_ERR_INVALID_ARG, "w_router and w_mask are required");
    if (cfg->n_shared > 0 && (!w->ws_gate || !w->ws_up || !w->ws_down))
        return fail(BEAM_ERR_INVALID_ARG, "a shared-expert weight pointer is NULL");
    beam_moe* h = new (std::nothrow) beam_moe();
    if (!h) return fail(BEAM_ERR_OOM, "host allocation failed");
    beam_status_t s = create_impl(cfg, w, static_cast<cudaStream_t>(stream), h, true);
    if (s != BEAM_OK) {
        cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        free_all(h);
        delete h;
        return s;
    }
    *out = h;
    return BEAM_OK;
}

beam_status_t beam_moe_ep_dispatch(beam_moe_t* h, const void* x, int32_t T, uint32_t flags,
                                   void* xperm, int32_t* counts, void* stream)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0 || T > h->Tmax) return fail(BEAM_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, h->Tmax);
    if (!counts) return fail(BEAM_ERR_INVALID_ARG, "counts is required");
    if (T > 0 && (!xperm || (reinterpret_cast<uintptr_t>(xperm) & 15)))
        return fail(BEAM_ERR_INVALID_ARG, "xperm must be non-NULL and 16-byte aligned");
    if (T > 0 && !x) return fail(BEAM_ERR_INVALID_ARG, "x is NULL");
    if (T > 0 && (reinterpret_cast<uintptr_t>(x) & 15))
        return fail(BEAM_ERR_INVALID_ARG, "x must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(counts) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "counts must be 4-byte aligned");
    if (flags & ~(BEAM_MASK_OFF | BEAM_PATH_STREAM | BEAM_PATH_TENSOR))
        return fail(BEAM_ERR_INVALID_ARG, "flags: BEAM_MASK_OFF, BEAM_PATH_STREAM or BEAM_PATH_TENSOR");
    if ((flags & BEAM_PATH_STREAM) && (flags & BEAM_PATH_TENSOR))
        return fail(BEAM_ERR_INVALID_ARG, "BEAM_PATH_STREAM and BEAM_PATH_TENSOR are exclusive");
    if ((flags & BEAM_PATH_TENSOR) && !h->tc_ok)
        return fail(BEAM_ERR_UNSUPPORTED, "the tensor-core path needs a bf16 layer with d_model a "
                    "multiple of 256");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool use_tc = (flags & BEAM_PATH_TENSOR) ? true : (flags & BEAM_PATH_STREAM) ? false : h->tc_ok;
    trace("ep_dispatch T=%d flags=0x%x tc=%d Ew=%d Fsh=%d xperm=%p counts=%p", T, flags, (int)use_tc,
          h->Ew, h->Fsh, xperm, (void*)counts);
    if (T > 0) {
        // the compaction gathers the kept rows straight into the caller's buffer (the handle's
        // own X_perm is only read by its expert GEMMs, which a dispatch does not run)
        void* own = h->xperm;
        h->xperm = xperm;
        beam_status_t r = (h->cfg.dtype == BEAM_DTYPE_BF16)
            ? forward_impl<__nv_bfloat16>(h, static_cast<const __nv_bfloat16*>(x), T, nullptr, flags,
                                          use_tc, st, nullptr, true)
            : forward_impl<float>(h, static_cast<const float*>(x), T, nullptr, flags, use_tc, st,
                                  nullptr, true);
        h->xperm = own;
        trace("ep_dispatch forward status %d", (int)r);
        BEAM_TRY(r);
        BEAM_CUDA(cudaMemcpyAsync(counts, h->counts, sizeof(int32_t) * h->E,
                                  cudaMemcpyDeviceToDevice, st));
    } else {
        BEAM_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * h->E, st));
        h->ep_T = 0;
        h->ep_fork = false;
    }
    h->cur = own_routing(h);
    h->last_T = T;
    h->last_train = false;
    h->last_pipelined = false;
    BEAM_CUDA(cudaEventRecord(h->done, st));
    return BEAM_OK;
}

beam_status_t beam_moe_ep_combine(beam_moe_t* h, const float* y_perm, float* y, void* stream)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (h->ep_T < 0) return fail(BEAM_ERR_NO_FORWARD, "no beam_moe_ep_dispatch has run on this handle");
    const int T_ = h->ep_T;
    if (T_ == 0) return BEAM_OK;
    if (!y || (reinterpret_cast<uintptr_t>(y) & 15) || (reinterpret_cast<uintptr_t>(y_perm) & 15))
        return fail(BEAM_ERR_INVALID_ARG, "y and y_perm must be non-NULL and 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h->ep_fork) BEAM_CUDA(cudaStreamWaitEvent(st, h->ev_join, 0));
    YOut yr;
    yr.base = y_perm; yr.splits = 1; yr.stride = 0; yr.f16 = false;
    YOut ysh = h->ep_ysh;
    if (!h->Fsh) ysh.f16 = false;
    cudaError_t e = ysh.f16 ? launch_combine<float, __half>(h, yr, ysh, h->ghat, T_, y, st)
                            : launch_combine<float, float>(h, yr, ysh, h->ghat, T_, y, st);
    BEAM_CUDA(e);
    BEAM_CUDA(cudaEventRecord(h->done, st));
    return BEAM_OK;
}

beam_status_t beam_ep_expert_range(int32_t E, int32_t P, int32_t q, int32_t* first, int32_t* count)
{
    g_err[0] = 0;
    if (E < 1 || P < 1 || q < 0 || q >= P || !first || !count)
        return fail(BEAM_ERR_INVALID_ARG, "need E >= 1, P >= 1, 0 <= q < P and output pointers");
    const long long a = (long long)q * E / P, b = (long long)(q + 1) * E / P;
    *first = (int32_t)a;
    *count = (int32_t)(b - a);
    return BEAM_OK;
}

beam_status_t beam_ep_recv_routing(const int32_t* recv_counts, int32_t P, int32_t E_local,
                                   int32_t n_rows, int32_t* topk_id, uint8_t* keep, float* ghat,
                                   int32_t* n_keep, float* lreg, void* stream)
{
    g_err[0] = 0;
    if (P < 1 || E_local < 0 || (long long)P * E_local > kEpMaxBlocks || n_rows < 0)
        return fail(BEAM_ERR_INVALID_ARG, "need P >= 1, E_local >= 0, P*E_local <= %d, n_rows >= 0",
                    kEpMaxBlocks);
    if (n_rows == 0) return BEAM_OK;
    if (E_local == 0) return fail(BEAM_ERR_INVALID_ARG, "rows received for a rank with no experts");
    if (!recv_counts || !topk_id || !keep || !ghat || !n_keep || !lreg)
        return fail(BEAM_ERR_INVALID_ARG, "a pointer is NULL");
    if ((reinterpret_cast<uintptr_t>(recv_counts) | reinterpret_cast<uintptr_t>(topk_id) |
         reinterpret_cast<uintptr_t>(ghat) | reinterpret_cast<uintptr_t>(n_keep) |
         reinterpret_cast<uintptr_t>(lreg)) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "the 32-bit arrays must be 4-byte aligned");
    const int grid = std::min(ceil_div(n_rows, 256), 148 * 4);
    BEAM_CUDA(launch(nullptr, 0, ep_recv_routing_kernel, dim3(grid), dim3(256), 0,
                     static_cast<cudaStream_t>(stream), (const int*)recv_counts, P * E_local,
                     (int)E_local, (int)n_rows, (int*)topk_id, keep, ghat, (int*)n_keep, lreg));
    return BEAM_OK;
}

// The forward behind beam_moe_forward (rin == nullptr) and beam_moe_forward_routed: argument
// checks shared by both, then the fused decode launch, a graph replay, or direct launches.
static beam_status_t forward_entry(beam_moe* h, const void* x, int32_t T, float* y, uint32_t flags,
                                   const RouteIn* rin, void* stream)
{
    if (h->Ew == 0)
        return fail(BEAM_ERR_UNSUPPORTED, "a routing-only handle (beam_moe_create_ep) runs "
                    "beam_moe_ep_dispatch / beam_moe_ep_combine, not a forward");
    if (T < 0 || T > h->Tmax) return fail(BEAM_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, h->Tmax);
    if (T > 0 && (!x || !y)) return fail(BEAM_ERR_INVALID_ARG, "x or y is NULL");
    if ((flags & BEAM_PATH_STREAM) && (flags & BEAM_PATH_TENSOR))
        return fail(BEAM_ERR_INVALID_ARG, "BEAM_PATH_STREAM and BEAM_PATH_TENSOR are exclusive");
    if (flags & ~(BEAM_MASK_OFF | BEAM_PATH_STREAM | BEAM_PATH_TENSOR | BEAM_NO_GRAPH |
                  BEAM_FUSED_DECODE | BEAM_TRAIN | BEAM_Y_BF16))
        return fail(BEAM_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if ((flags & BEAM_Y_BF16) && (flags & BEAM_FUSED_DECODE))
        return fail(BEAM_ERR_INVALID_ARG, "BEAM_Y_BF16 excludes BEAM_FUSED_DECODE");
    if (T > 0 && (flags & BEAM_Y_BF16) && (reinterpret_cast<uintptr_t>(y) & 7))
        return fail(BEAM_ERR_INVALID_ARG, "a bf16 y must be 8-byte aligned");
    if ((flags & BEAM_TRAIN) && (flags & (BEAM_MASK_OFF | BEAM_FUSED_DECODE)))
        return fail(BEAM_ERR_INVALID_ARG, "BEAM_TRAIN excludes BEAM_MASK_OFF and BEAM_FUSED_DECODE");
    if ((flags & BEAM_PATH_TENSOR) && !h->tc_ok)
        return fail(BEAM_ERR_UNSUPPORTED, "the tensor-core expert path needs a bf16 layer with "
                    "d_model a multiple of 256");
    if (T > 0 && (reinterpret_cast<uintptr_t>(x) & 15))
        return fail(BEAM_ERR_INVALID_ARG, "x must be 16-byte aligned");
    bool use_tc;
    if (flags & BEAM_PATH_TENSOR) use_tc = true;
    else if (flags & BEAM_PATH_STREAM) use_tc = false;
    else use_tc = h->tc_ok && T >= kTcMinTokens;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h->prof && h->prof_forwards >= h->prof_max) h->prof = false;
    if (h->prof) ++h->prof_forwards;
    auto run = [&]() -> beam_status_t {
        return (h->cfg.dtype == BEAM_DTYPE_BF16)
            ? forward_impl<__nv_bfloat16>(h, static_cast<const __nv_bfloat16*>(x), T, y, flags, use_tc, st, rin)
            : forward_impl<float>(h, static_cast<const float*>(x), T, y, flags, use_tc, st, rin);
    };
    if (T > 0 && !rin && fused_eligible(h, T, flags, use_tc)) {
        // one launch: nothing to gain from a graph
        BEAM_TRY(forward_fused(h, static_cast<const __nv_bfloat16*>(x), T, y, flags, st));
    } else if (T > 0) {
        // Replay: the whole forward (8-10 kernels, their tensor maps and split choices) was
        // captured as a CUDA graph for these exact arguments; one launch replays it.  Not
        // used while profiling, on the legacy default stream, or with BEAM_NO_GRAPH.
        const bool graphable = !(flags & BEAM_NO_GRAPH) && !h->prof && st != nullptr;
        const uint32_t key_flags = flags & ~BEAM_NO_GRAPH;
        const bool same_routing = rin ? (h->g_routed && h->g_rin == *rin) : !h->g_routed;
        if (graphable && h->graph_exec && h->g_x == x && h->g_y == y && h->g_T == T &&
            h->g_flags == key_flags && h->g_tc == use_tc && same_routing) {
            BEAM_CUDA(cudaGraphLaunch(h->graph_exec, st));
            h->launches += h->g_kernels;
            h->cur = rin ? *rin : own_routing(h);
            h->last_yr = h->g_yr;
        } else {
            bool captured = false;
            if (graphable) {
                cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
                if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone &&
                    cudaStreamBeginCapture(st, cudaStreamCaptureModeThreadLocal) == cudaSuccess) {
                    const long long n0 = h->launches;
                    beam_status_t s1 = run();
                    cudaGraph_t g = nullptr;
                    cudaError_t e1 = cudaStreamEndCapture(st, &g);
                    h->launches = n0;  // counted again when the graph runs
                    if (s1 != BEAM_OK) {
                        if (g) cudaGraphDestroy(g);
                        return s1;
                    }
                    cudaGraphExec_t ex = nullptr;
                    if (e1 == cudaSuccess && g && cudaGraphInstantiate(&ex, g, 0) == cudaSuccess) {
                        size_t nn = 0;
                        cudaGraphGetNodes(g, nullptr, &nn);
                        drop_graph(h);
                        h->graph_exec = ex;
                        h->g_x = x; h->g_y = y; h->g_T = T; h->g_flags = key_flags; h->g_tc = use_tc;
                        h->g_routed = rin != nullptr;
                        h->g_rin = rin ? *rin : RouteIn();
                        h->g_kernels = (int)nn;
                        h->g_yr = h->last_yr;
                        captured = true;
                    }
                    if (g) cudaGraphDestroy(g);
                    cudaGetLastError();
                    if (captured) {
                        BEAM_CUDA(cudaGraphLaunch(h->graph_exec, st));
                        h->launches += h->g_kernels;
                    }
                } else {
                    cudaGetLastError();
                }
            }
            if (!captured) BEAM_TRY(run());
        }
    }
    h->last_T = T;
    h->last_train = (flags & BEAM_TRAIN) != 0;
    h->last_pipelined = false;
    BEAM_CUDA(cudaEventRecord(h->done, st));
    return BEAM_OK;
}

beam_status_t beam_moe_forward(beam_moe_t* h, const void* x, int32_t T, float* y, uint32_t flags,
                               void* stream)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    return forward_entry(h, x, T, y, flags, nullptr, stream);
}

beam_status_t beam_moe_forward_routed(beam_moe_t* h, const void* x, int32_t T,
                                      const beam_routing_t* r, float* y, uint32_t flags,
                                      void* stream)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (!r) return fail(BEAM_ERR_INVALID_ARG, "routing is NULL");
    if (flags & (BEAM_MASK_OFF | BEAM_FUSED_DECODE | BEAM_TRAIN))
        return fail(BEAM_ERR_INVALID_ARG, "BEAM_MASK_OFF, BEAM_FUSED_DECODE and BEAM_TRAIN do not "
                    "apply to a forward with given routing (the mask is part of the routing)");
    if (T > 0 && (!r->topk_id || !r->keep || !r->ghat || !r->n_keep || !r->lreg))
        return fail(BEAM_ERR_INVALID_ARG, "routing needs topk_id, keep, ghat, n_keep and lreg");
    // the compaction reads a token's K slots as one vector when K is 4, 8 or 16
    const bool vec = h->K == 4 || h->K == 8 || h->K == 16;
    if (T > 0 && ((reinterpret_cast<uintptr_t>(r->topk_id) & (vec ? 15 : 3)) ||
                  (reinterpret_cast<uintptr_t>(r->keep) & (vec ? h->K - 1 : 0))))
        return fail(BEAM_ERR_INVALID_ARG, "topk_id must be 4-byte aligned and keep 1-byte aligned "
                    "(top_k 4, 8 or 16: topk_id 16-byte, keep top_k-byte aligned)");
    if (T > 0 && ((reinterpret_cast<uintptr_t>(r->ghat) | reinterpret_cast<uintptr_t>(r->n_keep) |
                   reinterpret_cast<uintptr_t>(r->lreg)) & 3))
        return fail(BEAM_ERR_INVALID_ARG, "ghat, n_keep and lreg must be 4-byte aligned");
    RouteIn rin;
    rin.topk_id = r->topk_id; rin.keep = r->keep; rin.ghat = r->ghat; rin.nkeep = r->n_keep;
    rin.lreg = r->lreg; rin.gate = r->gate; rin.mlogit = r->mask_logit;
    return forward_entry(h, x, T, y, flags, &rin, stream);
}

beam_status_t beam_moe_forward_host(beam_moe_t* h, const void* x_host, int32_t T, void* y_host,
                                    uint32_t flags, void* stream)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0 || T > h->Tmax) return fail(BEAM_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, h->Tmax);
    if (T > 0 && (!x_host || !y_host)) return fail(BEAM_ERR_INVALID_ARG, "x or y is NULL");
    if (flags & BEAM_Y_BF16)
        return fail(BEAM_ERR_INVALID_ARG, "host calls take BEAM_HOST_Y_BF16 for a bf16 y, not BEAM_Y_BF16");
    if ((flags & BEAM_HOST_Y_BF16) && (flags & BEAM_FUSED_DECODE))
        return fail(BEAM_ERR_INVALID_ARG, "BEAM_HOST_Y_BF16 excludes BEAM_FUSED_DECODE");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (flags & BEAM_HOST_ASYNC) {
        if (flags & ~(BEAM_MASK_OFF | BEAM_PATH_STREAM | BEAM_PATH_TENSOR | BEAM_NO_GRAPH | BEAM_HOST_Y_BF16 |
                      BEAM_HOST_ASYNC))
            return fail(BEAM_ERR_INVALID_ARG, "BEAM_HOST_ASYNC takes only BEAM_MASK_OFF, BEAM_PATH_*, "
                        "BEAM_NO_GRAPH and BEAM_HOST_Y_BF16 (flags 0x%x)", flags);
        if ((flags & BEAM_PATH_STREAM) && (flags & BEAM_PATH_TENSOR))
            return fail(BEAM_ERR_INVALID_ARG, "BEAM_PATH_STREAM and BEAM_PATH_TENSOR are exclusive");
        if ((flags & BEAM_PATH_TENSOR) && !h->tc_ok)
            return fail(BEAM_ERR_UNSUPPORTED, "the tensor-core expert path needs a bf16 layer with "
                        "d_model a multiple of 256");
        if (h->Ew == 0) return fail(BEAM_ERR_UNSUPPORTED, "a routing-only handle has no expert forward");
        if (T == 0) return BEAM_OK;
        if (h->prof && h->prof_forwards >= h->prof_max) h->prof = false;
        if (h->prof) ++h->prof_forwards;
        beam_status_t r = (h->cfg.dtype == BEAM_DTYPE_BF16)
            ? forward_host_async<__nv_bfloat16>(h, static_cast<const __nv_bfloat16*>(x_host), T, y_host, flags, st)
            : forward_host_async<float>(h, static_cast<const float*>(x_host), T, y_host, flags, st);
        BEAM_TRY(r);
        h->cur = own_routing(h);
        h->last_T = T;
        h->last_train = false;
        h->last_pipelined = false;
        BEAM_CUDA(cudaEventRecord(h->done, st));
        return BEAM_OK;
    }
    BEAM_CUDA(join_async(h, st));
    if ((flags & BEAM_HOST_PIPELINE) && T >= kHostPipelineMinTokens && h->Ew > 0) {
        if (flags & (BEAM_TRAIN | BEAM_FUSED_DECODE))
            return fail(BEAM_ERR_INVALID_ARG, "BEAM_HOST_PIPELINE excludes BEAM_TRAIN and BEAM_FUSED_DECODE");
        if (flags & ~(BEAM_MASK_OFF | BEAM_PATH_STREAM | BEAM_PATH_TENSOR | BEAM_NO_GRAPH | BEAM_HOST_PIPELINE |
                      BEAM_HOST_Y_BF16))
            return fail(BEAM_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
        if ((flags & BEAM_PATH_STREAM) && (flags & BEAM_PATH_TENSOR))
            return fail(BEAM_ERR_INVALID_ARG, "BEAM_PATH_STREAM and BEAM_PATH_TENSOR are exclusive");
        if ((flags & BEAM_PATH_TENSOR) && !h->tc_ok)
            return fail(BEAM_ERR_UNSUPPORTED, "the tensor-core expert path needs a bf16 layer with "
                        "d_model a multiple of 256");
        if (h->prof && h->prof_forwards >= h->prof_max) h->prof = false;
        if (h->prof) ++h->prof_forwards;
        beam_status_t r = (h->cfg.dtype == BEAM_DTYPE_BF16)
            ? forward_host_pipelined<__nv_bfloat16>(h, static_cast<const __nv_bfloat16*>(x_host), T,
                                                    y_host, flags, st)
            : forward_host_pipelined<float>(h, static_cast<const float*>(x_host), T, y_host, flags, st);
        BEAM_TRY(r);
        h->cur = own_routing(h);
        h->last_T = T;
        h->last_train = false;
        h->last_pipelined = true;
        BEAM_CUDA(cudaEventRecord(h->done, st));
        BEAM_CUDA(cudaStreamSynchronize(st));
        return BEAM_OK;
    }
    const size_t xb = (size_t)T * h->D * h->esz;
    const bool y16 = (flags & BEAM_HOST_Y_BF16) != 0;
    if (T > 0) BEAM_CUDA(cudaMemcpyAsync(h->x_stage, x_host, xb, cudaMemcpyHostToDevice, st));
    BEAM_TRY(beam_moe_forward(h, h->x_stage, T, host_y_dev(h, h->y_stage, h->y16_stage, y16),
                              (flags & ~(BEAM_HOST_PIPELINE | BEAM_HOST_Y_BF16)) | (y16 ? BEAM_Y_BF16 : 0u),
                              stream));
    if (T > 0) BEAM_CUDA(copy_y_out(h, y_host, 0, T, y16, st));
    BEAM_CUDA(cudaStreamSynchronize(st));
    return BEAM_OK;
}

beam_status_t beam_moe_host_wait(beam_moe_t* h)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (h->copy_in) BEAM_CUDA(cudaStreamSynchronize(h->copy_in));
    if (h->copy_out) BEAM_CUDA(cudaStreamSynchronize(h->copy_out));
    if (h->done) BEAM_CUDA(cudaEventSynchronize(h->done));
    return BEAM_OK;
}

beam_status_t beam_moe_stats(beam_moe_t* h, beam_moe_stats_t* out, int32_t* counts_host)
{
    g_err[0] = 0;
    if (!h || !out) return fail(BEAM_ERR_INVALID_ARG, "handle or out is NULL");
    if (h->last_T < 0) return fail(BEAM_ERR_NO_FORWARD, "no forward has run on this handle");
    BEAM_CUDA(cudaEventSynchronize(h->done));
    memset(out, 0, sizeof *out);
    if (h->last_T == 0) {
        if (counts_host) memset(counts_host, 0, sizeof(int32_t) * h->E);
        return BEAM_OK;
    }
    DevStats ds;
    BEAM_CUDA(cudaMemcpy(&ds, h->dstats, sizeof ds, cudaMemcpyDeviceToHost));
    if (ds.err & ~ERR_FP16_RANGE)
        return fail(BEAM_ERR_TIMEOUT, "a bounded device wait ran out (code %d)", ds.err);
    if (ds.err & ERR_FP16_RANGE)
        return fail(BEAM_ERR_RANGE, "an fp16 intermediate of the last forward (H = silu(gate) * up, "
                    "or an expert output) was outside the fp16 range; y holds infinities");
    out->tokens = ds.tokens;
    out->avg_k = ds.tokens ? (double)ds.keep_sum / ds.tokens : 0.0;
    out->l_reg = ds.tokens ? ds.lreg_sum / ds.tokens : 0.0;
    out->n_active_experts = ds.n_active;
    out->n_tokens_all_masked = ds.n_all_masked;
    out->n_kept = ds.n_kept;
    if (counts_host)
        BEAM_CUDA(cudaMemcpy(counts_host, h->counts, sizeof(int32_t) * h->E, cudaMemcpyDeviceToHost));
    return BEAM_OK;
}

beam_status_t beam_moe_get_routing(beam_moe_t* h, int32_t* topk_id, float* gate, float* mask_logit,
                                   uint8_t* keep, int32_t* offsets, int32_t* perm, int32_t* inv)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (h->last_T < 0) return fail(BEAM_ERR_NO_FORWARD, "no forward has run on this handle");
    BEAM_CUDA(cudaEventSynchronize(h->done));
    const size_t n = (size_t)h->last_T * h->K;
    if (h->last_T == 0) {
        if (offsets) memset(offsets, 0, sizeof(int32_t) * (h->E + 1));
        return BEAM_OK;
    }
    if (h->last_pipelined && (offsets || perm || inv))
        return fail(BEAM_ERR_UNSUPPORTED, "after a pipelined host call (BEAM_HOST_PIPELINE) only "
                    "topk_id, gate, mask_logit and keep are available: the compaction ran per chunk");
    // the arrays the last forward read: its own, or those given to beam_moe_forward_routed
    const RouteIn& c = h->cur;
    if ((gate && !c.gate) || (mask_logit && !c.mlogit))
        return fail(BEAM_ERR_INVALID_ARG, "the last forward was given no gate / mask_logit array");
    if (topk_id) BEAM_CUDA(cudaMemcpy(topk_id, c.topk_id, n * 4, cudaMemcpyDeviceToHost));
    if (gate) BEAM_CUDA(cudaMemcpy(gate, c.gate, n * 4, cudaMemcpyDeviceToHost));
    if (mask_logit) BEAM_CUDA(cudaMemcpy(mask_logit, c.mlogit, n * 4, cudaMemcpyDeviceToHost));
    if (keep) BEAM_CUDA(cudaMemcpy(keep, c.keep, n, cudaMemcpyDeviceToHost));
    if (inv) BEAM_CUDA(cudaMemcpy(inv, h->inv, n * 4, cudaMemcpyDeviceToHost));
    int nk = 0;
    BEAM_CUDA(cudaMemcpy(&nk, h->offsets + h->E, sizeof nk, cudaMemcpyDeviceToHost));
    if (offsets) BEAM_CUDA(cudaMemcpy(offsets, h->offsets, sizeof(int32_t) * (h->E + 1), cudaMemcpyDeviceToHost));
    if (perm && nk > 0) BEAM_CUDA(cudaMemcpy(perm, h->perm, sizeof(int32_t) * nk, cudaMemcpyDeviceToHost));
    return BEAM_OK;
}

beam_status_t beam_moe_profile_begin(beam_moe_t* h, int32_t max_forwards)
{
    g_err[0] = 0;
    if (!h || max_forwards < 1 || max_forwards > 100000)
        return fail(BEAM_ERR_INVALID_ARG, "handle NULL or max_forwards outside [1, 100000]");
    prof_release(h);
    const size_t n = (size_t)max_forwards * 2 * 16;  // <= 16 launches per forward
    h->prof_pool.reserve(n);
    for (size_t i = 0; i < n; ++i) {
        cudaEvent_t e;
        cudaError_t err = cudaEventCreate(&e);
        if (err != cudaSuccess) {
            prof_release(h);
            return fail(BEAM_ERR_CUDA, "cudaEventCreate failed: %s", cudaGetErrorString(err));
        }
        h->prof_pool.push_back(e);
    }
    h->prof_recs.reserve(n / 2);
    h->prof_max = max_forwards;
    h->prof_forwards = 0;
    h->prof = true;
    return BEAM_OK;
}

beam_status_t beam_moe_profile_end(beam_moe_t* h, float* stage_ms, int32_t* stage_launches,
                                   int32_t* n_forwards)
{
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    float ms[ST_COUNT] = {0};
    int32_t cnt[ST_COUNT] = {0};
    for (auto& r : h->prof_recs) {
        cudaError_t e = cudaEventSynchronize(r.b);
        float t = 0.f;
        if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
        if (e != cudaSuccess) {
            prof_release(h);
            return fail(BEAM_ERR_CUDA, "profiling events failed: %s", cudaGetErrorString(e));
        }
        ms[r.stage] += t;
        cnt[r.stage] += 1;
    }
    if (stage_ms) memcpy(stage_ms, ms, sizeof ms);
    if (stage_launches) memcpy(stage_launches, cnt, sizeof cnt);
    if (n_forwards) *n_forwards = h->prof_forwards;
    prof_release(h);
    return BEAM_OK;
}

const char* beam_moe_stage_name(int32_t stage)
{
    return (stage >= 0 && stage < ST_COUNT) ? kStageNames[stage] : "";
}

int64_t beam_moe_launch_count(const beam_moe_t* h) { return h ? h->launches : 0; }

static __device__ int g_wait_selftest_result;

beam_status_t beam_moe_backward_router(beam_moe_t* h, const void* x, const float* dy, int32_t T,
                                       float reg_scale, float* dw_router, float* dw_mask,
                                       float* dx, float* d_gate_logit, float* d_mask_logit,
                                       float* dghat, void* stream)
{
    if (h && h->Ew == 0)
        return fail(BEAM_ERR_UNSUPPORTED, "a routing-only handle (beam_moe_create_ep) has no "
                    "expert outputs to differentiate");
    g_err[0] = 0;
    if (!h) return fail(BEAM_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0 || T > h->Tmax) return fail(BEAM_ERR_INVALID_ARG, "T=%d outside [0, %d]", T, h->Tmax);
    if (T == 0) return BEAM_OK;
    if (!h->last_train || h->last_T != T)
        return fail(BEAM_ERR_NO_FORWARD, "the routing gradient needs the handle's last forward to "
                    "be a BEAM_TRAIN forward of the same T (last forward: T=%d, %s)", h->last_T,
                    h->last_train ? "training" : "not training");
    if (!x || !dy || !dw_router || !dw_mask || !dx)
        return fail(BEAM_ERR_INVALID_ARG, "x, dy, dw_router, dw_mask and dx are required");
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy) |
         reinterpret_cast<uintptr_t>(dx)) & 15)
        return fail(BEAM_ERR_INVALID_ARG, "x, dy and dx must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(dw_router) | reinterpret_cast<uintptr_t>(dw_mask) |
         reinterpret_cast<uintptr_t>(d_gate_logit) | reinterpret_cast<uintptr_t>(d_mask_logit) |
         reinterpret_cast<uintptr_t>(dghat)) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "the float32 outputs must be 4-byte aligned");
    if (!std::isfinite(reg_scale))
        return fail(BEAM_ERR_INVALID_ARG, "reg_scale must be finite");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (h->cfg.dtype == BEAM_DTYPE_BF16)
        BEAM_TRY(backward_impl<__nv_bfloat16>(h, static_cast<const __nv_bfloat16*>(x), dy, T,
                                              reg_scale, dw_router, dw_mask, dx, d_gate_logit,
                                              d_mask_logit, dghat, st));
    else
        BEAM_TRY(backward_impl<float>(h, static_cast<const float*>(x), dy, T, reg_scale, dw_router,
                                      dw_mask, dx, d_gate_logit, d_mask_logit, dghat, st));
    return BEAM_OK;
}

// ---------------------------------------------------------------- SoftTopK
beam_status_t beam_softtopk_forward(const float* logits, int32_t T, int32_t E, int32_t K,
                                    float tau, float* y, uint8_t* mask, float* nu, void* stream)
{
    g_err[0] = 0;
    BEAM_TRY(softtopk_check(T, E, tau, logits, y, y));
    if (K < 1 || K > E) return fail(BEAM_ERR_INVALID_ARG, "K=%d must be in [1, E=%d]", K, E);
    if (reinterpret_cast<uintptr_t>(nu) & 3)
        return fail(BEAM_ERR_INVALID_ARG, "nu must be 4-byte aligned");
    if (T == 0) return BEAM_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch ((E + 31) / 32) {
        case 1: e = launch_softtopk_fwd<1>(logits, T, E, K, tau, y, mask, nu, st); break;
        case 2: e = launch_softtopk_fwd<2>(logits, T, E, K, tau, y, mask, nu, st); break;
        case 3: e = launch_softtopk_fwd<3>(logits, T, E, K, tau, y, mask, nu, st); break;
        case 4: e = launch_softtopk_fwd<4>(logits, T, E, K, tau, y, mask, nu, st); break;
        case 5: e = launch_softtopk_fwd<5>(logits, T, E, K, tau, y, mask, nu, st); break;
        case 6: e = launch_softtopk_fwd<6>(logits, T, E, K, tau, y, mask, nu, st); break;
        case 7: e = launch_softtopk_fwd<7>(logits, T, E, K, tau, y, mask, nu, st); break;
        default: e = launch_softtopk_fwd<8>(logits, T, E, K, tau, y, mask, nu, st); break;
    }
    BEAM_CUDA(e);
    return BEAM_OK;
}

beam_status_t beam_softtopk_backward(const float* y, const float* dy, int32_t T, int32_t E,
                                     float tau, float* dlogits, void* stream)
{
    g_err[0] = 0;
    BEAM_TRY(softtopk_check(T, E, tau, y, dy, dlogits));
    if (T == 0) return BEAM_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    switch ((E + 31) / 32) {
        case 1: e = launch_softtopk_bwd<1>(y, dy, T, E, tau, dlogits, st); break;
        case 2: e = launch_softtopk_bwd<2>(y, dy, T, E, tau, dlogits, st); break;
        case 3: e = launch_softtopk_bwd<3>(y, dy, T, E, tau, dlogits, st); break;
        case 4: e = launch_softtopk_bwd<4>(y, dy, T, E, tau, dlogits, st); break;
        case 5: e = launch_softtopk_bwd<5>(y, dy, T, E, tau, dlogits, st); break;
        case 6: e = launch_softtopk_bwd<6>(y, dy, T, E, tau, dlogits, st); break;
        case 7: e = launch_softtopk_bwd<7>(y, dy, T, E, tau, dlogits, st); break;
        default: e = launch_softtopk_bwd<8>(y, dy, T, E, tau, dlogits, st); break;
    }
    BEAM_CUDA(e);
    return BEAM_OK;
}

beam_status_t beam_moe_wait_selftest(int32_t timeout_us, void* stream)
{
    g_err[0] = 0;
    if (timeout_us < 1 || timeout_us > 2000000)
        return fail(BEAM_ERR_INVALID_ARG, "timeout_us=%d outside [1, 2000000]", timeout_us);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* res = nullptr;
    BEAM_CUDA(cudaGetSymbolAddress((void**)&res, g_wait_selftest_result));
    const int minus_one = -1;
    BEAM_CUDA(cudaMemcpyAsync(res, &minus_one, sizeof(int), cudaMemcpyHostToDevice, st));
    tc::wait_selftest_kernel<<<1, 32, 0, st>>>((unsigned long long)timeout_us * 1000ull, res);
    BEAM_CUDA(cudaGetLastError());
    int out = -1;
    BEAM_CUDA(cudaMemcpyAsync(&out, res, sizeof(int), cudaMemcpyDeviceToHost, st));
    BEAM_CUDA(cudaStreamSynchronize(st));
    if (out == 2) return fail(BEAM_ERR_TIMEOUT, "the bounded wait expired after %d us, as designed", timeout_us);
    return fail(BEAM_ERR_CUDA, "the self-test wait did not expire (result %d)", out);
}

void beam_moe_destroy(beam_moe_t* h)
{
    if (!h) return;
    if (h->done) cudaEventSynchronize(h->done);
    // copies of asynchronous host calls may still read the staging buffers
    if (h->copy_in) cudaStreamSynchronize(h->copy_in);
    if (h->copy_out) cudaStreamSynchronize(h->copy_out);
    free_all(h);
    delete h;
}

const char* beam_moe_last_error(void) { return g_err; }

const char* beam_moe_version(void) { return "beam_moe 0.1 (sm_100a)"; }

}  // extern "C"
