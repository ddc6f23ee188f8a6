// router.cuh -- fused router of the BEAM layer: logits of x [W_r | W_m], then per token the
// Top-K (ties to the lower index), the K-way softmax, the mask test and the statistics.
//
// BEAM article on aitrends.kr ("BEAM: Dynamic MoE 라우팅을 위한 Binary Expert Activation
// Masking"), four-step pipeline: Step 1 (Top-K of r = x W_r, softmax over the K kept logits),
// Step 2 (m_hat = sigmoid(x W_m)), Step 3 (m_i = 1 iff m_hat_i >= 0.5, evaluated as mask logit
// >= 0), the training paragraph (L_reg = (1/K) sum_{i in TK} m_hat_i, recorded per token) and
// Stepped MoE's segment routing (core method: one decision per segment of S tokens, taken at
// the segment's first token).
#pragma once
#include "common.cuh"

namespace beam {

// ---------------------------------------------------------------- logits, SIMT
// L[i][j] = sum_d x[i*S][d] * Wrm[j][d] for routed rows i < Tr and columns j < n2E, where
// Wrm = [W_r | W_m]^T (one contiguous row of D per output column).  fp32 accumulation; L has
// leading dimension ldL >= n2E.  Used for decode-sized batches and fp32 layers; large bf16
// batches run the same product on the tensor cores (tc_experts.cuh, f32-store epilogue).
// One CTA per (column j, block of kGemvRows routed rows): its 256 threads split the D-long
// weight row with 16-byte loads, each thread keeps one partial per row, and the partials are
// reduced in a fixed order (warp butterfly, then the 8 warps in index order).
constexpr int kGemvRows = 16;
constexpr int kRouteMaxE = 256;  // most routed experts per layer

template <typename TW>
__global__ void __launch_bounds__(256)
router_gemv_kernel(const TW* __restrict__ x, int seg, int Tr, int D,
                   const TW* __restrict__ wrm, int n2E, int ldL, float* __restrict__ L)
{
    __shared__ float red[8][kGemvRows];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x;
    const int row0 = blockIdx.y * kGemvRows;
    const int nrows = min(kGemvRows, Tr - row0);
    const size_t xstride = (size_t)(seg > 1 ? seg : 1) * D;
    constexpr int VN = Vec<TW>::N;
    float acc[kGemvRows];
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) acc[r] = 0.f;
    const TW* wrow = wrm + (size_t)j * D;
    const TW* x0 = x + (size_t)row0 * xstride;
    for (int d = threadIdx.x * VN; d < D; d += 256 * VN) {
        float w[VN];
        Vec<TW>::widen(ldg_stream(wrow + d), w);
#pragma unroll
        for (int r = 0; r < kGemvRows; ++r) {
            if (r < nrows) {
                float xv[VN];
                Vec<TW>::widen(__ldg(reinterpret_cast<const uint4*>(x0 + r * xstride + d)), xv);
                float s = 0.f;
#pragma unroll
                for (int v = 0; v < VN; ++v) s = fmaf(w[v], xv[v], s);
                acc[r] += s;
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kGemvRows; ++r) {
        if (r < nrows) {
            const float s = warp_sum(acc[r]);
            if (lane == 0) red[warp][r] = s;
        }
    }
    __syncthreads();
    if (threadIdx.x < nrows) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += red[w][threadIdx.x];
        L[(size_t)(row0 + threadIdx.x) * ldL + j] = s;
    }
    (void)n2E;
    pdl_launch_dependents();
}

// The same logits for many columns (a cross-layer generator has L*2E of them, where one CTA
// per column would launch thousands of CTAs of a few hundred bytes each): one warp per column
// j and block of ROWS routed rows (1 for a single routed row, so that the warp keeps one
// partial and few registers); the lanes split the D-long weight row with 16-byte loads, each
// lane keeps one partial per row, and a warp butterfly reduces them.
template <typename TW, int ROWS>
__global__ void __launch_bounds__(256)
router_gemv_warp_kernel(const TW* __restrict__ x, int seg, int Tr, int D,
                        const TW* __restrict__ wrm, int n2E, int ldL, float* __restrict__ L)
{
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x * 8 + warp;
    const int row0 = blockIdx.y * ROWS;
    const int nrows = min(ROWS, Tr - row0);
    if (j < n2E) {
        const size_t xstride = (size_t)(seg > 1 ? seg : 1) * D;
        constexpr int VN = Vec<TW>::N;
        float acc[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r] = 0.f;
        const TW* wrow = wrm + (size_t)j * D;
        const TW* x0 = x + (size_t)row0 * xstride;
        // kU weight vectors per lane are loaded before any is used, so a warp has kU 512-byte
        // requests in flight instead of one load round trip per vector
        constexpr int kU = 4;
        for (int d0 = lane * VN; d0 < D; d0 += kU * 32 * VN) {
            uint4 wv[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int d = d0 + u * 32 * VN;
                wv[u] = d < D ? ldg_stream(wrow + d) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int d = d0 + u * 32 * VN;
                if (d < D) {
                    float w[VN];
                    Vec<TW>::widen(wv[u], w);
#pragma unroll
                    for (int r = 0; r < ROWS; ++r) {
                        if (r < nrows) {
                            float xv[VN];
                            Vec<TW>::widen(__ldg(reinterpret_cast<const uint4*>(x0 + r * xstride + d)), xv);
                            float s = 0.f;
#pragma unroll
                            for (int v = 0; v < VN; ++v) s = fmaf(w[v], xv[v], s);
                            acc[r] += s;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            if (r < nrows) {
                const float s = warp_sum(acc[r]);
                if (lane == 0) L[(size_t)(row0 + r) * ldL + j] = s;
            }
        }
    }
    pdl_launch_dependents();
}

// The same logits for a small batch (at most kRouterSmallRows routed rows).  CTA (column block
// b, chunk c) covers columns [8b, 8b + 8) and the D-range [c DC, (c + 1) DC), DC =
// kRouterChunkBytes: its threads first stage the chunk of every routed row in shared memory (one
// read of x per CTA), then warp w takes column 8b + w: lane l reads the 16-byte weight vectors
// v*32 + l of the chunk (coalesced; consecutive lanes hit consecutive shared-memory words) and
// keeps one partial per row.  The 32 row partials are reduced across the lanes by a transposing
// butterfly (lane r ends with row r, 31 shuffles).  With one chunk lane r writes L[r][column].
// With several, lane r writes its chunk's partial into slice c of L (slice c at c * slice_stride;
// slice 0 is L itself), and the CTA counts itself in on the block's arrival counter; the CTA
// that arrives last (the atomic only elects it) adds the block's slices in chunk order into
// slice 0 and resets the counter to zero for the next call.  The selection then reads one
// value per logit.  Deterministic; one read of each weight row; x read once per column block.
constexpr int kRouterSmallRows = 32;
constexpr int kRouterChunkBytes = 1024;   // a chunk of D: 512 bf16 or 256 fp32 elements
constexpr int kRouterMaxChunks = 16;      // D <= 8192 bf16 / 4096 fp32

template <typename TW>
__global__ void __launch_bounds__(256)
router_small_kernel(const TW* __restrict__ x, int seg, int Tr, int D,
                    const TW* __restrict__ wrm, int n2E, int ldL, long long slice_stride,
                    float* __restrict__ L, unsigned* __restrict__ arrive)
{
    constexpr int DC = kRouterChunkBytes / (int)sizeof(TW);   // elements per chunk
    constexpr int VN = Vec<TW>::N;                            // elements per 16-byte vector
    constexpr int NV = DC / (32 * VN);                        // vectors per lane
    __shared__ __align__(16) TW xs[kRouterSmallRows][DC];
    __shared__ int s_last;
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.y, nchunks = gridDim.y;
    const int d0 = c * DC;
    const int dn = min(DC, D - d0);                           // a multiple of VN
    const size_t xstride = (size_t)(seg > 1 ? seg : 1) * D;
    // stage the chunk of every routed row (zero beyond D and beyond Tr)
    for (int i = threadIdx.x; i < kRouterSmallRows * (DC / VN); i += blockDim.x) {
        const int r = i / (DC / VN), v = i % (DC / VN);
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (r < Tr && v * VN < dn)
            val = __ldg(reinterpret_cast<const uint4*>(x + r * xstride + d0) + v);
        reinterpret_cast<uint4*>(&xs[r][0])[v] = val;
    }
    __syncthreads();
    const int j = blockIdx.x * 8 + warp;
    if (j < n2E) {
        float w[NV][VN];
        const TW* wrow = wrm + (size_t)j * D + d0;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const int e = (v * 32 + lane) * VN;
            uint4 raw = make_uint4(0u, 0u, 0u, 0u);
            if (e < dn) raw = ldg_stream(wrow + e);
            Vec<TW>::widen(raw, w[v]);
        }
        float acc[kRouterSmallRows];
#pragma unroll
        for (int r = 0; r < kRouterSmallRows; ++r) {
            float a = 0.f;
            if (r < Tr) {
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    float xv[VN];
                    Vec<TW>::widen(reinterpret_cast<const uint4*>(&xs[r][0])[v * 32 + lane], xv);
#pragma unroll
                    for (int q = 0; q < VN; ++q) a = fmaf(w[v][q], xv[q], a);
                }
            }
            acc[r] = a;
        }
        // transposing butterfly: at step o the lanes with bit o set keep rows [o, 2o) of the
        // current numbering and send rows [0, o); after the five steps lane r holds row r
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool hi = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < o; ++i) {
                const float send = hi ? acc[i] : acc[i + o];
                const float keep = hi ? acc[i + o] : acc[i];
                acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        if (lane < Tr) L[(size_t)c * slice_stride + (size_t)lane * ldL + j] = acc[0];
    }
    if (nchunks > 1) {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = atomicAdd(arrive + blockIdx.x, 1u) == (unsigned)(nchunks - 1);
        __syncthreads();
        if (s_last) {
            __threadfence();   // the other chunks' slices are visible past this point
            if (j < n2E && lane < Tr) {
                float p[kRouterMaxChunks];
#pragma unroll
                for (int q = 0; q < kRouterMaxChunks; ++q)
                    if (q < nchunks) p[q] = __ldcg(L + (size_t)q * slice_stride + (size_t)lane * ldL + j);
                float a = p[0];
#pragma unroll
                for (int q = 1; q < kRouterMaxChunks; ++q)
                    if (q < nchunks) a += p[q];
                L[(size_t)lane * ldL + j] = a;
            }
            if (threadIdx.x == 0) arrive[blockIdx.x] = 0u;
        }
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- Top-K, softmax, mask
// One warp per routed row i (row i of L, leading dimension ldL: router logits in columns
// [0, E), mask logits in [E, 2E); `splits` K-split slices split_stride floats apart, added in
// slice order).  Lane l holds logits of experts l, l+32, ... (EPL per lane).
// K rounds of a warp arg-max under the total order (value desc, index asc) give the Top-K in
// rank order.  Lane k < K then owns slot k: g_k = exp(r_k - r_0) / sum, mask logit
// L[i][E + id_k], m = (logit >= 0) (1 for plain Top-K), g_hat = g * m, keep = m (1 for plain
// Top-K and in training mode).  The decision is written to every token of the routed row's
// segment (S = 1: the row's own token).
// Decision for one routed row, computed by one warp (all lanes return the same values except
// the per-slot ones, which lane k < K holds for slot k).
struct RowDecision {
    int id;        // lane k: expert of slot k
    float g;       // lane k: softmax gate of slot k
    float l;       // lane k: mask logit of slot k
    bool keep;     // lane k: slot's expert evaluated (kept; every slot in training mode)
    float ghat;    // lane k: g * m (the mask)
    int nkeep;     // all lanes: slots of the row whose mask is 1
    float lreg;    // all lanes: (1/K) sum_k sigmoid(l_k)
};

// Order bits of a logit: a larger value has larger bits (the float's sign-magnitude bits
// mapped to an unsigned order), and the map is one to one.
__device__ __forceinline__ uint32_t topk_ord(float v)
{
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float topk_value(uint32_t ord)
{
    return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7fffffffu) : ~ord);
}

template <int EPL>
__device__ __forceinline__ RowDecision select_row(const float* __restrict__ Li, int splits,
                                                  long long split_stride, int E, int K,
                                                  int mask_off, int lane)
{
    // the logits may arrive as split-K slices: add them in slice order
    auto logit = [&](int col) {
        float a = Li[col];
        for (int s = 1; s < splits; ++s) a += Li[s * split_stride + col];
        return a;
    };
    // Each lane sorts its experts lane, lane+32, ... once by value, descending; the sort is
    // stable, so equal values keep the lower expert first (lane padding: order 0 and an index
    // above every expert, after every real expert).  Every round then takes the warp maximum
    // of the lanes' first values, the lowest expert among the lanes holding that maximum
    // (two warp reductions), and the lane that owned it drops its first entry.  The rounds
    // yield the Top-K in rank order with ties to the lower index.
    uint32_t ord[EPL], idx[EPL];
    float mv[EPL];   // one slice: this lane's mask logits, loaded with the router logits
    if (splits == 1) {
        float rv[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            rv[j] = (e < E) ? Li[e] : 0.f;
            mv[j] = (e < E) ? Li[E + e] : 0.f;
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            ord[j] = (e < E) ? topk_ord(rv[j]) : 0u;
            idx[j] = (e < E) ? (uint32_t)e : 0xffffffffu;
        }
    } else {
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            ord[j] = (e < E) ? topk_ord(logit(e)) : 0u;
            idx[j] = (e < E) ? (uint32_t)e : 0xffffffffu;
            mv[j] = 0.f;
        }
    }
#pragma unroll
    for (int pass = 0; pass < EPL; ++pass) {
#pragma unroll
        for (int j = pass & 1; j + 1 < EPL; j += 2) {
            if (ord[j + 1] > ord[j]) {
                const uint32_t to = ord[j]; ord[j] = ord[j + 1]; ord[j + 1] = to;
                const uint32_t ti = idx[j]; idx[j] = idx[j + 1]; idx[j + 1] = ti;
            }
        }
    }
    uint32_t my_ord = 0u, my_idx = 0u;
    for (int k = 0; k < K; ++k) {
        const uint32_t best = __reduce_max_sync(0xffffffffu, ord[0]);
        const uint32_t win = __reduce_min_sync(0xffffffffu, ord[0] == best ? idx[0] : 0xffffffffu);
        if (idx[0] == win) {
#pragma unroll
            for (int j = 0; j + 1 < EPL; ++j) { ord[j] = ord[j + 1]; idx[j] = idx[j + 1]; }
            ord[EPL - 1] = 0u;
            idx[EPL - 1] = 0xffffffffu;
        }
        if (lane == k) { my_ord = best; my_idx = win; }
    }
    const int my_id = (int)my_idx;
    const float my_v = topk_value(my_ord);
    RowDecision d;
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    const bool active = lane < K;
    float ex = active ? expf(my_v - vmax) : 0.f;
    const float den = warp_sum(ex);
    d.id = my_id;
    d.g = ex / den;
    if (splits == 1) {
        // the mask logit of expert my_id is held by lane my_id % 32, entry my_id / 32
        float ml = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const float v = __shfl_sync(0xffffffffu, mv[j], my_id & 31);
            if ((my_id >> 5) == j) ml = v;
        }
        d.l = active ? ml : 0.f;
    } else {
        d.l = active ? logit(E + my_id) : 0.f;
    }
    // mask_off: 0 = BEAM mask, 1 = plain Top-K, 2 = training (every Top-K slot is evaluated,
    // so keep = 1 for the compaction, while the gate still carries the mask: g_hat = g * m)
    const bool m = active && (mask_off == 1 || d.l >= 0.f);
    d.keep = active && (mask_off != 0 || d.l >= 0.f);
    d.ghat = m ? d.g : 0.f;
    const float sg = active ? sigmoid_f(d.l) : 0.f;
    d.nkeep = __popc(__ballot_sync(0xffffffffu, m));
    d.lreg = warp_sum(sg) / (float)K;
    return d;
}

// One warp per (routed row i, layer l = blockIdx.y).  Row i of L has leading dimension ldL;
// layer l's router logits are its columns [2lE, 2lE + E), its mask logits [2lE + E, 2lE + 2E)
// (one layer: l = 0); `splits` K-split slices split_stride floats apart are added in slice
// order.  Lane l holds logits of experts l, l+32, ... (EPL per lane).
// K rounds of a warp arg-max under the total order (value desc, index asc) give the Top-K in
// rank order.  Lane k < K then owns slot k: g_k = exp(r_k - r_0) / sum, mask logit
// L[i][E + id_k], keep and g_hat as select_row gives them.  The decision is written
// to every token of the routed row's segment (S = 1: the row's own token), layer l's outputs
// out_ls ([T][K] arrays) or tok_ls ([T] arrays) elements after layer 0's.  With `active` set,
// bit e of layer l's word e/32 of active[l][nw] (nw = (E+31)/32, zeroed by the caller) is
// set for every expert e kept by one of the block's tokens (an OR: the result does not depend
// on the order of the updates).
template <int EPL>
__global__ void __launch_bounds__(256)
route_select_kernel(const float* __restrict__ L, int ldL, int splits, long long split_stride,
                    int Tr, int T, int E, int K, int seg,
                    int mask_off, int* __restrict__ topk_id, float* __restrict__ gate,
                    float* __restrict__ mlogit, uint8_t* __restrict__ keep,
                    float* __restrict__ ghat, int* __restrict__ nkeep_tok,
                    float* __restrict__ lreg_tok, long long out_ls, long long tok_ls,
                    uint32_t* __restrict__ active)
{
    __shared__ uint32_t s_act[kRouteMaxE / 32];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    const int layer = blockIdx.y;
    const int nw = (E + 31) >> 5;
    if (active) {
        if (threadIdx.x < nw) s_act[threadIdx.x] = 0u;
        __syncthreads();
    }
    if (i < Tr) {
        const RowDecision d = select_row<EPL>(L + (size_t)i * ldL + (size_t)layer * 2 * E, splits,
                                              split_stride, E, K, mask_off, lane);
        const int S = seg > 1 ? seg : 1;
        const int t0 = i * S, t1 = min(T, t0 + S);
        const size_t lo = (size_t)layer * out_ls, lt = (size_t)layer * tok_ls;
        if (S == 1) {
            if (lane < K) {
                const size_t o = lo + (size_t)t0 * K + lane;
                topk_id[o] = d.id;
                gate[o] = d.g;
                mlogit[o] = d.l;
                keep[o] = d.keep ? 1 : 0;
                ghat[o] = d.ghat;
            }
            if (lane == 0) { nkeep_tok[lt + t0] = d.nkeep; lreg_tok[lt + t0] = d.lreg; }
        } else {
            // the segment's rows [t0, t1) x K are one contiguous range of each output, holding
            // the same K slots per token: lane q writes elements q, q + 32, ..., taking slot
            // (element mod K) from the lane that owns it, so every store is a whole-warp run
            const int n = (t1 - t0) * K;
            const size_t base = lo + (size_t)t0 * K;
            // slot of element q = q mod K, carried from one pass to the next (no division)
            const int step = 32 % K;
            int src = lane % K;
            for (int q0 = 0; q0 < n; q0 += 32) {   // the same trip count on every lane
                const int q = q0 + lane;
                const int id = __shfl_sync(0xffffffffu, d.id, src);
                const float g = __shfl_sync(0xffffffffu, d.g, src);
                const float l = __shfl_sync(0xffffffffu, d.l, src);
                const int kp = __shfl_sync(0xffffffffu, d.keep ? 1 : 0, src);
                const float gh = __shfl_sync(0xffffffffu, d.ghat, src);
                if (q < n) {
                    topk_id[base + q] = id;
                    gate[base + q] = g;
                    mlogit[base + q] = l;
                    keep[base + q] = (uint8_t)kp;
                    ghat[base + q] = gh;
                }
                src += step;
                if (src >= K) src -= K;
            }
            for (int t = t0 + lane; t < t1; t += 32) {
                nkeep_tok[lt + t] = d.nkeep;
                lreg_tok[lt + t] = d.lreg;
            }
        }
        if (active && d.keep) atomicOr(&s_act[d.id >> 5], 1u << (d.id & 31));
    }
    if (active) {
        __syncthreads();
        if (threadIdx.x < nw && s_act[threadIdx.x])
            atomicOr(active + (size_t)layer * nw + threadIdx.x, s_act[threadIdx.x]);
    }
    pdl_launch_dependents();
}

}  // namespace beam
