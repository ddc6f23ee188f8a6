// decode_fused.cuh -- the whole BEAM layer forward for a batch of at most kSmallT tokens in one
// persistent launch: router logits, Top-K / softmax / mask (BEAM article on aitrends.kr,
// four-step pipeline, Steps 1-3), compaction, the kept experts' SwiGLU with the shared experts
// (Step 4, limitation (C)) and the fixed-order combine.  A decode forward has about 10-55 us of
// roofline work; as separate launches every kernel boundary costs a drain and a ramp, so here
// the phases are separated by grid barriers instead:
//   1. logits: (column, 256..512-element chunk of D) items over all warps of the grid, written
//      as per-chunk partial slices L[c][row][2E] (the selection adds them in chunk order);
//   2. routing and compaction: every block runs the small-batch routing on the slices (one
//      block publishes the results), then the blocks share the copy of the kept rows to X_perm;
//   3. gate/up of the kept groups and the shared group: the tcgen05 grouped GEMM, split K,
//      f32 partial slices;
//   4. SwiGLU of the summed partials (slices in order) -> fp16 H;
//   5. down projection: the grouped GEMM again, split K, f32 partial slices;
//   6. combine: y[t] = sum over the token's kept slots in rank order of g_hat * Y (slices in
//      order) + the shared term.
// All blocks are resident at once (a cooperative launch, one block per SM), so the barriers
// cannot wait on a block that is not running; each wait is bounded, and an expiry raises the
// error word and makes every later phase a no-op.
// Measured on B200 it is slower than the same forward as separate kernels chained with
// programmatic dependent launch and replayed from a CUDA graph (e.g. 95 against 86 us for the
// Mixtral-like layer at one token): the router and routing phases with their barriers take
// about 20 us, where the chained kernels overlap each launch's set-up with the previous one.
// It is therefore opt-in (BEAM_FUSED_DECODE).
#pragma once
#include "compact.cuh"
#include "tc_experts.cuh"

namespace beam {

struct FusedDecodeParams {
    tc::TcParams g1;     // gate/up, split-K f32 partials (routed + shared)
    tc::TcParams g2;     // down, split-K f32 partials (routed + shared)
    const __nv_bfloat16* x;
    const __nv_bfloat16* wrm;   // [n2E][D]
    float* L;                   // logit slices [lchunks][Tr][n2E]
    int lchunk, lchunks;        // elements of D per slice, number of slices
    int T, Tr, seg, D, E, K, n2E, mask_off;
    // routing outputs and compaction
    int* topk_id; float* gate; float* mlogit; uint8_t* keep; float* ghat;
    int* nkeep_tok; float* lreg_tok; int* counts; int* offsets; Group* groups; int* n_groups;
    DevStats* stats; int* perm; int* inv; Group* tile_group; __nv_bfloat16* xperm;
    // SwiGLU finish
    int F, Fsh;
    __half* h; __half* hsh;
    // combine
    float* y;
    unsigned* grid_bar;         // zero at launch
    int* err;
};

constexpr int ERR_GRID_TIMEOUT = 0x200;

// Grid barrier number `round` (1, 2, ...): every block arrives once per round on a counter that
// starts at zero, and waits for gridDim.x * round arrivals.  Memory written before it by any
// block is visible to every block after it (a device-scope fence on both sides).  The wait is
// bounded; on expiry the block raises its abort flag and the error word, and returns.
__device__ __forceinline__ void grid_barrier(unsigned* counter, unsigned round,
                                             volatile int* abort_flag, int* err)
{
    __syncthreads();
    if (threadIdx.x == 0 && !*abort_flag) {
        __threadfence();
        atomicAdd(counter, 1u);
        const unsigned target = round * gridDim.x;
        const unsigned long long t0 = tc::globaltimer();
        while (true) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
            if (v >= target) break;
            if (tc::globaltimer() - t0 > tc::kWaitLimitNs) {
                *abort_flag = 1;
                atomicOr(err, ERR_GRID_TIMEOUT);
                break;
            }
        }
        __threadfence();
    }
    __syncthreads();
}

// Writes of ordinary stores that a later TMA copy (the async proxy) of another block reads.
__device__ __forceinline__ void fence_for_tma_readers()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

template <int EPL>
__global__ void __launch_bounds__(tc::kThreads, 1)
fused_decode_kernel(const __grid_constant__ FusedDecodeParams P)
{
    extern __shared__ uint8_t smem_raw[];
    const tc::GemmSmem sm = tc::gemm_smem(smem_raw);
    if (threadIdx.x == 0) {
        tc::tma_prefetch_desc(&P.g1.a_routed); tc::tma_prefetch_desc(&P.g1.b_routed);
        tc::tma_prefetch_desc(&P.g1.a_shared); tc::tma_prefetch_desc(&P.g1.b_shared);
        tc::tma_prefetch_desc(&P.g2.a_routed); tc::tma_prefetch_desc(&P.g2.b_routed);
        tc::tma_prefetch_desc(&P.g2.a_shared); tc::tma_prefetch_desc(&P.g2.b_shared);
    }
    const uint32_t tmem_base = tc::gemm_setup(sm);
    volatile int* abort_flag = sm.abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    const int gwarp = blockIdx.x * nwarps + warp, gwarps = gridDim.x * nwarps;
    unsigned round = 0;

    // 1. logit slices: item = (column j, chunk c); a warp covers the chunk with 16-byte loads of
    // the weight row and of every routed token row, one partial per row, reduced across lanes
    {
        const size_t xstride = (size_t)(P.seg > 1 ? P.seg : 1) * P.D;
        const int items = P.n2E * P.lchunks;
        for (int it = gwarp; it < items; it += gwarps) {
            const int j = it % P.n2E, c = it / P.n2E;
            const int d0 = c * P.lchunk, d1 = min(P.D, d0 + P.lchunk);
            float acc[kSmallT];
#pragma unroll
            for (int r = 0; r < kSmallT; ++r) acc[r] = 0.f;
#pragma unroll 4
            for (int d = d0 + lane * 8; d < d1; d += 256) {
                float w[8];
                Vec<__nv_bfloat16>::widen(ldg_stream(P.wrm + (size_t)j * P.D + d), w);
#pragma unroll
                for (int r = 0; r < kSmallT; ++r) {
                    if (r < P.Tr) {
                        float xv[8];
                        Vec<__nv_bfloat16>::widen(__ldg(reinterpret_cast<const uint4*>(P.x + r * xstride + d)), xv);
                        float s = 0.f;
#pragma unroll
                        for (int v = 0; v < 8; ++v) s = fmaf(w[v], xv[v], s);
                        acc[r] += s;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kSmallT; ++r) {
                if (r < P.Tr) {
                    const float s = warp_sum(acc[r]);
                    if (lane == 0) P.L[((size_t)c * P.Tr + r) * P.n2E + j] = s;
                }
            }
        }
    }
    grid_barrier(P.grid_bar, ++round, abort_flag, P.err);

    // 2. routing and compaction in every block (block 0 publishes), then the row copies
    {
        SmallScratch& sc = *reinterpret_cast<SmallScratch*>(sm.gbase);  // the idle stage ring
        if (!*abort_flag)
            route_compact_small_body<EPL>(sc, blockIdx.x == 0, P.L, P.n2E, P.lchunks,
                                          (long long)P.Tr * P.n2E, P.Tr, P.T, P.E, P.K, P.seg,
                                          P.mask_off, P.topk_id, P.gate, P.mlogit, P.keep, P.ghat,
                                          P.nkeep_tok, P.lreg_tok, P.counts, P.offsets, P.groups,
                                          P.n_groups, P.stats, P.perm, P.inv, P.tile_group);
        if (!*abort_flag) gather_small_rows(sc, P.E, P.K, P.D, P.x, P.xperm, gwarp, gwarps);
        fence_for_tma_readers();
        // the scratch lives in the stage ring, which TMA (the async proxy) writes next
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    grid_barrier(P.grid_bar, ++round, abort_flag, P.err);

    // 3. gate/up GEMM
    tc::RoleState rs;
    rs.ok = !*abort_flag;
    tc::gemm_roles<tc::EPI_STORE_F32, 1, tc::MODE_PLAIN>(P.g1, sm, tmem_base, rs);
    grid_barrier(P.grid_bar, ++round, abort_flag, P.err);

    // 4. SwiGLU of the gate/up partial slices (added in slice order) -> fp16 H
    if (!*abort_flag) {
        const int nrow = __ldcg(P.offsets + P.E);
        const long long nr = (long long)nrow * P.F;
        const long long ns = (long long)P.g1.shared_rows * P.Fsh;
        const int splits = P.g1.k_splits_routed;
        for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < nr + ns;
             i += (long long)gridDim.x * blockDim.x) {
            const bool shared = i >= nr;
            const long long jj = shared ? i - nr : i;
            const int FF = shared ? P.Fsh : P.F;
            const long long r = jj / FF;
            const int f = (int)(jj % FF);
            const long long b = r * 2 * FF + (long long)(f >> 7) * 256 + (f & 127);
            const float* src = static_cast<const float*>(shared ? P.g1.out_shared : P.g1.out_routed);
            const long long st = shared ? P.g1.split_stride_shared : P.g1.split_stride_routed;
            float g = 0.f, u = 0.f;
            for (int q = 0; q < splits; ++q) {
                g += __ldcg(src + q * st + b);
                u += __ldcg(src + q * st + b + 128);
            }
            const float hv = silu_f(g) * u;
            if (fp16_out_of_range(hv)) atomicOr(P.err, ERR_FP16_RANGE);
            (shared ? P.hsh : P.h)[r * FF + f] = __float2half_rn(hv);
        }
        fence_for_tma_readers();
    }
    grid_barrier(P.grid_bar, ++round, abort_flag, P.err);

    // 5. down GEMM
    rs.ok = rs.ok && !*abort_flag;
    tc::gemm_roles<tc::EPI_STORE_F32, 0, tc::MODE_PLAIN>(P.g2, sm, tmem_base, rs);
    grid_barrier(P.grid_bar, ++round, abort_flag, P.err);

    // 6. combine: thread = (token, 4 columns); slots in rank order, split slices in order
    if (!*abort_flag) {
        const int D4 = P.D >> 2;
        const float* yr = static_cast<const float*>(P.g2.out_routed);
        const float* ys = static_cast<const float*>(P.g2.out_shared);
        const long long sr4 = P.g2.split_stride_routed >> 2, ss4 = P.g2.split_stride_shared >> 2;
        const int sr = P.g2.k_splits_routed, ss = P.g2.k_splits_shared;
        for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)P.T * D4;
             i += (long long)gridDim.x * blockDim.x) {
            const int t = (int)(i / D4), c = (int)(i % D4);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < P.K; ++k) {
                const int p = __ldcg(P.inv + (size_t)t * P.K + k);
                if (p < 0) continue;
                const float g = __ldcg(P.ghat + (size_t)t * P.K + k);
                float4 v = __ldcg(reinterpret_cast<const float4*>(yr) + (size_t)p * D4 + c);
                for (int q = 1; q < sr; ++q) {
                    const float4 w = __ldcg(reinterpret_cast<const float4*>(yr) + q * sr4 + (size_t)p * D4 + c);
                    v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                }
                acc.x = fmaf(g, v.x, acc.x); acc.y = fmaf(g, v.y, acc.y);
                acc.z = fmaf(g, v.z, acc.z); acc.w = fmaf(g, v.w, acc.w);
            }
            if (P.g2.shared_rows > 0) {
                for (int q = 0; q < ss; ++q) {
                    const float4 w = __ldcg(reinterpret_cast<const float4*>(ys) + q * ss4 + (size_t)t * D4 + c);
                    acc.x += w.x; acc.y += w.y; acc.z += w.z; acc.w += w.w;
                }
            }
            __stcs(reinterpret_cast<float4*>(P.y) + (size_t)t * D4 + c, acc);
        }
    }
    tc::gemm_teardown(sm, tmem_base, P.err);
}

}  // namespace beam
