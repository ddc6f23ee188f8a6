// tc_down_astat.cuh -- the down projection of the routed experts (Step 4 of the BEAM pipeline,
// BEAM article on aitrends.kr, masked aggregation) for layers whose expert intermediate size is
// small (F <= 256, e.g. the fine-grained 212-expert shape of "Stepped MoE: Segment-Level Routing
// with Configurable Inference Complexity"), on the tcgen05 tensor cores.
//
// With F <= 256 an output tile has at most 4 k-steps: the grouped GEMM's 4-stage ring then runs at
// most one tile ahead and every tile waits out a full round trip of its copies (its tensor pipe
// sat at about 12 % on the fine-grained layer).  Here the work unit is a group's 128-row M-tile
// with ALL of its N-tiles: the unit's H rows (the A operand, at most 4 slabs of 128 x 64 fp16)
// are loaded once into a stationary shared-memory region and reused for every N-tile, while
// the weight tiles (B, 256 rows x 64) stream through a 4-stage ring continuously across N-tiles
// and units (they do not depend on H).  Units are numbered like the grouped GEMM's M-tiles
// (across the groups, through the tile -> group table), so the M-tiles of one expert run on
// neighbouring CTAs at the same time and share its weight tiles through L2.
//   warp 0 lane 0: TMA (A slabs once per unit after the previous unit's MMAs released them;
//                  B tiles through the ring);
//   warp 1 lane 0: tcgen05.mma (kind::f16, fp32 accumulators in TMEM, two 256-column buffers);
//   warps 2..9:    epilogue, TMEM -> fp16 output rows (the grouped GEMM's f16-store epilogue).
// Every wait is bounded like the grouped GEMM's; on expiry the CTA records the error, drains its
// copies and MMAs, frees TMEM and returns.
#pragma once
#include "tc_experts.cuh"

namespace beam {
namespace tc {

constexpr int AS_MAX_KSTEPS = 4;                       // F <= 256
constexpr int AS_STAGES = 4;                           // B-only stages
constexpr int AS_SMEM_BYTES = AS_MAX_KSTEPS * A_BYTES + AS_STAGES * B_BYTES +
                              kEpiWarps * EPI_WARP_BYTES + 1024 /*alignment*/ + 256 /*barriers*/;
static_assert(AS_SMEM_BYTES <= 232448, "the A-stationary down kernel must fit 227 KB of shared memory");

struct AstatSmem {
    uint32_t a_base, b_base;   // shared-window addresses (1024-aligned)
    float* epi_buf;
    uint32_t bar0;
    uint32_t* tmem_slot;
    volatile int* abort_flag;
    __device__ uint32_t full_bar(int s) const { return bar0 + 8u * s; }
    __device__ uint32_t empty_bar(int s) const { return bar0 + 8u * (AS_STAGES + s); }
    __device__ uint32_t tfull_bar(int a) const { return bar0 + 8u * (2 * AS_STAGES + a); }
    __device__ uint32_t tempty_bar(int a) const { return bar0 + 8u * (2 * AS_STAGES + 2 + a); }
    __device__ uint32_t afull_bar() const { return bar0 + 8u * (2 * AS_STAGES + 4); }
    __device__ uint32_t aempty_bar() const { return bar0 + 8u * (2 * AS_STAGES + 5); }
    __device__ uint32_t drain_bar() const { return bar0 + 8u * (2 * AS_STAGES + 6); }
};

__device__ __forceinline__ AstatSmem astat_smem(uint8_t* smem_raw)
{
    AstatSmem m;
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    m.a_base = base;
    m.b_base = base + AS_MAX_KSTEPS * A_BYTES;
    m.epi_buf = reinterpret_cast<float*>(gbase + AS_MAX_KSTEPS * A_BYTES + AS_STAGES * B_BYTES);
    const uint32_t off_bar = AS_MAX_KSTEPS * A_BYTES + AS_STAGES * B_BYTES + kEpiWarps * EPI_WARP_BYTES;
    m.bar0 = base + off_bar;
    m.tmem_slot = reinterpret_cast<uint32_t*>(gbase + off_bar + 8 * (2 * AS_STAGES + 7));
    m.abort_flag = reinterpret_cast<volatile int*>(m.tmem_slot + 1);
    return m;
}

// p: the routed down problem (a_routed = H [rows][F] fp16 in 128-row boxes, b_routed = W_d
// [E * D][F] fp16 in 256-row boxes, out_routed = Y [rows][D] fp16, ld_routed = D,
// n_tiles_routed = D / 256, k_steps_routed = F / 64 <= AS_MAX_KSTEPS, b_rows_per_expert = D,
// tile_group / n_groups from the compaction).  Launched with AS_SMEM_BYTES of dynamic shared
// memory and kThreads threads.
__global__ void __launch_bounds__(kThreads, 1)
tc_down_astat_kernel(const __grid_constant__ TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    const AstatSmem sm = astat_smem(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        tma_prefetch_desc(&p.a_routed);
        tma_prefetch_desc(&p.b_routed);
        for (int s = 0; s < AS_STAGES; ++s) { mbar_init(sm.full_bar(s), 1); mbar_init(sm.empty_bar(s), 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(sm.tfull_bar(a), 1); mbar_init(sm.tempty_bar(a), kEpiWarps); }
        mbar_init(sm.afull_bar(), 1);
        mbar_init(sm.aempty_bar(), 1);
        mbar_init(sm.drain_bar(), 1);
        *sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(sm.tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;
    pdl_wait();   // H, the group table and the tile table come from the previous kernels
    volatile int* abort_flag = sm.abort_flag;
    const int total_mt = p.n_groups[1];
    const int NT = p.n_tiles_routed, KS = p.k_steps_routed;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        // Unit u's first ring-full of B tiles is issued before waiting for unit u - 1's MMAs to
        // release the A slabs, so the weight stream does not stop at unit boundaries.
        int s = 0;
        uint32_t ph = 0, ae = 0;
        bool ok = true;
        bool pend[AS_STAGES] = {false, false, false, false};
        uint32_t pend_ph[AS_STAGES] = {0u, 0u, 0u, 0u};
        int a_issued = 0;   // A loads issued: load i completes phase i of the A barrier
        const int nb = NT * KS;
        for (int u = blockIdx.x; ok && u < total_mt; u += gridDim.x) {
            const Group G = p.tile_group[u];
            const int arow = G.row0 + (u - G.mt0) * BM;
            const int early = a_issued == 0 ? 0 : min(AS_STAGES, nb - 1);
            for (int b = 0; ok && b < nb; ++b) {
                if (b == early) {
                    if (a_issued > 0) {
                        // the previous unit's MMAs have finished reading the A slabs
                        if (!mbar_wait(sm.aempty_bar(), ae, abort_flag)) { ok = false; break; }
                        ae ^= 1u;
                    }
                    mbar_expect_tx(sm.afull_bar(), (uint32_t)(KS * A_BYTES));
                    for (int k = 0; k < KS; ++k)
                        tma_load_2d(sm.a_base + k * A_BYTES, &p.a_routed, sm.afull_bar(), k * BK, arow);
                    ++a_issued;
                }
                const int n = b / KS, k = b % KS;
                if (!mbar_wait(sm.empty_bar(s), ph ^ 1u, abort_flag)) { ok = false; break; }
                mbar_expect_tx(sm.full_bar(s), B_BYTES);
                tma_load_2d(sm.b_base + s * B_BYTES, &p.b_routed, sm.full_bar(s), k * BK,
                            G.expert * p.b_rows_per_expert + n * BN);
                pend[s] = true;
                pend_ph[s] = ph;
                if (++s == AS_STAGES) { s = 0; ph ^= 1u; }
            }
        }
        if (!ok) {
            // drain: let every copy this thread issued land before the CTA can exit
            for (int i = 0; i < AS_STAGES; ++i) {
                if (!pend[i]) continue;
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(sm.full_bar(i), pend_ph[i]) && globaltimer() - t0 < kWaitLimitNs) {}
            }
            if (a_issued > 0) {
                const unsigned long long t0 = globaltimer();
                while (!mbar_try_wait(sm.afull_bar(), (uint32_t)((a_issued - 1) & 1)) &&
                       globaltimer() - t0 < kWaitLimitNs) {}
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ MMA issuer
        int s = 0, acc = 0;
        uint32_t ph = 0, aph = 0, af = 0;
        bool ok = true, issued = false;
        constexpr uint32_t idesc = make_idesc(0);   // f16 x f16 -> f32, N = 256
        for (int u = blockIdx.x; ok && u < total_mt; u += gridDim.x) {
            if (!mbar_wait(sm.afull_bar(), af, abort_flag)) { ok = false; break; }
            af ^= 1u;
            tc_fence_after();
            for (int n = 0; ok && n < NT; ++n) {
                if (!mbar_wait(sm.tempty_bar(acc), aph ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int k = 0; k < KS; ++k) {
                    if (!mbar_wait(sm.full_bar(s), ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sm.a_base + k * A_BYTES);
                    const uint64_t bd = sw128_desc(sm.b_base + s * B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma_f16(d_tmem, ad + 2ull * kk, bd + 2ull * kk, idesc,
                                   (k != 0 || kk != 0) ? 1u : 0u);
                    issued = true;
                    tc_commit(sm.empty_bar(s));
                    if (++s == AS_STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(sm.tfull_bar(acc));
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
            if (!ok) break;
            tc_commit(sm.aempty_bar());   // completes when this unit's MMAs have read A
        }
        if (!ok && issued) {
            tc_commit(sm.drain_bar());
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(sm.drain_bar(), 0) && globaltimer() - t0 < kWaitLimitNs) {}
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (TMEM -> fp16 rows)
        int acc = 0;
        uint32_t aph = 0;
        bool ok = true, bad = false;
        const int lb = 32 * (warp & 3);
        const int warp_e = warp - 2;
        const int half = warp_e / 4;
        float* buf = sm.epi_buf + warp_e * (32 * EPI_PITCH);
        __half* out = static_cast<__half*>(p.out_routed);
        const int ld = p.ld_routed;
        for (int u = blockIdx.x; ok && u < total_mt; u += gridDim.x) {
            const Group G = p.tile_group[u];
            const int r0 = (u - G.mt0) * BM + lb;
            const int nrows = max(0, min(32, G.m - r0));
            const size_t row_base = (size_t)(G.row0 + r0);
            for (int n = 0; n < NT; ++n) {
                if (!mbar_wait(sm.tfull_bar(acc), aph, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tbase = tmem_base + ((uint32_t)lb << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
                for (int j = half * (BN / 64); j < (half + 1) * (BN / 64); ++j) {
                    float v[32];
                    tmem_ld32(tbase + 32 * j, v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) buf[lane * EPI_PITCH + i] = v[i];
                    __syncwarp();
                    store_rows_f16(buf, out + row_base * ld + (size_t)n * BN + 32 * j, ld, nrows, lane, bad);
                    __syncwarp();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sm.tempty_bar(acc));
                if (++acc == 2) { acc = 0; aph ^= 1u; }
            }
        }
        if (bad) atomicOr(p.err, ERR_FP16_RANGE);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *sm.abort_flag) atomicOr(p.err, ERR_TC_TIMEOUT);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
    }
    pdl_launch_dependents();
}

}  // namespace tc
}  // namespace beam
