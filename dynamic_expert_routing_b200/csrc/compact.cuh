// compact.cuh -- grouping of the kept (token, slot) pairs by expert, so that only experts with
// mask 1 are run (ai-feeds.com summary "BEAM: 用于 MoE 动态路由的二进制专家激活掩码", Method,
// output and inference acceleration: masked experts' FFNs are skipped).
//
// Deterministic and free of atomics: the order of perm is fixed by (expert asc, token asc).
//   1. compact_bits: per 32-token chunk c and expert e, a warp ballot gives the word
//      bits[e][c] whose bit b says "token 32c+b keeps a slot routed to e".
//   2. compact_scan (one CTA): per expert, popcount prefix sums over chunks -> chunk_base;
//      counts; exclusive scan over experts -> offsets; the list of active groups; and the
//      forward's statistics, reduced in a fixed tree order.
//   3. compact_scatter_gather: the position of pair (t, k) routed to e is
//      offsets[e] + chunk_base[e][t/32] + popc(bits[e][t/32] & lanes_below(t%32)); it writes
//      perm / inv and copies x[t] into row pos of X_perm.
#pragma once
#include "common.cuh"

namespace beam {

constexpr int kMaxE = 256;

__global__ void __launch_bounds__(256)
compact_bits_kernel(const int* __restrict__ topk_id, const uint8_t* __restrict__ keep, int T,
                    int K, int E, int nch, uint32_t* __restrict__ bits)
{
    __shared__ uint32_t smask[8][kMaxE / 32][32];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x * 8 + warp;
    if (c < nch) {
        const int nw = (E + 31) >> 5;
        for (int w = 0; w < nw; ++w) smask[warp][w][lane] = 0u;
        const int t = c * 32 + lane;
        if (t < T) {
            for (int k = 0; k < K; ++k) {
                size_t o = (size_t)t * K + k;
                if (keep[o]) {
                    int e = topk_id[o];
                    smask[warp][e >> 5][lane] |= 1u << (e & 31);
                }
            }
        }
        __syncwarp();
        for (int w = 0; w < nw; ++w) {
            const uint32_t mine = smask[warp][w][lane];
            uint32_t word = 0;
#pragma unroll 4
            for (int b = 0; b < 32; ++b) {
                uint32_t bal = __ballot_sync(0xffffffffu, (mine >> b) & 1u);
                if (lane == b) word = bal;
            }
            const int e = w * 32 + lane;
            if (e < E) bits[(size_t)e * nch + c] = word;
        }
    }
    pdl_launch_dependents();
}

__global__ void __launch_bounds__(1024)
compact_scan_kernel(const uint32_t* __restrict__ bits, int nch, int E, int T,
                    const int* __restrict__ nkeep_tok, const float* __restrict__ lreg_tok,
                    int* __restrict__ counts, int* __restrict__ offsets,
                    int* __restrict__ chunk_base, Group* __restrict__ groups,
                    int* __restrict__ n_groups, DevStats* __restrict__ stats)
{
    __shared__ int s_counts[kMaxE];
    __shared__ long long s_keep[32];
    __shared__ double s_lreg[32];
    __shared__ int s_zero[32];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;

    // 1. per-expert chunk prefix sums
    for (int e = warp; e < E; e += nwarps) {
        int running = 0;
        for (int c0 = 0; c0 < nch; c0 += 32) {
            const int c = c0 + lane;
            const int p = (c < nch) ? __popc(bits[(size_t)e * nch + c]) : 0;
            int incl = p;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (c < nch) chunk_base[(size_t)e * nch + c] = running + incl - p;
            running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) { s_counts[e] = running; counts[e] = running; }
    }
    __syncthreads();

    // 2. offsets and the active-group list (warp 0; each lane owns 8 consecutive experts)
    if (warp == 0) {
        int loc[8], act[8];
        int sum = 0, nact = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int e = lane * 8 + j;
            loc[j] = (e < E) ? s_counts[e] : 0;
            act[j] = loc[j] > 0;
            sum += loc[j];
            nact += act[j];
        }
        int incl = sum, inca = nact;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, incl, o);
            int na = __shfl_up_sync(0xffffffffu, inca, o);
            if (lane >= o) { incl += n; inca += na; }
        }
        int run = incl - sum, runa = inca - nact;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int e = lane * 8 + j;
            if (e < E) {
                offsets[e] = run;
                if (act[j]) {
                    Group g;
                    g.row0 = run; g.m = loc[j]; g.expert = e; g.pad = 0;
                    groups[runa] = g;
                    ++runa;
                }
            }
            run += loc[j];
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const int tact = __shfl_sync(0xffffffffu, inca, 31);
        if (lane == 0) {
            offsets[E] = total;
            *n_groups = tact;
            stats->n_kept = total;
            stats->n_active = tact;
        }
    }

    // 3. statistics: strided per-thread sums, then a fixed-shape tree
    long long ks = 0;
    double ls = 0.0;
    int nz = 0;
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        int nk = nkeep_tok[t];
        ks += nk;
        ls += (double)lreg_tok[t];
        nz += (nk == 0);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ks += __shfl_xor_sync(0xffffffffu, ks, o);
        ls += __shfl_xor_sync(0xffffffffu, ls, o);
        nz += __shfl_xor_sync(0xffffffffu, nz, o);
    }
    if (lane == 0) { s_keep[warp] = ks; s_lreg[warp] = ls; s_zero[warp] = nz; }
    __syncthreads();
    if (warp == 0) {
        ks = lane < nwarps ? s_keep[lane] : 0;
        ls = lane < nwarps ? s_lreg[lane] : 0.0;
        nz = lane < nwarps ? s_zero[lane] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ks += __shfl_xor_sync(0xffffffffu, ks, o);
            ls += __shfl_xor_sync(0xffffffffu, ls, o);
            nz += __shfl_xor_sync(0xffffffffu, nz, o);
        }
        if (lane == 0) {
            stats->keep_sum = ks;
            stats->lreg_sum = ls;
            stats->n_all_masked = nz;
            stats->tokens = T;
            stats->err = 0;
        }
    }
    pdl_launch_dependents();
}

// One warp per (token, slot).  Kept slots get their position, write perm / inv and copy the
// token's activation row into X_perm; masked slots write inv = -1.
template <typename TW>
__global__ void __launch_bounds__(256)
compact_scatter_gather_kernel(const int* __restrict__ topk_id, const uint8_t* __restrict__ keep,
                              int T, int K, int D, int nch, const uint32_t* __restrict__ bits,
                              const int* __restrict__ offsets, const int* __restrict__ chunk_base,
                              const TW* __restrict__ x, int* __restrict__ perm,
                              int* __restrict__ inv, TW* __restrict__ xperm, int gather)
{
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long i = (long long)blockIdx.x * 8 + warp;
    if (i < (long long)T * K) {
        const int t = (int)(i / K);
        int pos = -1;
        if (keep[i]) {
            const int e = topk_id[i];
            const int c = t >> 5, b = t & 31;
            const uint32_t w = bits[(size_t)e * nch + c];
            pos = offsets[e] + chunk_base[(size_t)e * nch + c] + __popc(w & ((1u << b) - 1u));
        }
        if (lane == 0) {
            inv[i] = pos;
            if (pos >= 0) perm[pos] = (int)i;
        }
        if (gather && pos >= 0) {
            const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * D);
            uint4* dst = reinterpret_cast<uint4*>(xperm + (size_t)pos * D);
            const int nv = D * (int)sizeof(TW) / 16;
            for (int v = lane; v < nv; v += 32) dst[v] = src[v];
        }
    }
    pdl_launch_dependents();
}

}  // namespace beam
