// compact.cuh -- grouping of the kept (token, slot) pairs by expert, so that only experts with
// mask 1 are run (ai-feeds.com summary "BEAM: 用于 MoE 动态路由的二进制专家激活掩码", Method,
// output and inference acceleration: masked experts' FFNs are skipped).
//
// Deterministic: the order of perm is fixed by (expert asc, token asc), and no atomic decides
// any order (the scan's one atomic only elects the CTA that finishes).
//   1. compact_bits: per 32-token chunk c and expert e, a warp ballot gives the word
//      bits[e][c] whose bit b says "token 32c+b keeps a slot routed to e".
//   2. compact_scan: per expert (one warp each), popcount prefix sums over chunks ->
//      chunk_base and counts; then the last CTA: exclusive scan over experts -> offsets, the
//      list of active groups, and the forward's statistics, reduced in a fixed order.
//   3. compact_scatter_gather: the position of pair (t, k) routed to e is
//      offsets[e] + chunk_base[e][t/32] + popc(bits[e][t/32] & lanes_below(t%32)); it writes
//      perm / inv and copies x[t] into row pos of X_perm.
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace beam {

constexpr int kMaxE = kRouteMaxE;

// One warp copies a row of nv 16-byte vectors, 8 vectors per lane in flight at a time (all
// loads of a batch are issued before its stores).
__device__ __forceinline__ void copy_row_warp(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                              int nv, int lane)
{
    for (int v0 = 0; v0 < nv; v0 += 32 * 8) {
        uint4 r[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < nv) r[u] = __ldg(src + v);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int v = v0 + u * 32 + lane;
            if (v < nv) dst[v] = r[u];
        }
    }
}

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
            // a token's K slots are contiguous: with K = 4, 8 or 16, read them as 16-byte vectors
            // (all loads in flight at once); otherwise slot by slot
            if (K == 4 || K == 8 || K == 16) {
                const size_t o = (size_t)t * K;
                uint32_t kp[4];
                if (K == 16) {
                    const uint4 v = *reinterpret_cast<const uint4*>(keep + o);
                    kp[0] = v.x; kp[1] = v.y; kp[2] = v.z; kp[3] = v.w;
                } else if (K == 8) {
                    const uint2 v = *reinterpret_cast<const uint2*>(keep + o);
                    kp[0] = v.x; kp[1] = v.y; kp[2] = kp[3] = 0u;
                } else {
                    kp[0] = *reinterpret_cast<const uint32_t*>(keep + o); kp[1] = kp[2] = kp[3] = 0u;
                }
                int id[16];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (q * 4 < K) {
                        const int4 v = *reinterpret_cast<const int4*>(topk_id + o + q * 4);
                        id[4 * q] = v.x; id[4 * q + 1] = v.y; id[4 * q + 2] = v.z; id[4 * q + 3] = v.w;
                    }
                }
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    if (k < K && ((kp[k >> 2] >> (8 * (k & 3))) & 0xffu)) {
                        const int e = id[k];
                        smask[warp][e >> 5][lane] |= 1u << (e & 31);
                    }
                }
            } else {
                for (int k = 0; k < K; ++k) {
                    const size_t o = (size_t)t * K + k;
                    if (keep[o]) {
                        const int e = topk_id[o];
                        smask[warp][e >> 5][lane] |= 1u << (e & 31);
                    }
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

// compact_scan runs on several CTAs of kScanWarps warps: warp g of the grid scans the chunk
// words of experts g, g + (grid warps), ...; every thread adds the statistics of a strided set
// of tokens, and each CTA writes its sums to part[blockIdx.x].  The last CTA to arrive (an
// atomic counter decides which CTA that is, never the order of any sum) builds the offsets,
// the active-group list, the tile table and the statistics from the per-expert counts and
// the per-CTA sums, taken in index order.
constexpr int kScanWarps = 8;
constexpr int kScanMaxCtas = 64;

struct ScanPart {
    long long keep;   // kept slots of this CTA's tokens
    double lreg;      // their L_reg terms
    int zero;         // their tokens with no kept slot
    int pad;
};

// CTAs of one compact_scan launch: one warp per expert, and one thread per 2048 tokens at most
// for the statistics.
__host__ __device__ __forceinline__ int scan_ctas(int E, int T)
{
    int n = (E + kScanWarps - 1) / kScanWarps;
    const int nt = (T + 2047) / 2048;
    if (nt > n) n = nt;
    return n < 1 ? 1 : (n > kScanMaxCtas ? kScanMaxCtas : n);
}

__global__ void __launch_bounds__(32 * kScanWarps)
compact_scan_kernel(const uint32_t* __restrict__ bits, int nch, int E, int T,
                    const int* __restrict__ nkeep_tok, const float* __restrict__ lreg_tok,
                    int* __restrict__ counts, int* __restrict__ offsets,
                    int* __restrict__ chunk_base, Group* __restrict__ groups,
                    int* __restrict__ n_groups, DevStats* __restrict__ stats,
                    int* __restrict__ tail_cnt, int n_tail_cnt, Group* __restrict__ tile_group,
                    ScanPart* __restrict__ part, unsigned* __restrict__ arrive)
{
    __shared__ int s_counts[kMaxE];
    __shared__ Group s_groups[kMaxE];
    __shared__ int s_ngroups;
    __shared__ long long s_keep[kScanWarps];
    __shared__ double s_lreg[kScanWarps];
    __shared__ int s_zero[kScanWarps];
    __shared__ int s_last;
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthreads = gridDim.x * blockDim.x;
    const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
    // the arrival counters of the grouped GEMMs' tail split start every forward at zero
    for (int i = gtid; i < n_tail_cnt; i += nthreads) tail_cnt[i] = 0;

    // 0. per-thread sums of the token statistics, issued first so their loads overlap the rest
    long long ks = 0;
    double ls = 0.0;
    int nz = 0;
#pragma unroll 4
    for (int t = gtid; t < T; t += nthreads) {
        const int nk = nkeep_tok[t];
        ks += nk;
        ls += (double)lreg_tok[t];
        nz += (nk == 0);
    }

    // 1. per-expert chunk prefix sums: 8 words of 32 chunks loaded together, then scanned
    for (int e = blockIdx.x * kScanWarps + warp; e < E; e += gridDim.x * kScanWarps) {
        int run = 0;
        for (int c0 = 0; c0 < nch; c0 += 32 * 8) {
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + 32 * u + lane;
                w[u] = (c < nch) ? bits[(size_t)e * nch + c] : 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + 32 * u + lane;
                const int pc = __popc(w[u]);
                int incl = pc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int n = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += n;
                }
                if (c < nch) chunk_base[(size_t)e * nch + c] = run + incl - pc;
                run += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (lane == 0) counts[e] = run;
    }

    // 2. this CTA's statistics: warp trees, then the warps in index order
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        ks += __shfl_xor_sync(0xffffffffu, ks, o);
        ls += __shfl_xor_sync(0xffffffffu, ls, o);
        nz += __shfl_xor_sync(0xffffffffu, nz, o);
    }
    if (lane == 0) { s_keep[warp] = ks; s_lreg[warp] = ls; s_zero[warp] = nz; }
    __syncthreads();
    if (threadIdx.x == 0) {
        ScanPart q;
        q.keep = 0; q.lreg = 0.0; q.zero = 0; q.pad = 0;
        for (int w = 0; w < kScanWarps; ++w) { q.keep += s_keep[w]; q.lreg += s_lreg[w]; q.zero += s_zero[w]; }
        part[blockIdx.x] = q;
    }

    // 3. the last CTA to arrive finishes; counts and partial sums are visible to it
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(arrive, 1u) == gridDim.x - 1);
    __syncthreads();
    if (!s_last) {
        pdl_launch_dependents();
        return;
    }
    __threadfence();
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_counts[e] = __ldcg(counts + e);
    __syncthreads();

    // 4. offsets and the active-group list (warp 0; each lane owns 8 consecutive experts)
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
        // tiles of kGroupTileRows rows: this lane's experts, then an exclusive scan over lanes
        int mtl = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) mtl += (loc[j] + kGroupTileRows - 1) / kGroupTileRows;
        int inclm = mtl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, inclm, o);
            if (lane >= o) inclm += n;
        }
        int run = incl - sum, runa = inca - nact, runm = inclm - mtl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            int e = lane * 8 + j;
            if (e < E) {
                offsets[e] = run;
                if (act[j]) {
                    Group g;
                    g.row0 = run; g.m = loc[j]; g.expert = e; g.mt0 = runm;
                    groups[runa] = g;
                    s_groups[runa] = g;
                    ++runa;
                    runm += (loc[j] + kGroupTileRows - 1) / kGroupTileRows;
                }
            }
            run += loc[j];
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const int tact = __shfl_sync(0xffffffffu, inca, 31);
        const int mt = __shfl_sync(0xffffffffu, inclm, 31);
        if (lane == 0) {
            offsets[E] = total;
            n_groups[0] = tact;
            n_groups[1] = mt;
            s_ngroups = tact;
            stats->n_kept = total;
            stats->n_active = tact;
        }
    } else if (warp == 1 && lane == 0) {
        // 5. statistics: the CTAs' sums in CTA order
        long long k = 0;
        double l = 0.0;
        int z = 0;
        for (int b = 0; b < (int)gridDim.x; ++b) {
            k += __ldcg(&part[b].keep);
            l += __ldcg(&part[b].lreg);
            z += __ldcg(&part[b].zero);
        }
        stats->keep_sum = k;
        stats->lreg_sum = l;
        stats->n_all_masked = z;
        stats->tokens = T;
    }
    __syncthreads();
    // tile -> group table, from the block's copy of the group table
    for (int g = warp; g < s_ngroups; g += kScanWarps) {
        const Group G = s_groups[g];
        const int mts = (G.m + kGroupTileRows - 1) / kGroupTileRows;
        for (int q = lane; q < mts; q += 32) tile_group[G.mt0 + q] = G;
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
            copy_row_warp(dst, src, nv, lane);
        }
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- small batches, one kernel
// For T <= 32 tokens (one 32-token chunk) a single 1024-thread CTA does what route_select,
// compact_bits, compact_scan and compact_scatter_gather do for larger batches, saving three
// dependent launches on the decode path:
//   1. warp w < Tr selects routed row w (select_row) and writes the routing of its segment;
//   2. warp w builds, for experts e = w, w+32, ..., the ballot word of tokens keeping e;
//   3. warp 0 scans the per-expert counts into offsets, the active-group list and the
//      statistics (fixed reduction order);
//   4. every thread places one (token, slot) pair: pos = offsets[e] + popc(word[e] & below(t));
//   5. optionally, the warps copy the kept tokens' rows into X_perm (small batches only).
// The results are bit-identical to the multi-kernel path.
constexpr int kSmallT = 32;

// Working set of the small-batch routing (one block): at most kSmallT routed tokens.
struct SmallScratch {
    int id[kSmallT][32];
    uint8_t keep[kSmallT][32];
    uint32_t mask[kSmallT][kMaxE / 32 + 1];  // kept experts of each token (padded row)
    int nk[kSmallT];
    float lr[kSmallT];
    uint32_t word[kMaxE];
    int cnt[kMaxE];
    int off[kMaxE + 1];
    int perm[kSmallT * 32];
};

// The small-batch routing of one block, steps 1-4 above, on any number of warps.  Only a block
// with `outputs` set writes the results to global memory (the fused decode kernel runs this in
// every block and lets one of them publish); every block keeps offsets and perm in `sc`.
template <int EPL>
__device__ __forceinline__ void route_compact_small_body(
    SmallScratch& sc, bool outputs, const float* __restrict__ L, int ldL, int splits,
    long long split_stride, int Tr, int T, int E, int K, int seg, int mask_off,
    int* __restrict__ topk_id, float* __restrict__ gate, float* __restrict__ mlogit,
    uint8_t* __restrict__ keep, float* __restrict__ ghat, int* __restrict__ nkeep_tok,
    float* __restrict__ lreg_tok, int* __restrict__ counts, int* __restrict__ offsets,
    Group* __restrict__ groups, int* __restrict__ n_groups, DevStats* __restrict__ stats,
    int* __restrict__ perm, int* __restrict__ inv, Group* __restrict__ tile_group)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    for (int i = threadIdx.x; i < kSmallT * (kMaxE / 32 + 1); i += blockDim.x)
        (&sc.mask[0][0])[i] = 0u;
    __syncthreads();

    // 1. selection
    for (int r = warp; r < Tr; r += nwarps) {
        const RowDecision d = select_row<EPL>(L + (size_t)r * ldL, splits, split_stride, E, K,
                                              mask_off, lane);
        const int S = seg > 1 ? seg : 1;
        const int t0 = r * S, t1 = min(T, t0 + S);
        for (int t = t0; t < t1; ++t) {
            if (lane < K) {
                if (outputs) {
                    const size_t o = (size_t)t * K + lane;
                    topk_id[o] = d.id;
                    gate[o] = d.g;
                    mlogit[o] = d.l;
                    keep[o] = d.keep ? 1 : 0;
                    ghat[o] = d.ghat;
                }
                sc.id[t][lane] = d.id;
                sc.keep[t][lane] = d.keep ? 1 : 0;
                if (d.keep) atomicOr(&sc.mask[t][d.id >> 5], 1u << (d.id & 31));  // order-free OR
            }
            if (lane == 0) {
                if (outputs) { nkeep_tok[t] = d.nkeep; lreg_tok[t] = d.lreg; }
                sc.nk[t] = d.nkeep;
                sc.lr[t] = d.lreg;
            }
        }
    }
    __syncthreads();

    // 2. one ballot word per expert (lane = token)
    for (int e = warp; e < E; e += nwarps) {
        const bool has = lane < T && ((sc.mask[lane][e >> 5] >> (e & 31)) & 1u);
        const uint32_t word = __ballot_sync(0xffffffffu, has);
        if (lane == 0) {
            sc.word[e] = word;
            sc.cnt[e] = __popc(word);
            if (outputs) counts[e] = __popc(word);
        }
    }
    __syncthreads();

    // 3. offsets, active groups, statistics
    if (warp == 0) {
        int loc[8], act[8];
        int sum = 0, nact = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            loc[j] = (e < E) ? sc.cnt[e] : 0;
            act[j] = loc[j] > 0;
            sum += loc[j];
            nact += act[j];
        }
        int incl = sum, inca = nact;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            const int na = __shfl_up_sync(0xffffffffu, inca, o);
            if (lane >= o) { incl += n; inca += na; }
        }
        // tiles of kGroupTileRows rows: this lane's experts, then an exclusive scan over lanes
        int mtl = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) mtl += (loc[j] + kGroupTileRows - 1) / kGroupTileRows;
        int inclm = mtl;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, inclm, o);
            if (lane >= o) inclm += n;
        }
        int run = incl - sum, runa = inca - nact, runm = inclm - mtl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            if (e < E) {
                sc.off[e] = run;
                if (outputs) offsets[e] = run;
                if (act[j]) {
                    const int mts = (loc[j] + kGroupTileRows - 1) / kGroupTileRows;
                    if (outputs) {
                        Group g;
                        g.row0 = run; g.m = loc[j]; g.expert = e; g.mt0 = runm;
                        groups[runa] = g;
                        // at most 32 tokens: a group has at most 8 tiles, written here directly
                        for (int q = 0; q < mts; ++q) tile_group[runm + q] = g;
                    }
                    ++runa;
                    runm += mts;
                }
            }
            run += loc[j];
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const int tact = __shfl_sync(0xffffffffu, inca, 31);
        const int mt = __shfl_sync(0xffffffffu, inclm, 31);
        long long ks = lane < T ? sc.nk[lane] : 0;
        double ls = lane < T ? (double)sc.lr[lane] : 0.0;
        int nz = (lane < T && sc.nk[lane] == 0) ? 1 : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ks += __shfl_xor_sync(0xffffffffu, ks, o);
            ls += __shfl_xor_sync(0xffffffffu, ls, o);
            nz += __shfl_xor_sync(0xffffffffu, nz, o);
        }
        if (lane == 0) {
            sc.off[E] = total;
            if (outputs) {
                offsets[E] = total;
                n_groups[0] = tact;
                n_groups[1] = mt;
                stats->n_kept = total;
                stats->n_active = tact;
                stats->keep_sum = ks;
                stats->lreg_sum = ls;
                stats->n_all_masked = nz;
                stats->tokens = T;
            }
        }
    }
    __syncthreads();

    // 4. placement of every (token, slot) pair
    for (int i = threadIdx.x; i < T * K; i += blockDim.x) {
        const int t = i / K, k = i - t * K;
        int pos = -1;
        if (sc.keep[t][k]) {
            const int e = sc.id[t][k];
            pos = sc.off[e] + __popc(sc.word[e] & ((1u << t) - 1u));
            sc.perm[pos] = i;
            if (outputs) perm[pos] = i;
        }
        if (outputs) inv[i] = pos;
    }
    __syncthreads();
}

// X_perm[pos] = x[perm[pos] / K] for the kept pairs pos = w, w + nw, ... (warp w of nw).
template <typename TW>
__device__ __forceinline__ void gather_small_rows(const SmallScratch& sc, int E, int K, int D,
                                                  const TW* __restrict__ x, TW* __restrict__ xperm,
                                                  int w, int nw)
{
    const int lane = threadIdx.x & 31;
    const int nk = sc.off[E];
    const int nv = D * (int)sizeof(TW) / 16;
    for (int pos = w; pos < nk; pos += nw) {
        const int t = sc.perm[pos] / K;
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * D);
        uint4* dst = reinterpret_cast<uint4*>(xperm + (size_t)pos * D);
        copy_row_warp(dst, src, nv, lane);
    }
}

template <int EPL, typename TW>
__global__ void __launch_bounds__(1024)
route_compact_small_kernel(const float* __restrict__ L, int ldL, int splits, long long split_stride,
                           int Tr, int T, int E, int K, int seg, int mask_off,
                           int* __restrict__ topk_id, float* __restrict__ gate,
                           float* __restrict__ mlogit, uint8_t* __restrict__ keep,
                           float* __restrict__ ghat, int* __restrict__ nkeep_tok,
                           float* __restrict__ lreg_tok, int* __restrict__ counts,
                           int* __restrict__ offsets, Group* __restrict__ groups,
                           int* __restrict__ n_groups, DevStats* __restrict__ stats,
                           int* __restrict__ perm, int* __restrict__ inv,
                           const TW* __restrict__ x, TW* __restrict__ xperm, int D, int gather,
                           int* __restrict__ tail_cnt, int n_tail_cnt, Group* __restrict__ tile_group)
{
    __shared__ SmallScratch sc;
    pdl_wait();
    // the arrival counters of the grouped GEMMs' tail split start every forward at zero
    for (int i = threadIdx.x; i < n_tail_cnt; i += blockDim.x) tail_cnt[i] = 0;
    route_compact_small_body<EPL>(sc, true, L, ldL, splits, split_stride, Tr, T, E, K, seg,
                                  mask_off, topk_id, gate, mlogit, keep, ghat, nkeep_tok, lreg_tok,
                                  counts, offsets, groups, n_groups, stats, perm, inv, tile_group);
    if (gather) gather_small_rows(sc, E, K, D, x, xperm, threadIdx.x >> 5, blockDim.x >> 5);
    pdl_launch_dependents();
}

// X_perm[pos] = x[perm[pos] / K] for every kept pair (one warp per row, grid-stride).
template <typename TW>
__global__ void __launch_bounds__(256)
gather_rows_kernel(const int* __restrict__ perm, const int* __restrict__ n_kept_ptr, int K, int D,
                   const TW* __restrict__ x, TW* __restrict__ xperm)
{
    pdl_wait();
    const int nk = *n_kept_ptr;
    const int nv = D * (int)sizeof(TW) / 16;
    const int lane = threadIdx.x & 31;
    for (int pos = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; pos < nk;
         pos += (gridDim.x * blockDim.x) >> 5) {
        const int t = perm[pos] / K;
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * D);
        uint4* dst = reinterpret_cast<uint4*>(xperm + (size_t)pos * D);
        copy_row_warp(dst, src, nv, lane);
    }
    pdl_launch_dependents();
}

}  // namespace beam
