// stream_experts.cuh -- weight-streaming SwiGLU experts for decode-sized groups (and the fp32
// layer), step 4 of the BEAM pipeline (BEAM article on aitrends.kr, masked aggregation), run
// only for the device-built list of groups with at least one kept slot, plus the always-on
// shared experts (same article, limitation (C)).
//
// For a handful of tokens per expert the expert FFN is a GEMV: every weight byte is used for
// at most a few FMAs, so the kernels are HBM-bound and are built to stream weights: 128-bit
// read-only loads, several independent loads in flight per lane, the group's activations
// staged in shared memory and reused for every weight row, split-K over the 32 lanes of a
// warp with a fixed butterfly reduction (deterministic, no atomics).
//
// Work items are (group, block of kStreamR weight rows); the shared group (when present)
// comes first.  A persistent grid walks the item list; groups with no kept token are absent
// from the list, so their weights are never read.
#pragma once
#include "common.cuh"

namespace beam {

constexpr int kStreamMT = 8;   // tokens per pass over a weight row
constexpr int kStreamR = 16;   // weight rows per work item (2 per warp, 8 warps)
constexpr int kStreamNR = 2;   // rows a warp streams at once

struct StreamArgs {
    const void* xperm;   // routed activations, row g.row0 + i = i-th kept pair of group g
    const void* x;       // shared-expert activations [T][D]
    const void* wgu;     // routed gate/up [E][F/128][2][128][D] (gate block then up block)
    const void* wsgu;    // shared gate/up [Fsh/128][2][128][D]
    const void* wd;      // routed down [E][D][F], in the type of H
    const void* wsd;     // shared down [D][Fsh], in the type of H
    void* h;             // routed H [rows][F] (fp16 for bf16 layers, fp32 for fp32 layers)
    void* hsh;           // shared H [T][Fsh]
    float* yperm;        // routed Y [rows][D]
    float* ysh;          // shared Y [T][D]
    const Group* groups;
    const int* n_groups;
    int D, F, Fsh, T;
};

struct ItemView {
    const void* act;   // first activation row of the group
    int expert;        // routed expert index, -1 for the shared group
    void* hrow;        // first H row of the group
    float* yrow;       // first Y row of the group
    int m;             // rows (tokens) in the group
    int FF;            // intermediate size of the group
    int rb;            // row block inside the group
};

template <typename T, typename TH>
__device__ __forceinline__ ItemView stream_item(const StreamArgs& a, long item, int rb_shared,
                                                int rb_routed, int ng)
{
    ItemView v;
    if (item < rb_shared) {
        v.act = a.x; v.m = a.T; v.FF = a.Fsh; v.rb = (int)item;
        v.expert = -1; v.hrow = a.hsh; v.yrow = a.ysh;
    } else {
        const long r = item - rb_shared;
        const Group g = a.groups[r / rb_routed];
        v.rb = (int)(r % rb_routed);
        v.m = g.m; v.FF = a.F;
        v.act = static_cast<const T*>(a.xperm) + (size_t)g.row0 * a.D;
        v.hrow = static_cast<TH*>(a.h) + (size_t)g.row0 * a.F;
        v.yrow = a.yperm + (size_t)g.row0 * a.D;
        v.expert = g.expert;
    }
    return v;
}

// H[i][f] = silu(sum_d Wg[f][d] x_i[d]) * (sum_d Wu[f][d] x_i[d]) for the group's tokens i.
// T: storage type of x and the gate/up weights; TH: type of H.
template <typename T, typename TH>
__global__ void __launch_bounds__(256)
stream_gateup_kernel(StreamArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T* xs = reinterpret_cast<T*>(smem_raw);  // [kStreamMT][D]
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = a.D;
    constexpr int VN = Vec<T>::N;
    const int ng = *a.n_groups;
    const int rb_routed = a.F / kStreamR;
    const int rb_shared = a.Fsh / kStreamR;
    const long total = (long)rb_shared + (long)ng * rb_routed;
    const void* cached = nullptr;
    int cached_rows = 0;

    for (long item = blockIdx.x; item < total; item += gridDim.x) {
        ItemView v = stream_item<T, TH>(a, item, rb_shared, rb_routed, ng);
        const T* wbase = v.expert < 0 ? static_cast<const T*>(a.wsgu)
                                      : static_cast<const T*>(a.wgu) + (size_t)v.expert * 2 * a.F * D;
        for (int p0 = 0; p0 < v.m; p0 += kStreamMT) {
            const int mp = min(kStreamMT, v.m - p0);
            const T* src = static_cast<const T*>(v.act) + (size_t)p0 * D;
            if (src != cached || mp != cached_rows) {
                __syncthreads();
                const int nv = mp * D / VN;
                const uint4* s4 = reinterpret_cast<const uint4*>(src);
                uint4* d4 = reinterpret_cast<uint4*>(xs);
                for (int q = threadIdx.x; q < nv; q += blockDim.x) d4[q] = s4[q];
                __syncthreads();
                cached = src;
                cached_rows = mp;
            }
            const int f0 = v.rb * kStreamR + warp * kStreamNR;
            const T* wg[kStreamNR];
            const T* wu[kStreamNR];
#pragma unroll
            for (int q = 0; q < kStreamNR; ++q) {
                const int f = f0 + q;
                wg[q] = wbase + ((size_t)(f >> 7) * 256 + (f & 127)) * D;
                wu[q] = wg[q] + (size_t)128 * D;
            }
            float ag[kStreamNR][kStreamMT], au[kStreamNR][kStreamMT];
#pragma unroll
            for (int q = 0; q < kStreamNR; ++q)
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) { ag[q][i] = 0.f; au[q][i] = 0.f; }

            for (int d = lane * VN; d < D; d += 32 * VN) {
                uint4 rg[kStreamNR], ru[kStreamNR];
#pragma unroll
                for (int q = 0; q < kStreamNR; ++q) { rg[q] = ldg_stream(wg[q] + d); ru[q] = ldg_stream(wu[q] + d); }
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) {
                    if (i < mp) {
                        float xv[VN];
                        Vec<T>::widen(*reinterpret_cast<const uint4*>(xs + (size_t)i * D + d), xv);
#pragma unroll
                        for (int q = 0; q < kStreamNR; ++q) {
                            float wgv[VN], wuv[VN];
                            Vec<T>::widen(rg[q], wgv);
                            Vec<T>::widen(ru[q], wuv);
                            float sg = 0.f, su = 0.f;
#pragma unroll
                            for (int j = 0; j < VN; ++j) { sg = fmaf(wgv[j], xv[j], sg); su = fmaf(wuv[j], xv[j], su); }
                            ag[q][i] += sg;
                            au[q][i] += su;
                        }
                    }
                }
            }
            TH* hout = static_cast<TH*>(v.hrow);
#pragma unroll
            for (int q = 0; q < kStreamNR; ++q) {
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) {
                    if (i < mp) {
                        const float g = warp_sum(ag[q][i]);
                        const float u = warp_sum(au[q][i]);
                        if (lane == 0)
                            hout[(size_t)(p0 + i) * v.FF + f0 + q] = from_float<TH>(silu_f(g) * u);
                    }
                }
            }
        }
    }
    pdl_launch_dependents();
}

// Y[i][j] = sum_f Wd[j][f] H[i][f] for the group's tokens i; H is staged in shared memory in
// chunks of kFC elements and every warp keeps its two output rows' partial sums in registers.
// T: type of H and of the down weights.
template <typename T>
__global__ void __launch_bounds__(256)
stream_down_kernel(StreamArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int kFC = 65536 / (kStreamMT * (int)sizeof(T));  // 64 KB of H per stage
    T* hs = reinterpret_cast<T*>(smem_raw);                    // [kStreamMT][kFC]
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = a.D;
    constexpr int VN = Vec<T>::N;
    const int ng = *a.n_groups;
    const int rb_routed = D / kStreamR;
    const int rb_shared = a.Fsh > 0 ? D / kStreamR : 0;
    const long total = (long)rb_shared + (long)ng * rb_routed;

    for (long item = blockIdx.x; item < total; item += gridDim.x) {
        ItemView v = stream_item<T, T>(a, item, rb_shared, rb_routed, ng);
        const T* wbase = v.expert < 0 ? static_cast<const T*>(a.wsd)
                                      : static_cast<const T*>(a.wd) + (size_t)v.expert * D * a.F;
        const int FF = v.FF;
        const int j0 = v.rb * kStreamR + warp * kStreamNR;
        for (int p0 = 0; p0 < v.m; p0 += kStreamMT) {
            const int mp = min(kStreamMT, v.m - p0);
            const T* hsrc = static_cast<const T*>(v.hrow) + (size_t)p0 * FF;
            float acc[kStreamNR][kStreamMT];
#pragma unroll
            for (int q = 0; q < kStreamNR; ++q)
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) acc[q][i] = 0.f;
            for (int c0 = 0; c0 < FF; c0 += kFC) {
                const int fl = min(kFC, FF - c0);
                __syncthreads();
                const int vpr = fl / VN;
                for (int q = threadIdx.x; q < mp * vpr; q += blockDim.x) {
                    const int i = q / vpr, c = q - i * vpr;
                    reinterpret_cast<uint4*>(hs + (size_t)i * kFC)[c] =
                        reinterpret_cast<const uint4*>(hsrc + (size_t)i * FF + c0)[c];
                }
                __syncthreads();
                const T* wr[kStreamNR];
#pragma unroll
                for (int q = 0; q < kStreamNR; ++q) wr[q] = wbase + (size_t)(j0 + q) * FF + c0;
                for (int f = lane * VN; f < fl; f += 32 * VN) {
                    uint4 rw[kStreamNR];
#pragma unroll
                    for (int q = 0; q < kStreamNR; ++q) rw[q] = ldg_stream(wr[q] + f);
#pragma unroll
                    for (int i = 0; i < kStreamMT; ++i) {
                        if (i < mp) {
                            float hv[VN];
                            Vec<T>::widen(*reinterpret_cast<const uint4*>(hs + (size_t)i * kFC + f), hv);
#pragma unroll
                            for (int q = 0; q < kStreamNR; ++q) {
                                float wv[VN];
                                Vec<T>::widen(rw[q], wv);
                                float s = 0.f;
#pragma unroll
                                for (int j = 0; j < VN; ++j) s = fmaf(wv[j], hv[j], s);
                                acc[q][i] += s;
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kStreamNR; ++q) {
#pragma unroll
                for (int i = 0; i < kStreamMT; ++i) {
                    if (i < mp) {
                        const float s = warp_sum(acc[q][i]);
                        if (lane == 0) v.yrow[(size_t)(p0 + i) * D + j0 + q] = s;
                    }
                }
            }
        }
    }
    pdl_launch_dependents();
}

// ---------------------------------------------------------------- combine
// y[t] = sum over slots k in rank order with keep = 1 of g_hat[t][k] * Y_perm[inv[t][k]],
// plus the shared-expert output; a fixed order, so the result is bit-reproducible.
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ yperm, const float* __restrict__ ysh,
               const int* __restrict__ inv, const float* __restrict__ ghat, int T, int K, int D,
               float* __restrict__ y)
{
    pdl_wait();
    const int t = blockIdx.x;
    if (t < T) {
        const int D4 = D >> 2;
        const float4* Y = reinterpret_cast<const float4*>(yperm);
        for (int c = threadIdx.x; c < D4; c += blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k = 0; k < K; ++k) {
                const int p = inv[(size_t)t * K + k];
                if (p >= 0) {
                    const float g = ghat[(size_t)t * K + k];
                    const float4 v = Y[(size_t)p * D4 + c];
                    acc.x = fmaf(g, v.x, acc.x); acc.y = fmaf(g, v.y, acc.y);
                    acc.z = fmaf(g, v.z, acc.z); acc.w = fmaf(g, v.w, acc.w);
                }
            }
            if (ysh) {
                const float4 s = reinterpret_cast<const float4*>(ysh)[(size_t)t * D4 + c];
                acc.x += s.x; acc.y += s.y; acc.z += s.z; acc.w += s.w;
            }
            reinterpret_cast<float4*>(y)[(size_t)t * D4 + c] = acc;
        }
    }
    pdl_launch_dependents();
}

}  // namespace beam
