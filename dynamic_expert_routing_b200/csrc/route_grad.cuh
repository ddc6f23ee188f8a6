// route_grad.cuh -- training-side gradient of the BEAM routing: the router W_r and the mask
// router W_m under the straight-through estimator, plus the L_reg term (BEAM article on
// aitrends.kr, training paragraph: L = L_lm + alpha L_bal + beta L_reg with
// L_reg = (1/K) sum_{i in TK} |m_hat_i|, and the binary mask's gradient passed straight to
// m_hat; ai-feeds.com summary, Method, binarisation and straight-through estimator).
//
// It runs after a training forward, in which every Top-K slot's expert is evaluated (the mask
// only scales the gates, g_hat = g * m), so Y_perm holds E_i(x_t) for every slot.  Given
// dy = dL/dy [T][D] (fp32) and reg = dL/dL_reg / (T K) (L_reg being the mean over tokens):
//   s_tk  = <dy_t, E_i(x_t)>                                (dL/dg_hat)
//   dg_k  = sum over the routed row's tokens of s_tk m_k;   dmh_k = sum of (s_tk g_k + reg)
//   d_l_k = dmh_k sigmoid(l_k) (1 - sigmoid(l_k));          d_r_k = g_k (dg_k - sum_j g_j dg_j)
//   dx[row] = sum_k d_r_k W_r[:, i_k] + d_l_k W_m[:, i_k]    (other tokens of a segment: 0)
//   dW_r[:, e] = sum over routed rows whose Top-K holds e of x[row] d_r;  dW_m likewise.
// Everything is summed in a fixed order (no atomics), so the results are bit-reproducible.
//
// Kernels:
//   route_grad_kernel      one CTA per routed row: the K dots, the row's logit gradients, dx.
//   route_dw_partial_kernel one CTA per (unit, column slice): a unit is up to R consecutive
//                          (expert, token)-ordered pairs of one expert (the compaction's perm);
//                          it sums x[row] * (d_r, d_l) over them into a partial column.
//   route_dw_reduce_kernel adds each expert's partials in unit order into dW_r / dW_m [D][E].
#pragma once
#include "common.cuh"
#include "router.cuh"
#include "stream_experts.cuh"

namespace beam {

constexpr int kGradThreads = 256;

// KM: the smallest of 4, 8, 16, 32 that holds K (each thread keeps KM partial dots).
template <typename TY, typename TX, int KM>
__global__ void __launch_bounds__(kGradThreads)
route_grad_kernel(const TY* __restrict__ yperm, int splits, long long stride,
                  const int* __restrict__ inv, const int* __restrict__ topk_id,
                  const float* __restrict__ gate, const float* __restrict__ mlogit,
                  const float* __restrict__ dy, const TX* __restrict__ wrm, int T, int K, int E,
                  int D, int S, float reg, float* __restrict__ dghat, float* __restrict__ d_r,
                  float* __restrict__ d_l, float2* __restrict__ pair_grad, float* __restrict__ dx)
{
    constexpr int NW = kGradThreads / 32;
    __shared__ float red[NW][KM];
    __shared__ int s_inv[KM];
    __shared__ float s_dr[KM], s_dl[KM];
    __shared__ int s_e[KM];
    pdl_wait();
    const int row = blockIdx.x;
    const int t0 = row * S, t1 = min(T, t0 + S);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D4 = D >> 2;
    const long long s4 = stride >> 2;
    // warp 0, lane k < K: slot k of the routed row and its sums over the row's tokens
    float g_k = 0.f, l_k = 0.f, dg = 0.f, dmh = 0.f;
    int e_k = 0;
    if (warp == 0 && lane < K) {
        const size_t o = (size_t)t0 * K + lane;
        g_k = gate[o];
        l_k = mlogit[o];
        e_k = topk_id[o];
    }
    for (int t = t0; t < t1; ++t) {
        if (threadIdx.x < K) s_inv[threadIdx.x] = inv[(size_t)t * K + threadIdx.x];
        __syncthreads();
        float acc[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k) acc[k] = 0.f;
        for (int c = threadIdx.x; c < D4; c += kGradThreads) {
            const float4 g4 = __ldcs(reinterpret_cast<const float4*>(dy) + (size_t)t * D4 + c);
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                if (k < K && s_inv[k] >= 0) {   // a training forward evaluated every slot
                    float4 v = load4(yperm, (size_t)s_inv[k] * D4 + c);
                    for (int s = 1; s < splits; ++s) {
                        const float4 w = load4(yperm, s * s4 + (size_t)s_inv[k] * D4 + c);
                        v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
                    }
                    float a = acc[k];
                    a = fmaf(g4.x, v.x, a); a = fmaf(g4.y, v.y, a);
                    a = fmaf(g4.z, v.z, a); a = fmaf(g4.w, v.w, a);
                    acc[k] = a;
                }
            }
        }
        // each slot's dot: the warp's lanes, then the warps in index order
#pragma unroll
        for (int k = 0; k < KM; ++k) {
            if (k < K) {
                const float v = warp_sum(acc[k]);
                if (lane == 0) red[warp][k] = v;
            }
        }
        __syncthreads();
        if (warp == 0 && lane < K) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) s += red[w][lane];
            const size_t o = (size_t)t * K + lane;
            if (dghat) dghat[o] = s;
            if (l_k >= 0.f) dg += s;          // dL/dg = s m
            dmh += fmaf(s, g_k, reg);         // dL/dm_hat = s g (straight through) + L_reg
            if (t != t0) {
                if (d_r) d_r[o] = 0.f;
                if (d_l) d_l[o] = 0.f;
            }
        }
        __syncthreads();
    }
    if (warp == 0) {
        const float c = warp_sum(lane < K ? g_k * dg : 0.f);
        if (lane < K) {
            const float sg = sigmoid_f(l_k);
            const float gl = dmh * (sg * (1.f - sg));
            const float gr = g_k * (dg - c);
            s_dr[lane] = gr;
            s_dl[lane] = gl;
            s_e[lane] = e_k;
            const size_t o = (size_t)t0 * K + lane;
            if (d_r) d_r[o] = gr;
            if (d_l) d_l[o] = gl;
            pair_grad[o] = make_float2(gr, gl);
        }
    }
    __syncthreads();
    // dx of the routed row from the repacked router rows (row e: W_r[:, e]; row E + e: W_m[:, e])
    constexpr int N = Vec<TX>::N;
    const int DV = D / N;
    for (int c = threadIdx.x; c < DV; c += kGradThreads) {
        float a[N];
#pragma unroll
        for (int j = 0; j < N; ++j) a[j] = 0.f;
        for (int k = 0; k < K; ++k) {
            float wr[N], wm[N];
            Vec<TX>::widen(*reinterpret_cast<const uint4*>(wrm + (size_t)s_e[k] * D + (size_t)c * N), wr);
            Vec<TX>::widen(*reinterpret_cast<const uint4*>(wrm + (size_t)(E + s_e[k]) * D + (size_t)c * N), wm);
            const float gr = s_dr[k], gl = s_dl[k];
#pragma unroll
            for (int j = 0; j < N; ++j) a[j] = fmaf(gl, wm[j], fmaf(gr, wr[j], a[j]));
        }
        float4* o = reinterpret_cast<float4*>(dx + (size_t)t0 * D + (size_t)c * N);
#pragma unroll
        for (int j = 0; j < N; j += 4) __stcs(o + j / 4, make_float4(a[j], a[j + 1], a[j + 2], a[j + 3]));
    }
    for (int t = t0 + 1; t < t1; ++t)
        for (int c = threadIdx.x; c < D4; c += kGradThreads)
            __stcs(reinterpret_cast<float4*>(dx) + (size_t)t * D4 + c, make_float4(0.f, 0.f, 0.f, 0.f));
    pdl_launch_dependents();
}

// Units of the dW pass: expert e's pairs [offsets[e], offsets[e+1]) cut into pieces of R;
// unit numbers are given expert by expert.  u[e] = first unit of e, u[E] = the total.
__device__ __forceinline__ void dw_units(const int* __restrict__ offsets, int E, int R, int* u)
{
    if (threadIdx.x == 0) {
        int n = 0;
        for (int e = 0; e < E; ++e) {
            u[e] = n;
            n += (offsets[e + 1] - offsets[e] + R - 1) / R;
        }
        u[E] = n;
    }
    __syncthreads();
}

template <typename TX>
__global__ void __launch_bounds__(256)
route_dw_partial_kernel(const int* __restrict__ offsets, const int* __restrict__ perm,
                        const float2* __restrict__ pair_grad, const TX* __restrict__ x, int K,
                        int E, int D, int S, int R, float* __restrict__ part)
{
    __shared__ int s_off[kRouteMaxE + 1];
    __shared__ int s_u[kRouteMaxE + 1];
    pdl_wait();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    dw_units(s_off, E, R, s_u);
    const int unit = blockIdx.x;
    if (unit < s_u[E]) {
        // the expert owning this unit: the largest e with s_u[e] <= unit (experts without pairs
        // share their successor's first unit and are skipped)
        int lo = 0, hi = E - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_u[mid] <= unit) lo = mid; else hi = mid - 1;
        }
        const int e = lo;
        const int r0 = s_off[e] + (unit - s_u[e]) * R, r1 = min(s_off[e + 1], r0 + R);
        constexpr int N = Vec<TX>::N;
        const int d0 = (blockIdx.y * blockDim.x + threadIdx.x) * N;
        if (d0 < D) {
            float ar[N], am[N];
#pragma unroll
            for (int j = 0; j < N; ++j) ar[j] = am[j] = 0.f;
            constexpr int U = 4;   // rows whose loads are in flight together
            for (int i0 = r0; i0 < r1; i0 += U) {
                int tt[U];
                float2 gv[U];
                uint4 raw[U];
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    tt[q] = -1;
                    if (i0 + q < r1) {
                        const int p = perm[i0 + q];
                        const int t = p / K;
                        if (t % S == 0) { tt[q] = t; gv[q] = pair_grad[p]; }
                    }
                }
#pragma unroll
                for (int q = 0; q < U; ++q)
                    if (tt[q] >= 0) raw[q] = *reinterpret_cast<const uint4*>(x + (size_t)tt[q] * D + d0);
#pragma unroll
                for (int q = 0; q < U; ++q) {
                    if (tt[q] >= 0) {
                        float xv[N];
                        Vec<TX>::widen(raw[q], xv);
#pragma unroll
                        for (int j = 0; j < N; ++j) {
                            ar[j] = fmaf(xv[j], gv[q].x, ar[j]);
                            am[j] = fmaf(xv[j], gv[q].y, am[j]);
                        }
                    }
                }
            }
            float* pr = part + (size_t)unit * 2 * D + d0;
#pragma unroll
            for (int j = 0; j < N; j += 4) {
                reinterpret_cast<float4*>(pr)[j / 4] = make_float4(ar[j], ar[j + 1], ar[j + 2], ar[j + 3]);
                reinterpret_cast<float4*>(pr + D)[j / 4] = make_float4(am[j], am[j + 1], am[j + 2], am[j + 3]);
            }
        }
    }
    pdl_launch_dependents();
}

// dW_r[d][e] and dW_m[d][e] = the sums of expert e's partials in unit order (0 without pairs).
__global__ void __launch_bounds__(256)
route_dw_reduce_kernel(const int* __restrict__ offsets, const float* __restrict__ part, int E,
                       int D, int R, float* __restrict__ dw_r, float* __restrict__ dw_m)
{
    __shared__ int s_off[kRouteMaxE + 1];
    __shared__ int s_u[kRouteMaxE + 1];
    pdl_wait();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    dw_units(s_off, E, R, s_u);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (long long)E * D) {
        const int e = (int)(i / D), d = (int)(i % D);
        float ar = 0.f, am = 0.f;
        for (int u = s_u[e]; u < s_u[e + 1]; ++u) {
            ar += part[(size_t)u * 2 * D + d];
            am += part[(size_t)u * 2 * D + D + d];
        }
        dw_r[(size_t)d * E + e] = ar;
        dw_m[(size_t)d * E + e] = am;
    }
    pdl_launch_dependents();
}

}  // namespace beam
