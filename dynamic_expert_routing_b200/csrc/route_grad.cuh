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
//   route_grad_kernel  one CTA per routed row (a token, or a segment): the K dots in 4-column
//                      units, the row's logit gradients, dx.
//   route_dw_kernel    one warp per (unit, column chunk): a unit is up to R consecutive
//                      (expert, token)-ordered pairs of one expert (the compaction's perm); the
//                      warp sums x[row] * (d_r, d_l) over them into a partial column pair.  The
//                      last warp to finish a (expert, chunk) adds that expert's partials in
//                      unit order into dW_r / dW_m [D][E] (an arrival counter only elects it;
//                      the order of the sum is fixed).
#pragma once
#include "common.cuh"
#include "router.cuh"
#include "stream_experts.cuh"

namespace beam {

constexpr int kGradThreads = 256;
constexpr int kGradWarps = kGradThreads / 32;

// One column unit is 4 consecutive columns: one float4 of dy and of each slot's Y row (fp16
// rows: one 8-byte load).  Narrow units keep the kernel near 40 registers, so that six CTAs
// share an SM: a CTA's phases (loads, block reduction, dx) alternate, and occupancy, not
// per-thread load depth, is what keeps HBM busy.
template <typename TY>
__device__ __forceinline__ float unit_dot(const TY* __restrict__ yperm, int splits, long long s4,
                                          size_t idx, float4 g, float a)
{
    float4 v = load4(yperm, idx);
    for (int s = 1; s < splits; ++s) {
        const float4 w = load4(yperm, s * s4 + idx);
        v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
    }
    a = fmaf(g.x, v.x, a); a = fmaf(g.y, v.y, a);
    a = fmaf(g.z, v.z, a); a = fmaf(g.w, v.w, a);
    return a;
}

template <int KM> constexpr int grad_min_blocks() { return KM <= 4 ? 6 : (KM <= 8 ? 5 : (KM <= 16 ? 4 : 2)); }

// KM: the smallest of 2, 4, 8, 16, 32 that holds K.  One CTA per routed row (a token, or a
// segment of S tokens sharing the first token's decision).  Threads take column units of the
// row's tokens; each thread keeps KM partial dots, summed over the segment's tokens unless the
// per-token s (dghat) is asked for; the warps' partials are added in warp order.
template <typename TY, typename TX, int KM>
__global__ void __launch_bounds__(kGradThreads, grad_min_blocks<KM>())
route_grad_kernel(const TY* __restrict__ yperm, int splits, long long stride,
                  const int* __restrict__ inv, const int* __restrict__ topk_id,
                  const float* __restrict__ gate, const float* __restrict__ mlogit,
                  const float* __restrict__ dy, const TX* __restrict__ wrm, int T, int K, int E,
                  int D, int S, float reg, float* __restrict__ dghat, float* __restrict__ d_r,
                  float* __restrict__ d_l, float2* __restrict__ pair_grad, float* __restrict__ dx)
{
    __shared__ float red[kGradWarps][KM];
    __shared__ int s_inv[KM];
    __shared__ float s_gr[KM], s_gl[KM];
    __shared__ int s_e[KM];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * S, t1 = min(T, t0 + S);
    const int DU = D >> 2;                 // column units of a row
    const long long sN = stride >> 2;      // split-slice stride in units
    // warp 0, lane k < K: slot k of the routed row, fetched up front (one round trip with the
    // first token's slot positions)
    const bool on = warp == 0 && lane < K;
    const size_t o0 = (size_t)t0 * K + lane;
    float g = 0.f, l = 0.f;
    int e_k = 0, pos = -1;
    if (on) { g = gate[o0]; l = mlogit[o0]; e_k = topk_id[o0]; pos = inv[o0]; }
    float acc[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) acc[k] = 0.f;
    float run = 0.f;                       // warp 0, lane k: sum over the row's tokens of s_tk
    for (int t = t0; t < t1; ++t) {
        if (t == t0) {
            if (on) s_inv[lane] = pos;
        } else if (threadIdx.x < K) {
            s_inv[threadIdx.x] = inv[(size_t)t * K + threadIdx.x];
        }
        __syncthreads();
        int p[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k) p[k] = (k < K) ? s_inv[k] : -1;
        const float4* dyr = reinterpret_cast<const float4*>(dy) + (size_t)t * DU;
#pragma unroll 1
        for (int u = threadIdx.x; u < DU; u += kGradThreads) {
            const float4 g4 = __ldcs(dyr + u);
#pragma unroll
            for (int k = 0; k < KM; ++k)
                if (p[k] >= 0)   // a training forward evaluated every slot
                    acc[k] = unit_dot(yperm, splits, sN, (size_t)p[k] * DU + u, g4, acc[k]);
        }
        // per-token s only when asked for (or at the row's last token): the warps' sums in
        // warp order
        if (dghat || t + 1 == t1) {
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                if (k < K) {
                    const float v = warp_sum(acc[k]);
                    if (lane == 0) red[warp][k] = v;
                }
                acc[k] = 0.f;
            }
            __syncthreads();
            if (warp == 0 && lane < K) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kGradWarps; ++w) sum += red[w][lane];
                run += sum;
                if (dghat) dghat[(size_t)t * K + lane] = sum;
            }
        }
        if (warp == 0 && lane < K && t != t0) {
            const size_t o = (size_t)t * K + lane;
            if (d_r) d_r[o] = 0.f;
            if (d_l) d_l[o] = 0.f;
        }
        __syncthreads();   // s_inv and red are reused
    }
    if (warp == 0) {
        // lane k: dg = S m, dmh = S g + n reg, d_l = dmh sigmoid'(l), d_r = g (dg - sum g dg)
        const size_t o = o0;
        const float dg = (on && l >= 0.f) ? run : 0.f;
        const float dmh = fmaf(run, g, (float)(t1 - t0) * reg);
        const float c = warp_sum(on ? g * dg : 0.f);
        const float sg = sigmoid_f(l);
        if (on) {
            const float gl = dmh * (sg * (1.f - sg));
            const float gr = g * (dg - c);
            s_gr[lane] = gr;
            s_gl[lane] = gl;
            s_e[lane] = e_k;
            if (d_r) d_r[o] = gr;
            if (d_l) d_l[o] = gl;
            if (pos >= 0) pair_grad[pos] = make_float2(gr, gl);
        }
    }
    __syncthreads();
    // dx of the routed row from the repacked router rows (row e: W_r[:, e]; row E + e:
    // W_m[:, e]); the segment's other tokens get 0
    constexpr int N = Vec<TX>::N;
    const int DV = D / N;
    for (int cv = threadIdx.x; cv < DV; cv += kGradThreads) {
        float a[N];
#pragma unroll
        for (int j = 0; j < N; ++j) a[j] = 0.f;
#pragma unroll 1
        for (int k = 0; k < K; ++k) {
            float wr[N], wm[N];
            const int e = s_e[k];
            Vec<TX>::widen(__ldg(reinterpret_cast<const uint4*>(wrm + (size_t)e * D) + cv), wr);
            Vec<TX>::widen(__ldg(reinterpret_cast<const uint4*>(wrm + (size_t)(E + e) * D) + cv), wm);
            const float gr = s_gr[k], gl = s_gl[k];
#pragma unroll
            for (int j = 0; j < N; ++j) a[j] = fmaf(gl, wm[j], fmaf(gr, wr[j], a[j]));
        }
        float4* o = reinterpret_cast<float4*>(dx + (size_t)t0 * D + (size_t)cv * N);
#pragma unroll
        for (int j = 0; j < N; j += 4) __stcs(o + j / 4, make_float4(a[j], a[j + 1], a[j + 2], a[j + 3]));
    }
    const int D4 = D >> 2;
    for (int t = t0 + 1; t < t1; ++t)
        for (int c = threadIdx.x; c < D4; c += kGradThreads)
            __stcs(reinterpret_cast<float4*>(dx) + (size_t)t * D4 + c, make_float4(0.f, 0.f, 0.f, 0.f));
    pdl_launch_dependents();
}

// Units of the dW pass: expert e's pairs [offsets[e], offsets[e+1]) cut into pieces of R;
// unit numbers are given expert by expert.  u[e] = first unit of e, u[E] = the total.  Warp 0
// scans: lane l counts experts 8l .. 8l + 7 (E <= 256), then a warp prefix sum.
__device__ __forceinline__ void dw_units(const int* __restrict__ offsets, int E, int R, int* u)
{
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int c[8], n = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            c[j] = e < E ? (offsets[e + 1] - offsets[e] + R - 1) / R : 0;
            n += c[j];
        }
        int incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int base = incl - n;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = lane * 8 + j;
            if (e < E) u[e] = base;
            base += c[j];
        }
        if (lane == 31) u[E] = incl;
    }
    __syncthreads();
}

// Column chunk of one warp: 32 lanes x one 16-byte vector of x each.
template <typename TX> constexpr int dw_chunk_cols() { return 32 * Vec<TX>::N; }

// part: [units][2][D] partial columns; cnt: [E][chunks] arrival counters (zero between calls:
// zeroed at create, reset by the warp that reduces).
template <typename TX>
__global__ void __launch_bounds__(256)
route_dw_kernel(const int* __restrict__ offsets, const int* __restrict__ perm,
                const float2* __restrict__ pair_grad, const TX* __restrict__ x, int K, int E,
                int D, int S, int R, int chunks, float* __restrict__ part, int* __restrict__ cnt,
                float* __restrict__ dw_r, float* __restrict__ dw_m)
{
    __shared__ int s_off[kRouteMaxE + 1];
    __shared__ int s_u[kRouteMaxE + 1];
    pdl_wait();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    dw_units(s_off, E, R, s_u);
    // experts that no pair reaches have zero gradient columns
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)E * D;
         i += (long long)gridDim.x * blockDim.x) {
        const int e = (int)(i % E);
        if (s_off[e + 1] == s_off[e]) { dw_r[i] = 0.f; dw_m[i] = 0.f; }
    }
    constexpr int N = Vec<TX>::N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x * (blockDim.x >> 5) + warp;
    if (item < s_u[E] * chunks) {
        const int unit = item / chunks, chunk = item - unit * chunks;
        int lo = 0, hi = E - 1;   // the largest e with s_u[e] <= unit
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_u[mid] <= unit) lo = mid; else hi = mid - 1;
        }
        const int e = lo;
        const int r0 = s_off[e] + (unit - s_u[e]) * R, r1 = min(s_off[e + 1], r0 + R);
        const int d0 = (chunk * 32 + lane) * N;
        const bool col = d0 < D;
        float ar[N], am[N];
#pragma unroll
        for (int j = 0; j < N; ++j) ar[j] = am[j] = 0.f;
        for (int b0 = r0; b0 < r1; b0 += 32) {
            // lane j fetches pair b0 + j; rows of a segment's later tokens are skipped
            int tj = -1;
            float gx = 0.f, gy = 0.f;
            if (b0 + lane < r1) {
                // pair gradients are stored at the pair's perm position (routed rows only)
                const int p = __ldg(perm + b0 + lane);
                const float2 gv = __ldg(pair_grad + b0 + lane);
                const int t = p / K;
                if (t % S == 0) {
                    tj = t;
                    gx = gv.x; gy = gv.y;
                }
            }
            // the batch's rows that carry a gradient (all of them without segments), in order
            uint32_t live = __ballot_sync(0xffffffffu, tj >= 0);
            while (live) {
                int tt[8];
                float ga[8], gb[8];
                uint4 raw[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int src = live ? __ffs(live) - 1 : 0;
                    tt[q] = live ? __shfl_sync(0xffffffffu, tj, src) : -1;
                    ga[q] = __shfl_sync(0xffffffffu, gx, src);
                    gb[q] = __shfl_sync(0xffffffffu, gy, src);
                    live &= live - 1;
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (tt[q] >= 0 && col)
                        raw[q] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)tt[q] * D + d0));
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    if (tt[q] >= 0 && col) {
                        float xv[N];
                        Vec<TX>::widen(raw[q], xv);
#pragma unroll
                        for (int j = 0; j < N; ++j) {
                            ar[j] = fmaf(xv[j], ga[q], ar[j]);
                            am[j] = fmaf(xv[j], gb[q], am[j]);
                        }
                    }
                }
            }
        }
        if (col) {
            float* pr = part + (size_t)unit * 2 * D + d0;
#pragma unroll
            for (int j = 0; j < N; j += 4) {
                __stcg(reinterpret_cast<float4*>(pr) + j / 4, make_float4(ar[j], ar[j + 1], ar[j + 2], ar[j + 3]));
                __stcg(reinterpret_cast<float4*>(pr + D) + j / 4, make_float4(am[j], am[j + 1], am[j + 2], am[j + 3]));
            }
        }
        // the last warp of (expert, chunk) to arrive adds the expert's partials in unit order
        __threadfence();
        __syncwarp();
        int last = 0;
        const int nu = s_u[e + 1] - s_u[e];
        if (lane == 0) last = atomicAdd(cnt + (size_t)e * chunks + chunk, 1) == nu - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
            __threadfence();
            float sr[N], sm[N];
#pragma unroll
            for (int j = 0; j < N; ++j) sr[j] = sm[j] = 0.f;
            if (col) {
#pragma unroll 4
                for (int u = s_u[e]; u < s_u[e + 1]; ++u) {
                    const float* pu = part + (size_t)u * 2 * D + d0;
#pragma unroll
                    for (int j = 0; j < N; j += 4) {
                        const float4 a = __ldcg(reinterpret_cast<const float4*>(pu) + j / 4);
                        const float4 b = __ldcg(reinterpret_cast<const float4*>(pu + D) + j / 4);
                        sr[j] += a.x; sr[j + 1] += a.y; sr[j + 2] += a.z; sr[j + 3] += a.w;
                        sm[j] += b.x; sm[j + 1] += b.y; sm[j + 2] += b.z; sm[j + 3] += b.w;
                    }
                }
#pragma unroll
                for (int j = 0; j < N; ++j) {
                    dw_r[(size_t)(d0 + j) * E + e] = sr[j];
                    dw_m[(size_t)(d0 + j) * E + e] = sm[j];
                }
            }
            if (lane == 0) cnt[(size_t)e * chunks + chunk] = 0;   // ready for the next call
        }
    }
    pdl_launch_dependents();
}

}  // namespace beam
