// softtopk.cuh -- SoftTopK, the differentiable top-k of "Stepped MoE: Segment-Level Routing with
// Configurable Inference Complexity" (SoftTopK entry and core method: the mask generator's
// routing logits pass through a continuous relaxation of the top-k indicator, so the expert
// choice is trained end to end, while the layers receive the {0,1} top-k mask).
//
// The page gives no formula; the relaxation used is the limited-multi-label projection (Amos,
// Xu and Kolter, 2019): y_i = sigmoid((r_i - nu) / tau) with nu set so that sum_i y_i = K (the
// entropy-regularised projection of r / tau onto {0 <= y <= 1, sum y = K}).  Its backward,
// through nu, is dr_j = h_j (dy_j - sum_i h_i dy_i / sum_i h_i) with h_i = y_i (1 - y_i) / tau.
//
// One warp per token row; lane l holds logits l, l + 32, ... (EPL = ceil(E/32) per lane).
//   forward:  the hard Top-K indicator first (K rounds of a warp arg-max under (value desc,
//             index asc), and one more round for the (K+1)-th value); then nu by safeguarded
//             Newton in fp32 on f(nu) = sum_i sigmoid((r_i - nu)/tau) - K (strictly
//             decreasing), started halfway between the K-th and the (K+1)-th largest logit
//             (the root when tau is small against their gap) inside the sign bracket
//             [min r - 40 tau, max r + 40 tau], bisecting whenever a step leaves the bracket,
//             until a Newton step is below 2^-16 tau; every lane evaluates f with the same
//             xor-butterfly sum, so the iteration is bitwise identical across the warp.  Then y.
//   backward: two butterfly sums per row (sum h, sum h dy), then dr.
// Deterministic: fixed reduction order, no atomics.  HBM-bound: 4 B per logit read, 4 + 1 B
// written (y, mask) forward; 8 B read and 4 B written per logit backward.
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace beam {

constexpr int kSoftTopkMaxE = 256;

template <int EPL>
__global__ void __launch_bounds__(256)
softtopk_fwd_kernel(const float* __restrict__ r, int T, int E, int K, float tau,
                    float* __restrict__ y, uint8_t* __restrict__ mask, float* __restrict__ nu_out)
{
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = (long long)blockIdx.x * 8 + warp;
    if (t < T) {
        const float* rt = r + t * E;
        float v[EPL];
        float lo = INFINITY, hi = -INFINITY;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            v[j] = e < E ? __ldg(rt + e) : 0.f;
            if (e < E) { lo = fminf(lo, v[j]); hi = fmaxf(hi, v[j]); }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        const float inv_tau = 1.0f / tau;
        // hard Top-K indicator: K rounds, each taking the largest remaining value, the lowest
        // expert among equal ones; a (K+1)-th round gives the next value, for the start of nu
        uint32_t ord[EPL];
#pragma unroll
        for (int j = 0; j < EPL; ++j) ord[j] = (lane + 32 * j < E) ? topk_ord(v[j]) : 0u;
        uint32_t sel = 0u;   // bit j: this lane's expert lane + 32 j is selected
        uint32_t kth = 0u, next = 0u;
        const int rounds = K < E ? K + 1 : K;
        for (int k = 0; k < rounds; ++k) {
            uint32_t best = 0u, bidx = 0xffffffffu;
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const uint32_t e = (uint32_t)(lane + 32 * j);
                if (!((sel >> j) & 1u) && e < (uint32_t)E && ord[j] > best) { best = ord[j]; bidx = e; }
                else if (!((sel >> j) & 1u) && e < (uint32_t)E && ord[j] == best && e < bidx) bidx = e;
            }
            const uint32_t wbest = __reduce_max_sync(0xffffffffu, best);
            if (k == K) { next = wbest; break; }
            const uint32_t widx = __reduce_min_sync(0xffffffffu, best == wbest ? bidx : 0xffffffffu);
            if ((widx & 31u) == (uint32_t)lane) sel |= 1u << (widx >> 5);
            kth = wbest;
        }
        float nu;
        if (K >= E) {
            nu = -INFINITY;   // y = 1 everywhere: the constraint leaves no freedom
        } else {
            // safeguarded Newton on f(nu) = sum_i sigmoid((r_i - nu)/tau) - K, which is strictly
            // decreasing with f' = -sum_i h_i: a Newton step that leaves the sign bracket
            // [lo, hi] is replaced by the bisection of the bracket.  It stops after a Newton step
            // below 2^-16 tau (that step taken): y then moves by less than 2^-18 per element,
            // under the float32 rounding noise of the sum f itself, which a tighter test could
            // only chase.  Every lane computes the same sums (xor butterfly), so the iteration is
            // identical across the warp.
            // With K > E/2 the sum is taken over the complements, f = (E - K) - sum_i
            // sigmoid((nu - r_i)/tau): the terms are then the small ones, and f keeps its
            // precision instead of being a difference of two numbers near K.
            lo -= 40.f * tau;
            hi += 40.f * tau;
            const float eps = 1.52587890625e-5f * tau;   // 2^-16 tau
            const bool comp = 2 * K > E;
            const float target = comp ? (float)(E - K) : (float)K;
            nu = 0.5f * (topk_value(kth) + topk_value(next));
            for (int it = 0; it < 100; ++it) {
                float s = 0.f, hs = 0.f;
#pragma unroll
                for (int j = 0; j < EPL; ++j) {
                    if (lane + 32 * j < E) {
                        const float zz = (v[j] - nu) * inv_tau;
                        const float y = sigmoid_f(comp ? -zz : zz);
                        s += y;
                        hs += y * (1.f - y);
                    }
                }
                s = warp_sum(s);
                hs = warp_sum(hs) * inv_tau;
                const float f = comp ? target - s : s - target;
                if (f > 0.f) lo = nu; else hi = nu;
                const float step = f / hs;
                float nn = nu + step;
                if (nn > lo && nn < hi) {
                    if (fabsf(step) <= eps) { nu = nn; break; }
                } else {
                    nn = 0.5f * (lo + hi);
                }
                if (nn == nu || nn <= lo || nn >= hi) break;   // the bracket is two adjacent floats
                nu = nn;
            }
        }
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E) y[t * E + e] = K >= E ? 1.f : sigmoid_f((v[j] - nu) * inv_tau);
        }
        if (nu_out && lane == 0) nu_out[t] = nu;
        if (mask) {
#pragma unroll
            for (int j = 0; j < EPL; ++j) {
                const int e = lane + 32 * j;
                if (e < E) mask[t * E + e] = (uint8_t)((sel >> j) & 1u);
            }
        }
    }
    pdl_launch_dependents();
}

template <int EPL>
__global__ void __launch_bounds__(256)
softtopk_bwd_kernel(const float* __restrict__ y, const float* __restrict__ dy, int T, int E,
                    float tau, float* __restrict__ dr)
{
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long t = (long long)blockIdx.x * 8 + warp;
    if (t < T) {
        const float inv_tau = 1.0f / tau;
        float h[EPL], g[EPL];
        float hs = 0.f, hd = 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            const float yv = e < E ? __ldg(y + t * E + e) : 0.f;
            g[j] = e < E ? __ldg(dy + t * E + e) : 0.f;
            h[j] = yv * (1.f - yv) * inv_tau;
            hs += h[j];
            hd += h[j] * g[j];
        }
        hs = warp_sum(hs);
        hd = warp_sum(hd);
        const float mean = hs > 0.f ? hd / hs : 0.f;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
            const int e = lane + 32 * j;
            if (e < E) dr[t * E + e] = h[j] * (g[j] - mean);
        }
    }
    pdl_launch_dependents();
}

}  // namespace beam
