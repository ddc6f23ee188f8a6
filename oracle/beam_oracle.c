/*
 * beam_oracle.c -- plain, slow, fp64 CPU oracle of the BEAM masked MoE-layer forward, and of
 * the training-side gradient of its routing (oracle_route_backward, at the end of the file).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference for the CUDA library.
 * Only the test suite, the package smoke check and the bench's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA library; the two only receive the
 * same seeded input tensors.
 *
 * What it computes follows the BEAM pages:
 *   [BEAM-KR] "BEAM: Dynamic MoE 라우팅을 위한 Binary Expert Activation Masking" (aitrends.kr
 *             article), the four-step pipeline paragraph: Step 1 Standard Top-K routing,
 *             Step 2 raw mask m_hat = sigmoid(x W_m), Step 3 binary masking m_i = 1 iff
 *             m_hat_i >= 0.5, Step 4 masked aggregation g_hat = g (.) m, y = sum g_hat_i E_i(x);
 *             training paragraph for L_reg = (1/K) sum_{i in TK} |m_hat_i|; results paragraph
 *             for Avg-K; limitation (C) for always-on shared experts.
 *   [BEAM-CN] "BEAM: 用于 MoE 动态路由的二进制专家激活掩码" (ai-feeds.com summary), Method,
 *             "输出与推理加速": experts whose mask is 0 are skipped.
 *   [SMoE]    "Stepped MoE: Segment-Level Routing with Configurable Inference Complexity"
 *             (paper.rainbus.top), 核心方法 / 方法步骤详情: experts are chosen once per segment
 *             of S tokens from the segment's first position.
 * Readings where the pages are silent (each also listed in the design notes):
 *   - softmax over the K kept logits; Top-K ties go to the lower expert index;
 *   - W_m has the shape of W_r ([D][E]); the mask acts only on the Top-K slots;
 *   - the threshold m_hat >= 0.5 is evaluated as mask logit >= 0 (equivalent in exact
 *     arithmetic because the sigmoid is increasing with sigmoid(0) = 1/2);
 *   - no renormalisation after masking; shared experts are added with weight 1;
 *   - the expert FFN is SwiGLU without biases: E(x) = W_d (silu(W_g x) * (W_u x));
 *   - L_reg and Avg-K are means over tokens; perm orders kept (token, slot) pairs by expert,
 *     then token.
 *
 * Storage: inputs are float32 (dtype 0) or bfloat16 bit patterns (dtype 1); every element is
 * widened exactly to double and all arithmetic is double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double load_elem(const void *base, int dtype, size_t i)
{
    if (dtype == 0) return (double)((const float *)base)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }
static double silu(double z) { return z / (1.0 + exp(-z)); }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One SwiGLU expert on one token: out[j] = sum_f Wd[j][f] * silu(sum_d Wg[f][d] x[d]) *
 * (sum_d Wu[f][d] x[d]).  Wg, Wu are [F][D]; Wd is [D][F]; x is double[D].
 */
static void expert_ffn(int D, int F, int dtype, const double *x,
                       const void *wg, const void *wu, const void *wd,
                       size_t wg_off, size_t wd_off, double *h, double *out)
{
    for (int f = 0; f < F; ++f) {
        double a = 0.0, b = 0.0;
        for (int d = 0; d < D; ++d) {
            a += load_elem(wg, dtype, wg_off + (size_t)f * D + d) * x[d];
            b += load_elem(wu, dtype, wg_off + (size_t)f * D + d) * x[d];
        }
        h[f] = silu(a) * b;
    }
    for (int j = 0; j < D; ++j) {
        double acc = 0.0;
        for (int f = 0; f < F; ++f)
            acc += load_elem(wd, dtype, wd_off + (size_t)j * F + f) * h[f];
        out[j] = acc;
    }
}

/* Public wrapper used by the closed-form pins: expert `e` of a stacked weight set. */
int oracle_expert(int D, int F, int dtype, const double *x, const void *wg, const void *wu,
                  const void *wd, int e, double *out)
{
    double *h = (double *)malloc(sizeof(double) * (size_t)F);
    if (!h) return 2;
    expert_ffn(D, F, dtype, x, wg, wu, wd, (size_t)e * F * D, (size_t)e * D * F, h, out);
    free(h);
    return 0;
}

/*
 * Routing, Steps 1-3 of [BEAM-KR] plus the per-token statistics, for every token.
 *
 *   r_e = sum_d x[src][d] W_r[d][e];  l_e = sum_d x[src][d] W_m[d][e]          (e < E)
 *   TK  = first K experts under the order (r desc, index asc)
 *   g_k = exp(r_k - r_max) / sum_{j in TK} exp(r_j - r_max)                   (k < K)
 *   keep_k = (l_k >= 0), or 1 when mask_off;  g_hat_k = g_k * keep_k
 *   nkeep(t) = sum_k keep_k;  lreg(t) = (1/K) sum_k sigmoid(l_k)
 *
 * src = t, or the first token of t's segment when seg > 1 ([SMoE]).
 * Diagnostics for the parity rule: r_gap(t) = r_(K) - r_(K+1) (+inf when K == E),
 * rank_gap(t) = min over adjacent Top-K ranks of r_(k) - r_(k+1) (+inf when K == 1),
 * m_margin(t) = min_k |l_k| over TK (+inf when mask_off).
 * Outputs are [T][K] in rank order, except the per-token arrays.
 */
int oracle_route(int T, int D, int E, int K, int dtype, int seg, int mask_off,
                 const void *x, const void *w_router, const void *w_mask,
                 int32_t *topk_id, double *g, double *mlogit, uint8_t *keep, double *ghat,
                 double *r_gap, double *rank_gap, double *m_margin,
                 int32_t *nkeep_tok, double *lreg_tok)
{
    if (T < 0 || D <= 0 || E <= 0 || K <= 0 || K > E || K > 256) return 1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 4)
    for (int t = 0; t < T; ++t) {
        double *r = (double *)malloc(sizeof(double) * (size_t)E);
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        char *chosen = (char *)calloc((size_t)E, 1);
        if (!r || !l || !chosen) {
            bad = 1;
            free(r); free(l); free(chosen);
            continue;
        }
        int src = (seg > 1) ? seg * (t / seg) : t;
        for (int e = 0; e < E; ++e) {
            double a = 0.0, b = 0.0;
            for (int d = 0; d < D; ++d) {
                double xv = load_elem(x, dtype, (size_t)src * D + d);
                a += xv * load_elem(w_router, dtype, (size_t)d * E + e);
                b += xv * load_elem(w_mask, dtype, (size_t)d * E + e);
            }
            r[e] = a;
            l[e] = b;
        }
        /* Top-K by repeated selection: the first maximum in index order wins a tie. */
        int ids[256];
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!chosen[e] && (best < 0 || r[e] > r[best])) best = e;
            chosen[best] = 1;
            ids[k] = best;
        }
        double next = -INFINITY;
        for (int e = 0; e < E; ++e)
            if (!chosen[e] && r[e] > next) next = r[e];
        r_gap[t] = (K < E) ? r[ids[K - 1]] - next : INFINITY;
        double rg = INFINITY;
        for (int k = 0; k + 1 < K; ++k) {
            double dlt = r[ids[k]] - r[ids[k + 1]];
            if (dlt < rg) rg = dlt;
        }
        rank_gap[t] = rg;

        double rmax = r[ids[0]], den = 0.0;
        for (int k = 0; k < K; ++k) den += exp(r[ids[k]] - rmax);
        int nk = 0;
        double ls = 0.0, mm = INFINITY;
        for (int k = 0; k < K; ++k) {
            size_t o = (size_t)t * K + k;
            int e = ids[k];
            topk_id[o] = e;
            g[o] = exp(r[e] - rmax) / den;
            mlogit[o] = l[e];
            keep[o] = mask_off ? 1 : (l[e] >= 0.0 ? 1 : 0);
            ghat[o] = g[o] * (double)keep[o];
            nk += keep[o];
            ls += sigmoid(l[e]);
            if (fabs(l[e]) < mm) mm = fabs(l[e]);
        }
        nkeep_tok[t] = nk;
        lreg_tok[t] = ls / (double)K;
        m_margin[t] = mask_off ? INFINITY : mm;
        free(r); free(l); free(chosen);
    }
    return bad ? 2 : 0;
}

/*
 * Avg-K = (1/T) sum_t nkeep(t) and L_reg = (1/T) sum_t lreg(t) ([BEAM-KR] results and
 * training paragraphs), plus the number of tokens with every Top-K slot masked.
 */
int oracle_stats(int T, const int32_t *nkeep_tok, const double *lreg_tok,
                 double *avg_k, double *l_reg, int32_t *n_all_masked)
{
    long long s = 0;
    double ls = 0.0;
    int nz = 0;
    for (int t = 0; t < T; ++t) {
        s += nkeep_tok[t];
        ls += lreg_tok[t];
        if (nkeep_tok[t] == 0) ++nz;
    }
    *avg_k = T ? (double)s / (double)T : 0.0;
    *l_reg = T ? ls / (double)T : 0.0;
    *n_all_masked = nz;
    return 0;
}

/*
 * Grouping of the kept (token, slot) pairs by expert ([BEAM-CN]: only kept experts run).
 * counts[e] = number of kept slots routed to e; offsets = exclusive prefix sum (E+1 entries);
 * perm lists t*K + k for every kept pair, ordered by expert, then token; inv[t*K+k] is the
 * position of that pair in perm, or -1 when the slot is masked.
 */
int oracle_compact(int T, int K, int E, const int32_t *topk_id, const uint8_t *keep,
                   int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int i = 0; i < T * K; ++i) {
        inv[i] = -1;
        if (keep[i]) {
            int e = topk_id[i];
            if (e < 0 || e >= E) return 1;
            counts[e]++;
        }
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int pos = 0;
    for (int e = 0; e < E; ++e)
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k) {
                int i = t * K + k;
                if (keep[i] && topk_id[i] == e) {
                    perm[pos] = i;
                    inv[i] = pos;
                    ++pos;
                }
            }
    return 0;
}

/*
 * Step 4 of [BEAM-KR] for the tokens listed in sel[0..n_sel):
 *   y[t] = sum_{k in rank order, keep_k = 1} g_hat_k E_{id_k}(x[t]) + sum_s E^sh_s(x[t]).
 * Routing arrays come from oracle_route (all T tokens); with segment routing they already
 * hold the leader's decision, while the experts always see the token's own x[t].
 * y is double[n_sel][D].  Shared weights may be NULL when S_sh == 0.
 */
int oracle_layer(int T, int D, int E, int K, int F, int S_sh, int Fs, int dtype,
                 const void *x, const void *wg, const void *wu, const void *wd,
                 const void *wsg, const void *wsu, const void *wsd,
                 const int32_t *topk_id, const double *ghat, const uint8_t *keep,
                 int n_sel, const int32_t *sel, double *y)
{
    (void)E;
    int bad = 0;
    int Fmax = F > Fs ? F : Fs;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_sel; ++i) {
        int t = sel[i];
        double *xv = (double *)malloc(sizeof(double) * (size_t)D);
        double *h = (double *)malloc(sizeof(double) * (size_t)(Fmax > 0 ? Fmax : 1));
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
        double *yt = y + (size_t)i * D;
        if (!xv || !h || !o || t < 0 || t >= T) {
            bad = 1;
            free(xv); free(h); free(o);
            continue;
        }
        for (int d = 0; d < D; ++d) {
            xv[d] = load_elem(x, dtype, (size_t)t * D + d);
            yt[d] = 0.0;
        }
        for (int k = 0; k < K; ++k) {
            size_t s = (size_t)t * K + k;
            if (!keep[s]) continue;            /* masked expert: skipped, never evaluated */
            int e = topk_id[s];
            expert_ffn(D, F, dtype, xv, wg, wu, wd, (size_t)e * F * D, (size_t)e * D * F, h, o);
            for (int d = 0; d < D; ++d) yt[d] += ghat[s] * o[d];
        }
        for (int sh = 0; sh < S_sh; ++sh) {
            expert_ffn(D, Fs, dtype, xv, wsg, wsu, wsd, (size_t)sh * Fs * D,
                       (size_t)sh * D * Fs, h, o);
            for (int d = 0; d < D; ++d) yt[d] += o[d];
        }
        free(xv); free(h); free(o);
    }
    return bad ? 1 : 0;
}

/*
 * Training-side gradient of the routing ([BEAM-KR] training paragraph: the loss
 * L = L_lm + alpha L_bal + beta L_reg with L_reg = (1/K) sum_{i in TK} |m_hat_i|, and the
 * straight-through estimator that lets the binary mask's gradient flow to m_hat; [BEAM-CN]
 * Method, "二值化与直通估计器": a step function forward, the continuous version's gradient
 * backward).  Readings: L_bal is not defined on the pages and is left out; L_reg is the mean
 * over tokens of the per-token term (as in the forward's statistics), so with reg_scale =
 * dL/dL_reg every (token, slot) adds reg_scale / (T K) to dL/dm_hat; the straight-through
 * estimator sets dm/dm_hat = 1; during training every Top-K expert is evaluated (the mask's
 * gradient needs E_i(x) of masked slots too) while the output uses g_hat = g * m.
 *
 * Given dy = dL_lm/dy [T][D], per token t and Top-K slot k (expert i):
 *   s_tk   = <dy_t, E_i(x_t)>                        (= dL/dg_hat_tk)
 *   dg_k   = sum over the routed row's tokens of s_tk * m_k
 *   dmh_k  = sum over the routed row's tokens of (s_tk * g_k + reg_scale / (T K))
 *   d_l_k  = dmh_k * sigmoid(l_k) (1 - sigmoid(l_k))       (mask logit)
 *   d_r_k  = g_k (dg_k - sum_j g_j dg_j)                  (softmax over the K)
 * with m_k = (l_k >= 0); logits outside TK get no gradient (the Top-K selection is piecewise
 * constant).  The routed row of token t is t itself, or its segment's first token ([SMoE]):
 * the segment's tokens share one decision, so their terms are summed at the leader.  Then
 *   dW_r[d][i] = sum over routed rows of x[row][d] d_r_k;  dW_m likewise with d_l_k
 *   dx[row][d] = sum_k d_r_k W_r[d][i_k] + d_l_k W_m[d][i_k]   (the routing's share of dx;
 *                rows that are not routed rows get 0)
 * s, d_r and d_l are [T][K] (d_r, d_l at routed rows, 0 elsewhere); dw_r, dw_m [D][E];
 * dx [T][D].  sel == NULL: every routed row and dW; otherwise only the n_sel routed rows
 * listed in sel (token indices of routed rows) and dw_r / dw_m are left untouched.
 * topk_id, g and mlogit are oracle_route's outputs (already carrying the leader's decision).
 */
int oracle_route_backward(int T, int D, int E, int K, int F, int dtype, int seg,
                          const void *x, const void *w_router, const void *w_mask,
                          const void *wg, const void *wu, const void *wd,
                          const int32_t *topk_id, const double *g, const double *mlogit,
                          const double *dy, double reg_scale, int n_sel, const int32_t *sel,
                          double *s_out, double *d_r, double *d_l,
                          double *dw_r, double *dw_m, double *dx)
{
    if (T < 0 || D <= 0 || E <= 0 || K <= 0 || K > E || K > 256 || F <= 0) return 1;
    const int S = seg > 1 ? seg : 1;
    const int n_rows = (T + S - 1) / S;
    const int n = sel ? n_sel : n_rows;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < n; ++q) {
        const int src = sel ? sel[q] : q * S;
        double *xv = (double *)malloc(sizeof(double) * (size_t)D);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
        double dg[256], dmh[256];
        if (!xv || !h || !o || src < 0 || src >= T || src % S) {
            bad = 1;
            free(xv); free(h); free(o);
            continue;
        }
        for (int k = 0; k < K; ++k) dg[k] = dmh[k] = 0.0;
        const int t_end = src + S < T ? src + S : T;
        for (int t = src; t < t_end; ++t) {
            for (int d = 0; d < D; ++d) xv[d] = load_elem(x, dtype, (size_t)t * D + d);
            for (int k = 0; k < K; ++k) {
                const size_t sl = (size_t)t * K + k;
                const int e = topk_id[sl];
                expert_ffn(D, F, dtype, xv, wg, wu, wd, (size_t)e * F * D, (size_t)e * D * F, h, o);
                double s = 0.0;
                for (int d = 0; d < D; ++d) s += dy[(size_t)t * D + d] * o[d];
                s_out[sl] = s;
                const double m = mlogit[sl] >= 0.0 ? 1.0 : 0.0;
                dg[k] += s * m;
                dmh[k] += s * g[sl] + reg_scale / ((double)T * (double)K);
                if (t != src) { d_r[sl] = 0.0; d_l[sl] = 0.0; }
            }
        }
        double c = 0.0;
        for (int k = 0; k < K; ++k) c += g[(size_t)src * K + k] * dg[k];
        for (int k = 0; k < K; ++k) {
            const size_t sl = (size_t)src * K + k;
            const double sg = sigmoid(mlogit[sl]);
            d_l[sl] = dmh[k] * sg * (1.0 - sg);
            d_r[sl] = g[sl] * (dg[k] - c);
        }
        for (int d = 0; d < D; ++d) {
            double a = 0.0;
            for (int k = 0; k < K; ++k) {
                const size_t sl = (size_t)src * K + k;
                const int e = topk_id[sl];
                a += d_r[sl] * load_elem(w_router, dtype, (size_t)d * E + e) +
                     d_l[sl] * load_elem(w_mask, dtype, (size_t)d * E + e);
            }
            dx[(size_t)src * D + d] = a;
        }
        for (int t = src + 1; t < t_end; ++t)
            for (int d = 0; d < D; ++d) dx[(size_t)t * D + d] = 0.0;
        free(xv); free(h); free(o);
    }
    if (bad) return 2;
    if (sel) return 0;
    for (size_t i = 0; i < (size_t)D * E; ++i) dw_r[i] = dw_m[i] = 0.0;
    for (int src = 0; src < T; src += S)
        for (int k = 0; k < K; ++k) {
            const size_t sl = (size_t)src * K + k;
            const int e = topk_id[sl];
            for (int d = 0; d < D; ++d) {
                const double xd = load_elem(x, dtype, (size_t)src * D + d);
                dw_r[(size_t)d * E + e] += xd * d_r[sl];
                dw_m[(size_t)d * E + e] += xd * d_l[sl];
            }
        }
    return 0;
}
