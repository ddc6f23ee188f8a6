"""Pins of the oracle's training-side routing gradient (straight-through estimator + L_reg).

What is pinned: `oracle.route_backward`, the gradient of L = <dy, y> + reg_scale * L_reg with
respect to the router W_r, the mask router W_m and the routing's share of x, where the binary
mask's gradient is passed straight through to m_hat (BEAM article on aitrends.kr, training
paragraph: L = L_lm + alpha L_bal + beta L_reg, L_reg = (1/K) sum_{i in TK} |m_hat_i|, STE;
ai-feeds.com summary, Method, binarisation and straight-through estimator).

The main pin is an independent one: a straight-through surrogate written below in numpy,
whose exact derivative is the STE gradient, differenced numerically.  The surrogate replaces
the mask m by m0 + sigmoid(l) - sigmoid(l0), which equals m at the base point and has
d/dl = sigmoid'(l); the Top-K set and the expert outputs are held at their base values (the
selection is piecewise constant; the experts' own gradient is not part of the routing's).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_oracle_pins import closed_form

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(t):
    return t.detach().cpu().double().numpy()


def _np_expert(xv, wg, wu, wd):
    a = wg @ xv
    b = wu @ xv
    return wd @ (a / (1.0 + np.exp(-a)) * b)


class _Surrogate:
    """Straight-through surrogate of the layer's routing part, fp64, written from the formulas."""

    def __init__(self, x, w, K, S, dy, reg):
        self.K, self.S, self.dy, self.reg = K, max(1, S), dy, reg
        self.x0 = _f64(x)
        self.wr0, self.wm0 = _f64(w["w_router"]), _f64(w["w_mask"])
        wg, wu, wd = _f64(w["w_gate"]), _f64(w["w_up"]), _f64(w["w_down"])
        T = self.x0.shape[0]
        self.ids = np.zeros((T, K), int)
        self.m0 = np.zeros((T, K))
        self.sh0 = np.zeros((T, K))
        for t in range(T):
            src = self.S * (t // self.S)
            r = self.x0[src] @ self.wr0
            l = self.x0[src] @ self.wm0
            ids = np.lexsort((np.arange(r.size), -r))[:K]   # r descending, index ascending
            self.ids[t] = ids
            self.m0[t] = (l[ids] >= 0).astype(float)
            self.sh0[t] = 1.0 / (1.0 + np.exp(-l[ids]))
        # expert outputs at the base x, every Top-K slot (training evaluates them all)
        self.Ek = np.stack([np.stack([_np_expert(self.x0[t], wg[e], wu[e], wd[e])
                                      for e in self.ids[t]]) for t in range(T)])

    def __call__(self, x, wr, wm):
        T, K = x.shape[0], self.K
        total = 0.0
        for t in range(T):
            src = self.S * (t // self.S)
            ids = self.ids[t]
            r = x[src] @ wr[:, ids]
            g = np.exp(r - r.max())
            g /= g.sum()
            sh = 1.0 / (1.0 + np.exp(-(x[src] @ wm[:, ids])))
            gate = g * (self.m0[t] + sh - self.sh0[t])
            total += self.dy[t] @ (gate[:, None] * self.Ek[t]).sum(0)
            total += self.reg / (T * K) * sh.sum()
        return total


def _case(K=3, S=0, T=7, seed=3, keep=0.5, mask_zero=False, const_segments=False):
    spec = synth.LayerSpec("bwd", 16, 6, K, 8, storage="fp32")
    w = synth.make_layer(spec, seed=seed, keep_rate=None if mask_zero else keep)
    if mask_zero:
        w["w_mask"] = torch.zeros_like(w["w_mask"])
    x = synth.make_tokens(spec, T, seed=seed)
    if const_segments:
        for t in range(T):
            x[t] = x[S * (t // S)]
    dy = np.random.default_rng(seed).standard_normal((T, spec.d_model))
    return spec, w, x, dy


@pytest.mark.parametrize("S", [0, 3])
def test_gradient_matches_finite_differences_of_the_ste_surrogate(S):
    K, reg = 3, 0.7
    spec, w, x, dy = _case(K=K, S=S)
    r = oracle.route(x, w["w_router"], w["w_mask"], K, segment_len=S)
    got = oracle.route_backward(x, w, r, dy, reg_scale=reg, segment_len=S)
    f = _Surrogate(x, w, K, S, dy, reg)
    assert np.array_equal(f.ids, r.topk_id)          # the same Top-K sets, in rank order
    assert 0 < r.keep.sum() < r.keep.size            # masked and kept slots both present
    x0, wr0, wm0 = f.x0, f.wr0, f.wm0
    h = 1e-5
    rng = np.random.default_rng(11)

    def fd(which, idx):
        args = [x0.copy(), wr0.copy(), wm0.copy()]
        args[which][idx] += h
        up = f(*args)
        args[which][idx] -= 2 * h
        dn = f(*args)
        return (up - dn) / (2 * h)

    D, E = wr0.shape
    T = x0.shape[0]
    scale = max(np.abs(got.dw_r).max(), np.abs(got.dw_m).max(), np.abs(got.dx).max())
    # every router column and mask column at a few rows, and a sample of x entries
    for e in range(E):
        for d in rng.choice(D, 3, replace=False):
            assert fd(1, (d, e)) == pytest.approx(got.dw_r[d, e], abs=1e-7 * scale)
            assert fd(2, (d, e)) == pytest.approx(got.dw_m[d, e], abs=1e-7 * scale)
    for t in range(T):
        for d in rng.choice(D, 3, replace=False):
            assert fd(0, (t, d)) == pytest.approx(got.dx[t, d], abs=1e-7 * scale)
    # s is dL/dg_hat: the dot of dy with the slot's expert output
    assert np.allclose(got.s, np.einsum("td,tkd->tk", dy, f.Ek), rtol=1e-12, atol=1e-12)


def test_top1_router_gets_no_gradient():
    # the softmax over a single kept logit is the constant 1
    spec, w, x, dy = _case(K=1)
    r = oracle.route(x, w["w_router"], w["w_mask"], 1)
    got = oracle.route_backward(x, w, r, dy, reg_scale=0.5)
    assert np.all(got.d_r == 0.0) and np.all(got.dw_r == 0.0)
    assert np.any(got.dw_m != 0.0)


def test_zero_mask_router_has_quarter_slope():
    # W_m = 0 (the zero initialisation of the training paragraph): every m_hat is 1/2, all
    # slots are kept, and the sigmoid's slope there is exactly 1/4
    K, reg = 2, 0.9
    spec, w, x, dy = _case(K=K, mask_zero=True)
    r = oracle.route(x, w["w_router"], w["w_mask"], K)
    got = oracle.route_backward(x, w, r, dy, reg_scale=reg)
    T = x.shape[0]
    assert np.all(r.keep == 1)
    want = 0.25 * (got.s * r.g + reg / (T * K))
    assert np.allclose(got.d_l, want, rtol=1e-14, atol=1e-16)


def test_regulariser_alone_pulls_every_top_k_mask_logit_down():
    # dy = 0: only L_reg acts, dW_m[:, e] = reg/(T K) * sum over tokens with e in TK of
    # sigmoid'(l) x_t, and the router gets nothing
    K, reg = 3, 1.3
    spec, w, x, _ = _case(K=K)
    T, D = x.shape
    r = oracle.route(x, w["w_router"], w["w_mask"], K)
    got = oracle.route_backward(x, w, r, np.zeros((T, D)), reg_scale=reg)
    assert np.all(got.s == 0.0) and np.all(got.dw_r == 0.0) and np.all(got.d_r == 0.0)
    xm, wm = _f64(x), _f64(w["w_mask"])
    lz = xm @ wm                                          # [T][E] mask logits, dense
    sel = np.zeros_like(lz)
    sel[np.arange(T)[:, None], r.topk_id] = 1.0           # 1 on each token's Top-K
    slope = sel / (1.0 + np.exp(-lz)) / (1.0 + np.exp(lz))
    assert np.allclose(got.dw_m, reg / (T * K) * xm.T @ slope, rtol=1e-12, atol=1e-15)
    assert np.all(got.d_l > 0.0)


def test_segment_gradient_is_the_sum_over_its_tokens():
    # with x constant inside each segment, segment routing equals per-token routing, and the
    # leader's gradient is the sum of its tokens' per-token gradients
    K, S, reg = 3, 3, 0.4
    spec, w, x, dy = _case(K=K, S=S, T=8, const_segments=True)
    r1 = oracle.route(x, w["w_router"], w["w_mask"], K)
    rs = oracle.route(x, w["w_router"], w["w_mask"], K, segment_len=S)
    g1 = oracle.route_backward(x, w, r1, dy, reg_scale=reg)
    gs = oracle.route_backward(x, w, rs, dy, reg_scale=reg, segment_len=S)
    assert np.allclose(gs.dw_r, g1.dw_r, rtol=1e-12, atol=1e-14)
    assert np.allclose(gs.dw_m, g1.dw_m, rtol=1e-12, atol=1e-14)
    T = x.shape[0]
    for src in range(0, T, S):
        members = slice(src, min(T, src + S))
        assert np.allclose(gs.dx[src], g1.dx[members].sum(0), rtol=1e-12, atol=1e-14)
        assert np.allclose(gs.d_r[src], g1.d_r[members].sum(0), rtol=1e-12, atol=1e-14)
        assert np.all(gs.dx[src + 1:members.stop] == 0.0)


def test_selected_rows_agree_with_the_full_pass():
    K, S = 2, 2
    spec, w, x, dy = _case(K=K, S=S, T=9)
    r = oracle.route(x, w["w_router"], w["w_mask"], K, segment_len=S)
    full = oracle.route_backward(x, w, r, dy, reg_scale=0.2, segment_len=S)
    part = oracle.route_backward(x, w, r, dy, reg_scale=0.2, segment_len=S, rows=[2, 6, 8])
    assert part.dw_r is None
    for t in (2, 6, 8):
        assert np.array_equal(part.dx[t], full.dx[t])
        assert np.array_equal(part.d_l[t], full.d_l[t])


def test_hand_worked_gradient():
    """A one-token layer whose gradient is derived by hand in tests/golden (closed forms)."""
    with open(os.path.join(GOLDEN, "hand_worked_backward.json")) as f:
        case = json.load(f)["cases"][0]
    f32 = lambda a: torch.tensor(np.array(a, dtype=np.float64), dtype=torch.float32)
    cf = lambda rows: np.array([[closed_form(v) for v in row] for row in rows])
    w = dict(w_router=f32(cf(case["w_router"])), w_mask=f32(cf(case["w_mask"])),
             w_gate=f32(case["w_gate"]), w_up=f32(case["w_up"]), w_down=f32(case["w_down"]))
    x = f32(case["x"])
    r = oracle.route(x, w["w_router"], w["w_mask"], case["K"])
    ex = case["expect"]
    np.testing.assert_array_equal(r.topk_id, np.array(ex["topk_id"]))
    got = oracle.route_backward(x, w, r, np.array(case["dy"]), reg_scale=case["reg_scale"])
    # ln 3 and 1/2 pass through float32 inputs, hence rtol 1e-6
    for name, val in (("s", got.s), ("d_gate_logit", got.d_r), ("d_mask_logit", got.d_l),
                      ("dw_router", got.dw_r), ("dw_mask", got.dw_m), ("dx", got.dx)):
        np.testing.assert_allclose(val, cf(ex[name]), rtol=1e-6, atol=1e-12, err_msg=name)
