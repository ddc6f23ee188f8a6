"""fp64 CPU oracle of SoftTopK, the differentiable top-k of "Stepped MoE: Segment-Level Routing
with Configurable Inference Complexity" (paper.rainbus.top), its SoftTopK entry and the core
method: the mask generator's routing logits go through SoftTopK, a continuous relaxation of the
top-k indicator, so that the choice of experts passes gradients to the generator, while the
mask it hands to the layers is the {0,1} top-k mask.

TEST INFRASTRUCTURE ONLY: imported by the test suite, never by the library.  It shares no code
with the CUDA library.

The page names the relaxation but prints no formula.  The reading used here is the
limited-multi-label projection of Amos, Xu and Kolter ("The Limited Multi-Label Projection
Layer", 2019): for logits r [E], a temperature tau > 0 and 1 <= K < E,

    y = argmax_{0 <= y <= 1, sum(y) = K}  <r, y> / tau + sum_i H(y_i)   (H: binary entropy)

whose solution is y_i = sigmoid((r_i - nu) / tau), with the scalar nu chosen so that
sum_i y_i = K.  As tau -> 0, y tends to the top-k indicator whenever r_(K) > r_(K+1).  For
K = E the constraint forces y = 1 (nu = -inf) and every gradient is zero.  The {0,1} mask is
the hard Top-K indicator (ties to the lower index, as in the layer's router), and the
backward is the relaxation's:

    h_i = y_i (1 - y_i) / tau,    dr_j = h_j (dy_j - sum_i h_i dy_i / sum_i h_i)

(the derivative of y through nu(r), obtained by differentiating sum_i y_i = K).

Here nu is found by plain bisection in float64 on f(nu) = sum_i sigmoid((r_i - nu)/tau) - K,
which is strictly decreasing, over a bracket where f changes sign, until the bracket stops
shrinking.  Everything is float64 and vectorised over tokens only.
"""
from __future__ import annotations

import numpy as np


def _sigmoid(z):
    # 1 / (1 + e^-z) for z >= 0, e^z / (1 + e^z) below: neither form overflows, and small
    # values keep their relative precision (no 1 - (almost 1) cancellation)
    z = np.asarray(z, np.float64)
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def softtopk_nu(r, K: int, tau: float) -> np.ndarray:
    """nu [T] with sum_i sigmoid((r[t, i] - nu[t]) / tau) = K, by bisection (float64)."""
    r = np.asarray(r, np.float64)
    T, E = r.shape
    if not (1 <= K <= E) or not tau > 0:
        raise ValueError("need 1 <= K <= E and tau > 0")
    if K == E:
        return np.full(T, -np.inf)
    # at nu = min(r) - 40 tau every term exceeds 1 - 5e-18, so f = E - K > 0 in float64 terms;
    # at nu = max(r) + 40 tau every term is below 5e-18, so f = -K < 0
    lo = r.min(axis=1) - 40.0 * tau
    hi = r.max(axis=1) + 40.0 * tau
    for _ in range(400):
        mid = 0.5 * (lo + hi)
        f = _sigmoid((r - mid[:, None]) / tau).sum(axis=1) - K
        lo = np.where(f > 0, mid, lo)
        hi = np.where(f > 0, hi, mid)
        if np.all(hi - lo <= 4 * np.spacing(np.maximum(np.abs(lo), np.abs(hi)))):
            break
    return 0.5 * (lo + hi)


def softtopk(r, K: int, tau: float):
    """(y [T][E] relaxed mask, nu [T]) of the logits r [T][E]."""
    r = np.asarray(r, np.float64)
    nu = softtopk_nu(r, K, tau)
    if K == r.shape[1]:
        return np.ones_like(r), nu
    return _sigmoid((r - nu[:, None]) / tau), nu


def hard_topk_mask(r, K: int) -> np.ndarray:
    """The {0,1} Top-K indicator [T][E] (uint8), ties to the lower index."""
    r = np.asarray(r, np.float64)
    T, E = r.shape
    m = np.zeros((T, E), np.uint8)
    for t in range(T):
        # stable sort by value descending: equal values keep the lower index first
        order = sorted(range(E), key=lambda e: (-r[t, e], e))
        m[t, order[:K]] = 1
    return m


def softtopk_backward(y, dy, tau: float) -> np.ndarray:
    """dr [T][E] = the relaxation's Jacobian (through nu) applied to the upstream gradient dy."""
    y = np.asarray(y, np.float64)
    dy = np.asarray(dy, np.float64)
    h = y * (1.0 - y) / tau
    hs = h.sum(axis=1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        mean = np.where(hs > 0, (h * dy).sum(axis=1, keepdims=True) / np.where(hs > 0, hs, 1.0), 0.0)
    return h * (dy - mean)
