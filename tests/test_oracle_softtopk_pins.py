"""Pins of the SoftTopK oracle (oracle/softtopk.py) to facts outside its own code.

SoftTopK ("Stepped MoE: Segment-Level Routing with Configurable Inference Complexity", its
SoftTopK entry) is read as the limited-multi-label projection: y = sigmoid((r - nu)/tau) with
sum(y) = K, the maximiser of <r, y>/tau + sum_i H(y_i) over {0 <= y <= 1, sum y = K}.  The pins:
  * closed forms: E = 2, K = 1 gives y_1 = sigmoid((r_1 - r_2) / (2 tau)); two equal-sized
    groups of equal logits with K = half of E give the same expression per group; equal logits
    give y = K / E; K = E gives y = 1;
  * the definition as an optimisation: y is feasible, and every feasible perturbation along
    sum-zero directions lowers the regularised objective;
  * the limit tau -> 0 is the hard Top-K indicator (a brute-force sort, ties to the lower index);
  * invariances: adding a constant to a row, scaling r and tau together;
  * the backward against central finite differences of <dy, y(r)>, and its two identities
    (rows of dr sum to zero; a constant dy gives dr = 0).
"""
import numpy as np
import pytest

from oracle.softtopk import hard_topk_mask, softtopk, softtopk_backward, softtopk_nu


def _sig(z):
    return 1.0 / (1.0 + np.exp(-z))


def _rand(T, E, seed, scale=2.0):
    return np.random.default_rng(seed).normal(0.0, scale, (T, E))


@pytest.mark.parametrize("tau", [0.05, 0.7, 3.0])
def test_two_experts_closed_form(tau):
    r = _rand(20, 2, 1)
    y, nu = softtopk(r, 1, tau)
    np.testing.assert_allclose(y[:, 0], _sig((r[:, 0] - r[:, 1]) / (2 * tau)), rtol=1e-12, atol=1e-15)
    # nu itself is pinned where f(nu) is not flat in float64 (|r_1 - r_2| well inside 40 tau)
    ok = np.abs(r[:, 0] - r[:, 1]) < 20 * tau
    assert ok.sum() >= 1
    np.testing.assert_allclose(nu[ok], r.mean(axis=1)[ok], rtol=1e-9, atol=1e-9)


def test_two_groups_closed_form():
    # n logits equal to a and n equal to b, K = n: by symmetry nu = (a + b) / 2
    n, a, b, tau = 5, 1.3, -0.4, 0.6
    r = np.array([[a] * n + [b] * n])
    y, _ = softtopk(r, n, tau)
    np.testing.assert_allclose(y[0, :n], _sig((a - b) / (2 * tau)), rtol=1e-12)
    np.testing.assert_allclose(y[0, n:], _sig((b - a) / (2 * tau)), rtol=1e-12)


@pytest.mark.parametrize("E,K", [(8, 3), (64, 6), (212, 16)])
def test_equal_logits_and_full_k(E, K):
    y, _ = softtopk(np.full((3, E), 0.37), K, 0.9)
    np.testing.assert_allclose(y, K / E, rtol=1e-12)
    y, nu = softtopk(_rand(3, E, 2), E, 0.9)
    assert (y == 1.0).all() and np.isneginf(nu).all()


@pytest.mark.parametrize("E,K,tau", [(8, 2, 0.5), (64, 6, 1.0), (212, 16, 0.2), (256, 200, 2.0)])
def test_feasible_and_optimal(E, K, tau):
    r = _rand(4, E, E + K)
    y, _ = softtopk(r, K, tau)
    assert ((y > 0) & (y < 1)).all()
    np.testing.assert_allclose(y.sum(axis=1), K, rtol=0, atol=1e-10 * E)

    def objective(yy, rr):
        yy = np.clip(yy, 1e-300, 1 - 1e-16)
        return (rr * yy).sum() / tau - (yy * np.log(yy) + (1 - yy) * np.log1p(-yy)).sum()

    # optimality on logits spread about tau, so that every y_i is well inside (0, 1) and a
    # second-order change of the objective is resolvable in float64
    r = _rand(4, E, E + K + 1, scale=tau)
    y, _ = softtopk(r, K, tau)
    rng = np.random.default_rng(7)
    for t in range(4):
        f0 = objective(y[t], r[t])
        for _ in range(20):
            d = rng.normal(size=E)
            d -= d.mean()                      # stays on sum(y) = K
            d *= 1e-3 * min(y[t].min(), 1 - y[t].max()) / np.abs(d).max()
            assert objective(y[t] + d, r[t]) < f0
            assert objective(y[t] - d, r[t]) < f0


@pytest.mark.parametrize("E,K", [(8, 2), (60, 4), (212, 16)])
def test_zero_temperature_limit_is_topk(E, K):
    rng = np.random.default_rng(E)
    # logits on a grid of step 0.01, shuffled: distinct values at least 0.01 apart
    r = np.stack([rng.permutation(E) * 0.01 for _ in range(6)]) - 0.5
    y, _ = softtopk(r, K, 1e-4)
    m = hard_topk_mask(r, K)
    np.testing.assert_allclose(y, m, atol=1e-12)
    # the brute-force sort of the hard mask: the K largest values, ties to the lower index
    for t in range(6):
        assert set(np.nonzero(m[t])[0]) == set(np.argsort(-r[t], kind="stable")[:K])
    tie = np.array([[1.0, 1.0, 0.0, 1.0]])
    np.testing.assert_array_equal(hard_topk_mask(tie, 2), [[1, 1, 0, 0]])


def test_invariances():
    r = _rand(5, 40, 3)
    y, nu = softtopk(r, 7, 0.8)
    y2, nu2 = softtopk(r + 3.25, 7, 0.8)
    np.testing.assert_allclose(y2, y, atol=1e-12)
    np.testing.assert_allclose(nu2, nu + 3.25, atol=1e-10)
    y3, _ = softtopk(2.5 * r, 7, 2.0)
    np.testing.assert_allclose(y3, y, atol=1e-12)


@pytest.mark.parametrize("E,K,tau", [(8, 2, 0.5), (33, 5, 1.3), (128, 16, 0.25)])
def test_backward_matches_finite_differences(E, K, tau):
    r = _rand(3, E, 11 + E, scale=1.0)
    dy = _rand(3, E, 12 + E, scale=1.0)
    y, _ = softtopk(r, K, tau)
    dr = softtopk_backward(y, dy, tau)
    eps = 1e-6
    fd = np.zeros_like(r)
    for j in range(E):
        rp = r.copy(); rp[:, j] += eps
        rm = r.copy(); rm[:, j] -= eps
        fd[:, j] = ((softtopk(rp, K, tau)[0] - softtopk(rm, K, tau)[0]) * dy).sum(axis=1) / (2 * eps)
    np.testing.assert_allclose(dr, fd, rtol=1e-5, atol=1e-8)
    np.testing.assert_allclose(dr.sum(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(softtopk_backward(y, np.full_like(y, 0.7), tau), 0.0, atol=1e-14)


def test_nu_bracket_and_arguments():
    r = _rand(2, 16, 5)
    nu = softtopk_nu(r, 4, 0.3)
    f = _sig((r - nu[:, None]) / 0.3).sum(axis=1)
    np.testing.assert_allclose(f, 4.0, atol=1e-10)
    with pytest.raises(ValueError):
        softtopk_nu(r, 0, 0.3)
    with pytest.raises(ValueError):
        softtopk_nu(r, 4, 0.0)
