"""SoftTopK on the GPU (beam_softtopk_forward / _backward) against the fp64 oracle.

The logits are float32 on both sides (the oracle widens the same values exactly).  Bars: the
hard Top-K mask bit-exact (selection on identical values, ties to the lower index); y within
2e-5 absolute (float32 bisection of nu and float32 sigmoids; y is in [0, 1]); the backward
within 1e-5 of the largest |dlogit| of the row plus 2e-5 relative (the same float32 error
carried through h = y (1 - y) / tau); nu where f(nu) is not flat within 1e-4 tau.
"""
import numpy as np
import pytest
import torch

from oracle.softtopk import hard_topk_mask, softtopk, softtopk_backward

pytestmark = pytest.mark.gpu


def _logits(T, E, seed, scale):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((T, E), generator=g, dtype=torch.float32) * scale


@pytest.mark.parametrize("T,E,K,tau,scale", [
    (1, 8, 2, 1.0, 1.0), (33, 8, 1, 0.3, 2.0), (100, 64, 6, 1.0, 1.0), (257, 60, 4, 0.5, 3.0),
    (64, 212, 16, 0.2, 1.0), (40, 256, 32, 2.0, 1.0), (17, 256, 255, 1.0, 1.0), (9, 33, 33, 1.0, 1.0),
    (1000, 212, 16, 1.0, 0.5),
], ids=["t1_e8", "k1_sharp", "e64", "e60_wide", "e212_sharp", "e256", "k_e_minus_1", "k_eq_e",
        "many_rows"])
def test_softtopk_matches_oracle(T, E, K, tau, scale):
    from dynamic_expert_routing_b200 import softtopk as gpu_softtopk
    from dynamic_expert_routing_b200 import softtopk_backward as gpu_backward
    r = _logits(T, E, T + E + K, scale)
    out = gpu_softtopk(r.cuda(), K, tau, mask=True, nu=True)
    y_ref, nu_ref = softtopk(r.double().numpy(), K, tau)
    y = out["y"].cpu().double().numpy()
    np.testing.assert_allclose(y, y_ref, atol=2e-5, rtol=0)
    np.testing.assert_array_equal(out["mask"].cpu().numpy(), hard_topk_mask(r.double().numpy(), K))
    nu = out["nu"].cpu().double().numpy()
    if K < E:
        h = y_ref * (1 - y_ref) / tau
        ok = h.sum(axis=1) > 1e-2 / tau       # nu is determined where f is not flat
        np.testing.assert_allclose(nu[ok], nu_ref[ok], atol=1e-4 * tau + 1e-5, rtol=1e-5)
    else:
        assert np.isneginf(nu).all()
    g = torch.Generator().manual_seed(99)
    dy = torch.randn((T, E), generator=g, dtype=torch.float32)
    dr = gpu_backward(out["y"], dy.cuda(), tau).cpu().double().numpy()
    dr_ref = softtopk_backward(y_ref, dy.double().numpy(), tau)
    bound = 1e-5 * np.abs(dr_ref).max(axis=1, keepdims=True) + 2e-5 * np.abs(dr_ref) + 1e-7 / tau
    assert (np.abs(dr - dr_ref) <= bound).all(), float(np.abs(dr - dr_ref).max())
    np.testing.assert_allclose(dr.sum(axis=1), 0.0, atol=1e-4 * (np.abs(dr).max() + 1e-6))


def test_softtopk_ties_and_deterministic():
    from dynamic_expert_routing_b200 import softtopk as gpu_softtopk
    r = _logits(50, 64, 5, 1.0)
    r[:, 9] = r[:, 3]          # exact ties: the lower index ranks first
    r[:, 40] = r[:, 3]
    a = gpu_softtopk(r.cuda(), 8, 0.7)
    b = gpu_softtopk(r.cuda(), 8, 0.7)
    assert torch.equal(a["y"], b["y"]) and torch.equal(a["mask"], b["mask"])
    np.testing.assert_array_equal(a["mask"].cpu().numpy(), hard_topk_mask(r.double().numpy(), 8))
    y = a["y"].cpu().numpy()
    np.testing.assert_array_equal(y[:, 9], y[:, 3])     # equal logits, equal relaxed mask
    np.testing.assert_allclose(y.sum(axis=1), 8.0, rtol=2e-6)


def test_softtopk_argument_checks():
    from dynamic_expert_routing_b200 import BeamError, softtopk as gpu_softtopk
    r = torch.zeros((4, 8), device="cuda")
    for K, tau in ((0, 1.0), (9, 1.0), (2, 0.0), (2, float("nan"))):
        with pytest.raises(BeamError):
            gpu_softtopk(r, K, tau)
    out = gpu_softtopk(torch.zeros((0, 8), device="cuda"), 2, 1.0)
    assert out["y"].shape == (0, 8)
