"""Training-side routing gradient on the GPU vs the fp64 oracle (same seeded inputs).

The call under test is beam_moe_backward_router after a BEAM_TRAIN forward: the gradient of
L = <dy, y> + reg_scale * L_reg with respect to the router W_r, the mask router W_m and the
routing's share of x, with the binary mask's gradient passed straight through to m_hat (BEAM
article on aitrends.kr, training paragraph; ai-feeds.com summary, Method, binarisation and
straight-through estimator).

Acceptance, carried over from the forward's (the gradient is linear in the slot dots s, which
read the same expert outputs as y):
  * every token's Top-K set is the oracle's (asserted on every token: near-ties only swap ranks
    inside the set, so per-slot outputs are compared per (token, expert), not per rank), and dy
    is zero on tokens whose mask logit is within 1e-3 of 0 (there the mask, hence dL/dg, may
    legitimately differ);
  * bf16 layers: relative L2 <= 5e-3 and max |err| <= 2e-2 of the largest reference magnitude,
    per output (dW_r, dW_m, dx, and the per-slot d_gate_logit, d_mask_logit, s);
  * fp32 layers: relative L2 <= 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from dynamic_expert_routing_b200 import BeamMoE, BeamError
from dynamic_expert_routing_b200._lib import BEAM_ERR_INVALID_ARG, BEAM_ERR_NO_FORWARD
from tests import parity
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def _tol(storage):
    return (parity.TOL_BF16_REL, parity.TOL_BF16_ABS) if storage == "bf16" else (parity.TOL_F32_REL, None)


def _close(name, got, ref, storage):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rel, mx = _tol(storage)
    rl = parity.rel_l2(got, ref)
    assert rl <= rel, f"{name}: relative L2 {rl:.3e} > {rel}"
    if mx is not None and ref.size:
        err = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)
        assert err <= mx, f"{name}: max error {err:.3e} of the largest magnitude > {mx}"
    return rl


def _run(spec, T, seed=0, reg=0.5, path=None, keep_rate=0.5, weights=None, x=None, calls=2):
    if weights is None:
        weights = synth.make_layer(spec, seed=seed, keep_rate=keep_rate)
    if x is None:
        x = synth.make_tokens(spec, T, seed=seed)
    orr = oracle.route(x, weights["w_router"], weights["w_mask"], spec.top_k,
                       segment_len=spec.segment_len)
    dy = np.random.default_rng(seed + 7).standard_normal((T, spec.d_model)).astype(np.float32)
    dy[orr.m_margin <= parity.MARGIN] = 0.0
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        layer = BeamMoE(to_dev(weights), spec.top_k, T, segment_len=spec.segment_len)
        xd = x.cuda()
        dyd = torch.from_numpy(dy).cuda()
        y = torch.empty((T, spec.d_model), dtype=torch.float32, device="cuda")
        outs = []
        for _ in range(calls):   # the second forward replays the captured graph
            layer.forward(xd, path=path, out=y, train=True)
            outs.append(layer.backward_router(xd, dyd, reg_scale=reg, slots=True))
    torch.cuda.synchronize()
    gr = layer.routing(T)
    _same_sets(gr["topk_id"], orr.topk_id)
    got = {k: v.cpu().numpy() for k, v in outs[-1].items()}
    for o in outs[:-1]:            # bit-reproducible
        for k, v in o.items():
            assert np.array_equal(v.cpu().numpy(), got[k]), f"{k} differs between calls"
    ref = oracle.route_backward(x, weights, orr, dy.astype(np.float64), reg_scale=reg,
                                segment_len=spec.segment_len)
    return dict(layer=layer, y=y.cpu().numpy(), got=got, ref=ref, orr=orr, weights=weights, x=x,
                dy=dy, ids=gr["topk_id"])


def _same_sets(gid, oid):
    for t in range(gid.shape[0]):
        assert set(gid[t].tolist()) == set(oid[t].tolist()), f"Top-K set differs at token {t}"


def _by_expert(v, ids, E):
    """[T][K] per-slot values in rank order -> [T][E] by expert (0 off the Top-K)."""
    out = np.zeros((v.shape[0], E))
    np.put_along_axis(out, ids.astype(np.int64), v.astype(np.float64), axis=1)
    return out


def _check(r, storage):
    got, ref = r["got"], r["ref"]
    E = got["dw_router"].shape[1]
    gid, oid = r["ids"], r["orr"].topk_id
    out = {}
    out["dw_router"] = _close("dW_r", got["dw_router"], ref.dw_r, storage)
    out["dw_mask"] = _close("dW_m", got["dw_mask"], ref.dw_m, storage)
    out["dx"] = _close("dx", got["dx"], ref.dx, storage)
    for name, a, b in (("d_gate_logit", got["d_gate_logit"], ref.d_r),
                       ("d_mask_logit", got["d_mask_logit"], ref.d_l),
                       ("dghat", got["dghat"], ref.s)):
        _close(name, _by_expert(a, gid, E), _by_expert(b, oid, E), storage)
    return out


def _small(**kw):
    return synth.LayerSpec("small", 512, 16, 4, 256, storage="bf16").with_(**kw)


def test_tiny_fp32_gradient():
    spec = synth.SPECS["tiny"]
    r = _run(spec, 64, reg=0.8)
    _check(r, "fp32")
    # the training forward gives the inference y: masked slots only add 0 * E_i(x)
    y_ref = oracle.layer(r["x"], r["weights"], r["orr"])
    parity.compare_y(r["y"], y_ref, "fp32")
    st = r["layer"].stats()
    avg_k, l_reg, _ = oracle.stats(r["orr"])
    assert st["avg_k"] == pytest.approx(avg_k, abs=1e-12)
    assert st["n_kept"] == 64 * spec.top_k     # every Top-K slot evaluated


@pytest.mark.parametrize("T,path", [(100, None), (37, "stream"), (20, None)])
def test_small_bf16_gradient(T, path):
    spec = _small(n_shared=1, d_ff_shared=128)
    r = _run(spec, T, seed=T, path=path)
    _check(r, "bf16")
    y_ref = oracle.layer(r["x"], r["weights"], r["orr"])
    clean = r["orr"].clean()
    parity.compare_y(r["y"][clean], y_ref[clean], "bf16")


@pytest.mark.parametrize("E,K", [(8, 1), (32, 32), (212, 16), (64, 6)])
def test_topk_widths(E, K):
    spec = _small(n_experts=E, top_k=K, d_ff=128)
    r = _run(spec, 48, seed=E + K)
    _check(r, "bf16")
    if K == 1:   # a softmax over one logit is constant: no router gradient at all
        assert not r["got"]["dw_router"].any() and not r["got"]["d_gate_logit"].any()


def test_segment_routing_gradient():
    spec = _small(segment_len=16, n_shared=1, d_ff_shared=128)
    r = _run(spec, 16 * 4 + 5, seed=4)
    _check(r, "bf16")
    dx = r["got"]["dx"]
    for t in range(dx.shape[0]):
        if t % 16:
            assert not dx[t].any() and not r["got"]["d_mask_logit"][t].any()


def test_regulariser_only_and_zero_mask_router():
    # dy = 0 leaves only L_reg; with W_m = 0 every mask logit is 0 and its slope is 1/4
    spec = _small()
    w = synth.make_layer(spec, seed=9, keep_rate=None)
    w["w_mask"] = torch.zeros_like(w["w_mask"])
    x = synth.make_tokens(spec, 40, seed=9)
    layer = BeamMoE(to_dev(w), spec.top_k, 40)
    xd = x.cuda()
    layer.forward(xd, train=True)
    g = layer.backward_router(xd, torch.zeros((40, spec.d_model), device="cuda"), reg_scale=2.0,
                              slots=True)
    torch.cuda.synchronize()
    assert not g["dw_router"].any() and not g["dghat"].any()
    want = 0.25 * 2.0 / (40 * spec.top_k)
    assert torch.all(g["d_mask_logit"] == torch.tensor(want, dtype=torch.float32))


@pytest.mark.parametrize("name,T,n_rows", [("mixtral", 512, 4), ("dsv2lite", 700, 8),
                                          ("fine_seg16", 1000, 12)])
def test_model_shapes_sampled(name, T, n_rows):
    # the tensor-core path at the layer shapes: per-row outputs on sampled routed rows against
    # the oracle, dW against x^T times the GPU's own per-slot logit gradients in fp64 (a
    # property that holds at any size)
    spec = synth.SPECS[name]
    big = spec.n_experts * spec.d_ff * spec.d_model * 3 > 50_000_000
    dev = "cuda" if big else "cpu"
    w = synth.make_layer(spec, seed=2, keep_rate=0.5, device=dev)
    w = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    x = synth.make_tokens(spec, T, seed=2)
    orr = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=spec.segment_len)
    S = max(1, spec.segment_len)
    dy = np.random.default_rng(5).standard_normal((T, spec.d_model)).astype(np.float32)
    dy[orr.m_margin <= parity.MARGIN] = 0.0
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        layer = BeamMoE(to_dev(w), spec.top_k, T, segment_len=spec.segment_len)
        xd = x.cuda()
        layer.forward(xd, train=True)
        g = layer.backward_router(xd, torch.from_numpy(dy).cuda(), reg_scale=0.3, slots=True)
    torch.cuda.synchronize()
    got = {k: v.cpu().numpy().astype(np.float64) for k, v in g.items()}
    gr = layer.routing(T)
    _same_sets(gr["topk_id"], orr.topk_id)
    rows = np.arange(0, T, S)
    sample = rows[np.linspace(0, rows.size - 1, n_rows).astype(int)]
    ref = oracle.route_backward(x, w, orr, dy.astype(np.float64), reg_scale=0.3,
                                segment_len=spec.segment_len, rows=sample)
    E = spec.n_experts
    _close("dx", got["dx"][sample], ref.dx[sample], "bf16")
    for name_, a, b in (("d_gate_logit", got["d_gate_logit"], ref.d_r),
                        ("d_mask_logit", got["d_mask_logit"], ref.d_l),
                        ("dghat", got["dghat"], ref.s)):
        _close(name_, _by_expert(a[sample], gr["topk_id"][sample], E),
               _by_expert(b[sample], orr.topk_id[sample], E), "bf16")
    # dW = sum over routed rows of x[row] (x) the row's per-slot gradients, in fp64
    xf = x.double().numpy()
    dlr = np.zeros((T, E))
    dlm = np.zeros((T, E))
    ids = gr["topk_id"]
    for k in range(spec.top_k):
        dlr[rows, ids[rows, k]] += got["d_gate_logit"][rows, k]
        dlm[rows, ids[rows, k]] += got["d_mask_logit"][rows, k]
    assert parity.rel_l2(got["dw_router"], xf.T @ dlr) <= 1e-5
    assert parity.rel_l2(got["dw_mask"], xf.T @ dlm) <= 1e-5
    layer.close()


def test_argument_and_order_checks():
    spec = _small()
    w = synth.make_layer(spec, seed=1, keep_rate=0.5)
    x = synth.make_tokens(spec, 16, seed=1).cuda()
    layer = BeamMoE(to_dev(w), spec.top_k, 32)
    dy = torch.zeros((16, spec.d_model), device="cuda")
    with pytest.raises(BeamError) as e:        # no forward yet
        layer.backward_router(x, dy)
    assert e.value.status == BEAM_ERR_NO_FORWARD
    layer.forward(x)                           # an inference forward does not qualify
    with pytest.raises(BeamError) as e:
        layer.backward_router(x, dy)
    assert e.value.status == BEAM_ERR_NO_FORWARD
    layer.forward(x, train=True)
    with pytest.raises(BeamError) as e:        # another T than the forward's
        layer.backward_router(x[:8], dy[:8])
    assert e.value.status == BEAM_ERR_NO_FORWARD
    layer.backward_router(x, dy)               # the matching call works
    with pytest.raises(BeamError) as e:
        layer.forward(x, train=True, mask_off=True)
    assert e.value.status == BEAM_ERR_INVALID_ARG
    with pytest.raises(BeamError) as e:
        layer.forward(x, train=True, fused=True)
    assert e.value.status == BEAM_ERR_INVALID_ARG
    torch.cuda.synchronize()
