"""GPU parity of cross-layer routing (the mask generator of 'Stepped MoE: Segment-Level Routing
with Configurable Inference Complexity', core method, combined with BEAM's Steps 1-3) and of
the layer forward that takes its routing.

Acceptance is the layer's: on clean tokens (Top-K gap and |mask logit| above 1e-3 in the
oracle) the Top-K set, the rank order where adjacent gaps exceed 1e-3 and the keep map are
bit-exact; gates within 1e-4; per-layer active-expert sets exact where every token is clean
and always consistent with the GPU's own decisions; y within the layer's bf16 / fp32 bounds.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

GATE_TOL = 1e-4


def _generator(spec, L, T, seed, keep_rate=0.5):
    from dynamic_expert_routing_b200 import BeamGenerator
    wr, wm = synth.make_generator(spec, L, seed=seed, keep_rate=keep_rate)
    z = synth.make_tokens(spec, T, seed=seed + 50)
    gen = BeamGenerator(wr.cuda(), wm.cuda(), spec.top_k, max_tokens=T,
                        segment_len=spec.segment_len)
    return gen, wr, wm, z


def _bits(active_row: np.ndarray, E: int) -> np.ndarray:
    words = active_row.astype(np.int64) & 0xffffffff
    return np.array([(words[e // 32] >> (e % 32)) & 1 for e in range(E)], bool)


def _check_layer(out: dict, l: int, orr, E: int, K: int, mask_off: bool = False):
    ids = out["topk_id"][l]
    keep = out["keep"][l]
    T = ids.shape[0]
    assert ((ids >= 0) & (ids < E)).all()
    for t in range(T):
        assert len(set(ids[t].tolist())) == K
    clean = orr.clean(parity.MARGIN)
    for t in np.nonzero(clean)[0]:
        assert set(ids[t].tolist()) == set(orr.topk_id[t].tolist()), f"layer {l} token {t}: Top-K set"
        if orr.rank_gap[t] > parity.MARGIN:
            np.testing.assert_array_equal(ids[t], orr.topk_id[t], err_msg=f"layer {l} token {t}: rank order")
            np.testing.assert_allclose(out["gate"][l][t], orr.g[t], rtol=0, atol=GATE_TOL)
            np.testing.assert_allclose(out["ghat"][l][t], orr.ghat[t], rtol=0, atol=GATE_TOL)
        gk = {int(e): int(k) for e, k in zip(ids[t], keep[t])}
        ok = {int(e): int(k) for e, k in zip(orr.topk_id[t], orr.keep[t])}
        assert gk == ok, f"layer {l} token {t}: keep"
        assert abs(out["lreg"][l][t] - orr.lreg[t]) <= 1e-5
    # the GPU's own outputs are consistent with each other on every token
    np.testing.assert_array_equal(out["n_keep"][l], keep.sum(axis=1))
    np.testing.assert_array_equal(out["ghat"][l], np.where(keep == 1, out["gate"][l], 0.0))
    if mask_off:
        assert (keep == 1).all()
    own = np.zeros(E, bool)
    own[ids[keep.astype(bool)]] = True
    np.testing.assert_array_equal(_bits(out["active"][l], E), own)
    if clean.all():
        np.testing.assert_array_equal(own, oracle.active_experts(orr, E))
    return int(clean.sum())


GEN_CASES = [
    # name, spec, layers, tokens: tensor-core logits (>= 64 routed rows) and CUDA-core GEMV
    ("fine-seg16-tc", synth.SPECS["fine_seg16"], 3, 1100),
    ("fine-seg16-gemv", synth.SPECS["fine_seg16"], 3, 300),
    ("mixtral-l4", synth.SPECS["mixtral"], 4, 200),
    ("dsv2lite-l2", synth.SPECS["dsv2lite"], 2, 130),
    ("tiny-fp32-l2", synth.SPECS["tiny"], 2, 64),
    # 5 layers x 424 logit columns: one warp per column, with 1, 4 and 16 rows per warp
    ("fine-decode1", synth.SPECS["fine"], 5, 1),
    ("fine-l5-t3", synth.SPECS["fine"], 5, 3),
    ("fine-l5-t40", synth.SPECS["fine"], 5, 40),
]


@pytest.mark.parametrize("name,spec,L,T", GEN_CASES, ids=[c[0] for c in GEN_CASES])
@pytest.mark.parametrize("mask_off", [False, True], ids=["mask", "mask_off"])
def test_generator_matches_oracle(name, spec, L, T, mask_off):
    gen, wr, wm, z = _generator(spec, L, T, seed=3)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = gen.route(z.cuda(), mask_off=mask_off)
    gen.sync()
    got = {k: v.cpu().numpy() for k, v in out.items()}
    orrs = oracle.route_layers(z, wr, wm, spec.top_k, segment_len=spec.segment_len,
                               mask_off=mask_off)
    n_clean = 0
    for l in range(L):
        n_clean += _check_layer(got, l, orrs[l], spec.n_experts, spec.top_k, mask_off)
    if L * T >= 50:
        assert n_clean >= 0.8 * L * T, f"only {n_clean} of {L * T} token decisions are clean"
    # segment routing: every token carries its segment leader's decision
    S = max(1, spec.segment_len)
    for t in range(T):
        lead = (t // S) * S
        np.testing.assert_array_equal(got["topk_id"][:, t], got["topk_id"][:, lead])
        np.testing.assert_array_equal(got["ghat"][:, t], got["ghat"][:, lead])
    gen.close()


def test_generator_is_deterministic_and_reuses_outputs():
    spec = synth.SPECS["fine_seg16"]
    gen, wr, wm, z = _generator(spec, 3, 1100, seed=4)
    zd = z.cuda()
    a = gen.route(zd)
    b = {k: torch.full_like(v, 7) for k, v in a.items()}
    gen.route(zd, out=b)
    gen.sync()
    for k in a:
        assert torch.equal(a[k], b[k]), k
    gen.close()


def _layer_and_generator(spec, T, seed):
    """A layer and a one-layer generator holding the same router and mask-router matrices."""
    from dynamic_expert_routing_b200 import BeamGenerator, BeamMoE
    w = synth.make_layer(spec, seed=seed, keep_rate=0.5)
    w = {k: v for k, v in w.items() if isinstance(v, torch.Tensor) or v is None}
    wd = to_dev({k: v for k, v in w.items() if v is not None})
    layer = BeamMoE(wd, spec.top_k, max_tokens=T, segment_len=spec.segment_len)
    gen = BeamGenerator(wd["w_router"][None].contiguous(), wd["w_mask"][None].contiguous(),
                        spec.top_k, max_tokens=T, segment_len=spec.segment_len)
    return layer, gen, w


ROUTED_CASES = [
    ("dsv2lite-130", synth.SPECS["dsv2lite"], 130),    # shared experts, separate routing kernels
    ("dsv2lite-20", synth.SPECS["dsv2lite"], 20),      # the forward's single-kernel small routing
    ("fine-seg16-700", synth.SPECS["fine_seg16"], 700),
    ("tiny-fp32-64", synth.SPECS["tiny"], 64),          # CUDA-core expert path
]


@pytest.mark.parametrize("name,spec,T", ROUTED_CASES, ids=[c[0] for c in ROUTED_CASES])
def test_forward_routed_equals_forward(name, spec, T):
    """The generator's routing of x with the layer's own matrices, given to forward_routed,
    reproduces forward bit for bit: output, statistics and compaction."""
    layer, gen, _ = _layer_and_generator(spec, T, seed=8)
    x = synth.make_tokens(spec, T, seed=9).cuda()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y0 = layer.forward(x)
        torch.cuda.current_stream().synchronize()
        r0 = layer.routing(T)
        st0 = layer.stats()
        rt = gen.route(x)
        one = gen.layer(rt, 0)
        y1 = torch.full_like(y0, float("nan"))
        layer.forward_routed(x, one, out=y1)          # captured as a graph
        y1.fill_(float("nan"))
        layer.forward_routed(x, one, out=y1)          # replayed
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    r1 = layer.routing(T)
    st1 = layer.stats()
    for k in ("topk_id", "gate", "mask_logit", "keep", "offsets", "perm", "inv"):
        np.testing.assert_array_equal(r0[k], r1[k], err_msg=k)
    for k in ("avg_k", "n_active_experts", "n_tokens_all_masked", "tokens", "n_kept"):
        assert st0[k] == st1[k], k
    # small batches sum L_reg inside the forward's single-kernel routing, in another order
    assert st1["l_reg"] == pytest.approx(st0["l_reg"], rel=1e-12)
    np.testing.assert_array_equal(st0["counts"], st1["counts"])
    layer.close()
    gen.close()


@pytest.mark.parametrize("spec,T", [(synth.SPECS["dsv2lite"], 150), (synth.SPECS["fine_seg16"], 600)],
                         ids=["dsv2lite", "fine_seg16"])
def test_forward_routed_matches_oracle(spec, T):
    """Two layers routed by one generator pass over z (not the layers' inputs): each layer's
    output against the oracle's Step 4 with the routing the GPU produced."""
    from dynamic_expert_routing_b200 import BeamMoE
    L = 2
    gen, wr, wm, z = _generator(spec, L, T, seed=11)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        rt = gen.route(z.cuda())
    gen.sync()
    got = {k: v.cpu().numpy() for k, v in rt.items()}
    for l in range(L):
        w = synth.make_layer(spec, seed=20 + l, keep_rate=0.5)
        w = {k: v for k, v in w.items() if isinstance(v, torch.Tensor) or v is None}
        layer = BeamMoE(to_dev({k: v for k, v in w.items() if v is not None}), spec.top_k,
                        max_tokens=T, segment_len=spec.segment_len)
        x = synth.make_tokens(spec, T, seed=30 + l)
        with torch.cuda.stream(s):
            y = layer.forward_routed(x.cuda(), gen.layer(rt, l))
        torch.cuda.synchronize()
        r = oracle.Routing(got["topk_id"][l], got["gate"][l].astype(np.float64),
                           got["mask_logit"][l].astype(np.float64), got["keep"][l],
                           got["ghat"][l].astype(np.float64), None, None, None,
                           got["n_keep"][l], got["lreg"][l].astype(np.float64))
        y_ref = oracle.layer(x, w, r)
        parity.compare_y(y.cpu().numpy(), y_ref, spec.storage)
        st = layer.stats()
        assert st["n_kept"] == int(got["keep"][l].sum())
        assert st["avg_k"] == got["keep"][l].sum() / T
        layer.close()
    gen.close()


def test_forward_routed_rejects_bad_arguments():
    from dynamic_expert_routing_b200 import _lib
    spec = synth.SPECS["tiny"]
    layer, gen, _ = _layer_and_generator(spec, 16, seed=2)
    x = synth.make_tokens(spec, 16, seed=2).cuda()
    rt = gen.layer(gen.route(x), 0)
    r = _lib.BeamRouting(*[rt[k].data_ptr() if k in rt else None for k in
                           ("topk_id", "gate", "mask_logit", "keep", "ghat", "n_keep", "lreg", "active")])
    y = torch.empty((16, spec.d_model), device="cuda")
    lib = _lib.load()
    import ctypes
    for flags in (_lib.BEAM_MASK_OFF, _lib.BEAM_FUSED_DECODE):
        assert lib.beam_moe_forward_routed(layer._h, ctypes.c_void_p(x.data_ptr()), 16,
                                           ctypes.byref(r), ctypes.c_void_p(y.data_ptr()), flags,
                                           None) == _lib.BEAM_ERR_INVALID_ARG
    r.ghat = None
    assert lib.beam_moe_forward_routed(layer._h, ctypes.c_void_p(x.data_ptr()), 16, ctypes.byref(r),
                                       ctypes.c_void_p(y.data_ptr()), 0, None) == _lib.BEAM_ERR_INVALID_ARG
    torch.cuda.synchronize()
    layer.close()
    gen.close()
