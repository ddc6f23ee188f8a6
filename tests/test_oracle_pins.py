"""Pins of the fp64 oracle against facts fixed by the BEAM pages and by mathematics.

None of these checks reuses the oracle's own code path: each compares it with a hand-worked
closed form, a library routine on a special case, an invariant, or a brute-force dense
evaluation written independently below.  Citations: the BEAM article on aitrends.kr
('BEAM: Dynamic MoE 라우팅을 위한 Binary Expert Activation Masking'), four-step pipeline
paragraph (Steps 1-4), training paragraph (L_reg, zero initialisation of the mask router),
results paragraph (Avg-K); the ai-feeds.com summary ('BEAM: 用于 MoE 动态路由的二进制专家激活掩码'),
Method (masked experts are skipped); and 'Stepped MoE: Segment-Level Routing with
Configurable Inference Complexity', core method (segment routing from the first position).
"""
import ast
import json
import math
import operator
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- closed-form evaluator
def _silu(z):
    return z / (1.0 + math.exp(-z))


def _sigmoid(z):
    return 1.0 / (1.0 + math.exp(-z))


_FUNCS = {"silu": _silu, "sigmoid": _sigmoid, "exp": math.exp}
_NAMES = {"ln3": math.log(3.0)}
_OPS = {ast.Add: operator.add, ast.Sub: operator.sub, ast.Mult: operator.mul,
        ast.Div: operator.truediv, ast.USub: operator.neg, ast.UAdd: operator.pos}


def closed_form(expr) -> float:
    """Evaluate a closed-form expression string (numbers, + - * /, silu, sigmoid, exp, ln3)."""
    if isinstance(expr, (int, float)):
        return float(expr)

    def ev(n):
        if isinstance(n, ast.Expression):
            return ev(n.body)
        if isinstance(n, ast.Constant):
            return float(n.value)
        if isinstance(n, ast.BinOp):
            return _OPS[type(n.op)](ev(n.left), ev(n.right))
        if isinstance(n, ast.UnaryOp):
            return _OPS[type(n.op)](ev(n.operand))
        if isinstance(n, ast.Call):
            return _FUNCS[n.func.id](*[ev(a) for a in n.args])
        if isinstance(n, ast.Name):
            return _NAMES[n.id]
        raise ValueError(f"unsupported node {n!r}")

    return ev(ast.parse(expr, mode="eval"))


def _f32(a):
    return torch.tensor(np.array(a, dtype=np.float64), dtype=torch.float32)


def _cf_matrix(rows):
    return _f32([[closed_form(v) for v in row] for row in rows])


# ---------------------------------------------------------------- hand-worked layers
def _hand_cases():
    with open(os.path.join(GOLDEN, "hand_worked.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", [c for c in _hand_cases() if "x" in c], ids=lambda c: c["name"])
def test_hand_worked_layer(case):
    x = _f32(case["x"])
    w = dict(w_router=_cf_matrix(case["w_router"]), w_mask=_cf_matrix(case["w_mask"]),
             w_gate=_f32(case["w_gate"]), w_up=_f32(case["w_up"]), w_down=_f32(case["w_down"]))
    if case.get("S", 0):
        w.update(ws_gate=_f32(case["ws_gate"]), ws_up=_f32(case["ws_up"]),
                 ws_down=_f32(case["ws_down"]))
    r = oracle.route(x, w["w_router"], w["w_mask"], case["K"])
    ex = case["expect"]
    np.testing.assert_array_equal(r.topk_id, np.array(ex["topk_id"]))
    np.testing.assert_array_equal(r.keep, np.array(ex["keep"]))
    # inputs were rounded to float32 (ln 3 is not representable), hence rtol 1e-6
    g = np.array([[closed_form(v) for v in row] for row in ex["g"]])
    np.testing.assert_allclose(r.g, g, rtol=1e-6, atol=1e-12)
    gh = np.array([[closed_form(v) for v in row] for row in ex["ghat"]])
    np.testing.assert_allclose(r.ghat, gh, rtol=1e-6, atol=1e-12)
    y = oracle.layer(x, w, r)
    ye = np.array([[closed_form(v) for v in row] for row in ex["y"]])
    np.testing.assert_allclose(y, ye, rtol=1e-6, atol=1e-12)
    avg_k, l_reg, _ = oracle.stats(r)
    assert avg_k == closed_form(ex["avg_k"])
    assert l_reg == pytest.approx(closed_form(ex["l_reg"]), rel=1e-12)


def test_hand_worked_swiglu_non_square():
    case = [c for c in _hand_cases() if c["name"] == "swiglu_non_square"][0]
    out = oracle.expert(np.array(case["x_vec"]), _f32(case["w_gate"]), _f32(case["w_up"]),
                        _f32(case["w_down"]))
    np.testing.assert_allclose(out, [closed_form(v) for v in case["expect"]["out"]],
                               rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------- independent dense evaluation
def _dense_reference(x, w, K, mask_off=False, segment_len=0, zero_mask_expected=False):
    """Brute force, written independently of the oracle: every expert is evaluated on every
    token with vectorised float64 numpy, then weighted by g_hat padded with zeros off TK."""
    xd = x.double().numpy()
    T, D = xd.shape
    wr = w["w_router"].double().numpy()
    wm = w["w_mask"].double().numpy()
    src = np.arange(T) if segment_len <= 1 else (np.arange(T) // segment_len) * segment_len
    r = xd[src] @ wr
    l = xd[src] @ wm
    E = r.shape[1]
    # stable sort of -r puts the lower index first among equal logits
    order = np.argsort(-r, axis=1, kind="stable")[:, :K]
    rk = np.take_along_axis(r, order, axis=1)
    g = np.exp(rk - rk[:, :1])
    g = g / g.sum(axis=1, keepdims=True)
    lk = np.take_along_axis(l, order, axis=1)
    keep = np.ones_like(lk) if mask_off else (lk >= 0).astype(np.float64)
    gfull = np.zeros((T, E))
    np.put_along_axis(gfull, order, g * keep, axis=1)
    wg = w["w_gate"].double().numpy()
    wu = w["w_up"].double().numpy()
    wd = w["w_down"].double().numpy()
    a = np.einsum("efd,td->tef", wg, xd)
    b = np.einsum("efd,td->tef", wu, xd)
    h = a / (1.0 + np.exp(-a)) * b
    ye = np.einsum("edf,tef->ted", wd, h)          # every expert on every token
    y = np.einsum("te,ted->td", gfull, ye)
    if w.get("ws_gate") is not None:
        sg = w["ws_gate"].double().numpy()
        su = w["ws_up"].double().numpy()
        sdn = w["ws_down"].double().numpy()
        a = np.einsum("sfd,td->tsf", sg, xd)
        b = np.einsum("sfd,td->tsf", su, xd)
        h = a / (1.0 + np.exp(-a)) * b
        y = y + np.einsum("sdf,tsf->td", sdn, h)
    sig = 1.0 / (1.0 + np.exp(-lk))
    return dict(order=order, g=g, keep=keep, y=y, lreg=sig.mean(axis=1), nkeep=keep.sum(axis=1))


def _small_spec(**kw):
    base = synth.LayerSpec("pin", 48, 6, 2, 32, storage="fp32")
    return base.with_(**kw)


@pytest.mark.parametrize("spec", [
    _small_spec(),
    _small_spec(n_shared=2, d_ff_shared=16),
    _small_spec(top_k=3, n_experts=7, storage="bf16"),
    _small_spec(segment_len=4, n_shared=1, d_ff_shared=8),
], ids=["plain", "shared", "bf16_k3", "segment4"])
def test_brute_force_dense(spec):
    T = 40
    x = synth.make_tokens(spec, T, seed=3)
    w = synth.make_layer(spec, seed=3, keep_rate=0.5)
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=spec.segment_len)
    ref = _dense_reference(x, w, spec.top_k, segment_len=spec.segment_len)
    np.testing.assert_array_equal(r.topk_id, ref["order"])
    np.testing.assert_allclose(r.g, ref["g"], rtol=1e-13, atol=0)
    np.testing.assert_array_equal(r.keep, ref["keep"])
    y = oracle.layer(x, w, r)
    scale = np.abs(ref["y"]).max()
    np.testing.assert_allclose(y, ref["y"], rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(r.lreg, ref["lreg"], rtol=1e-13)
    # some slots masked and some kept, so the check exercises both branches
    assert 0 < r.keep.sum() < r.keep.size


def test_zero_mask_router_is_standard_topk_moe():
    """W_m = 0 => sigmoid(0) = 1/2 >= 1/2 keeps every Top-K expert: BEAM reduces to Top-K MoE
    exactly (training paragraph, zero initialisation), and L_reg = 1/2 exactly."""
    spec = synth.SPECS["tiny"]
    x = synth.make_tokens(spec, 64)
    w = synth.make_layer(spec, zero_mask=True)
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    assert r.keep.all()
    np.testing.assert_array_equal(r.ghat, r.g)
    avg_k, l_reg, n0 = oracle.stats(r)
    assert avg_k == spec.top_k and l_reg == 0.5 and n0 == 0
    # standard Top-K MoE from library routines: torch.topk + torch.softmax in float64
    xd = x.double()
    logits = xd @ w["w_router"].double()
    val, idx = torch.topk(logits, spec.top_k, dim=1)
    gate = torch.softmax(val, dim=1)
    np.testing.assert_array_equal(r.topk_id, idx.numpy())
    np.testing.assert_allclose(r.g, gate.numpy(), rtol=1e-13)
    y = oracle.layer(x, w, r)
    yref = torch.zeros_like(xd)
    wg, wu, wd = (w[k].double() for k in ("w_gate", "w_up", "w_down"))
    for t in range(xd.shape[0]):
        for k in range(spec.top_k):
            e = int(idx[t, k])
            h = torch.nn.functional.silu(wg[e] @ xd[t]) * (wu[e] @ xd[t])
            yref[t] += gate[t, k] * (wd[e] @ h)
    np.testing.assert_allclose(y, yref.numpy(), rtol=0, atol=1e-12)


def test_mask_off_equals_zero_mask_router():
    spec = synth.SPECS["tiny"]
    x = synth.make_tokens(spec, 64)
    w = synth.make_layer(spec, keep_rate=0.5)
    w0 = dict(w, w_mask=torch.zeros_like(w["w_mask"]))
    a = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, mask_off=True)
    b = oracle.route(x, w0["w_router"], w0["w_mask"], spec.top_k)
    np.testing.assert_array_equal(a.topk_id, b.topk_id)
    np.testing.assert_array_equal(a.keep, b.keep)
    np.testing.assert_array_equal(a.ghat, b.ghat)
    np.testing.assert_array_equal(oracle.layer(x, w, a), oracle.layer(x, w0, b))


def test_k_equals_e_without_mask_is_dense_softmax_mixture():
    spec = _small_spec(top_k=6, n_experts=6)
    x = synth.make_tokens(spec, 16, seed=5)
    w = synth.make_layer(spec, seed=5)
    r = oracle.route(x, w["w_router"], w["w_mask"], 6, mask_off=True)
    y = oracle.layer(x, w, r)
    xd = x.double()
    p = torch.softmax(xd @ w["w_router"].double(), dim=1)
    yref = torch.zeros_like(xd)
    for e in range(6):
        h = torch.nn.functional.silu(xd @ w["w_gate"][e].double().T) * (xd @ w["w_up"][e].double().T)
        yref += p[:, e:e + 1] * (h @ w["w_down"][e].double().T)
    np.testing.assert_allclose(y, yref.numpy(), rtol=0, atol=1e-12)
    assert np.all(np.isinf(r.r_gap))


def test_all_masked_leaves_only_shared_experts():
    """No renormalisation (Step 4): a token with every Top-K slot masked gets the shared-expert
    term alone (zero without shared experts)."""
    spec = _small_spec(n_shared=2, d_ff_shared=16)
    x = synth.make_tokens(spec, 12, seed=7)
    w = synth.make_layer(spec, seed=7, mask_bias=-1.0e4)
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    assert r.keep.sum() == 0
    avg_k, _, n0 = oracle.stats(r)
    assert avg_k == 0 and n0 == 12
    y = oracle.layer(x, w, r)
    xd = x.double()
    ysh = torch.zeros_like(xd)
    for s in range(2):
        h = torch.nn.functional.silu(xd @ w["ws_gate"][s].double().T) * (xd @ w["ws_up"][s].double().T)
        ysh += h @ w["ws_down"][s].double().T
    np.testing.assert_allclose(y, ysh.numpy(), rtol=0, atol=1e-12)
    w_noshared = {k: v for k, v in w.items() if not k.startswith("ws_")}
    assert np.all(oracle.layer(x, w_noshared, r) == 0.0)


def test_avg_k_and_l_reg_definitions():
    """Avg-K is the mean number of kept experts per token; L_reg the mean of
    (1/K) sum_{i in TK} sigmoid(l_i), recomputed here from the exported mask logits."""
    spec = synth.SPECS["tiny"]
    x = synth.make_tokens(spec, 64)
    w = synth.make_layer(spec, keep_rate=0.5)
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    avg_k, l_reg, n0 = oracle.stats(r)
    assert avg_k == r.keep.sum() / 64.0
    sig = 1.0 / (1.0 + np.exp(-r.mask_logit))
    assert l_reg == pytest.approx(sig.mean(), rel=1e-14)
    assert n0 == int((r.keep.sum(axis=1) == 0).sum())
    np.testing.assert_array_equal(r.keep, (r.mask_logit >= 0).astype(np.uint8))


def test_exact_ties_lower_index_first():
    spec = _small_spec(n_experts=8, top_k=3)
    x = synth.make_tokens(spec, 32, seed=11)
    w = synth.make_layer(spec, seed=11)
    wr = w["w_router"].clone()
    wr[:, 5] = wr[:, 2]          # experts 2 and 5 now have identical logits
    wr[:, 7] = wr[:, 2]
    r = oracle.route(x, wr, w["w_mask"], 3)
    rl = x.double().numpy() @ wr.double().numpy()
    for t in range(32):
        want = sorted(range(8), key=lambda e: (-rl[t, e], e))[:3]
        assert list(r.topk_id[t]) == want
    assert (r.topk_id == 2).any()


def test_segment_routing_reuses_leader():
    spec = _small_spec(n_shared=1, d_ff_shared=8)
    T, S = 23, 5                              # last segment is partial
    x = synth.make_tokens(spec, T, seed=13)
    w = synth.make_layer(spec, seed=13, keep_rate=0.5)
    seg = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=S)
    per = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    for t in range(T):
        lead = (t // S) * S
        np.testing.assert_array_equal(seg.topk_id[t], per.topk_id[lead])
        np.testing.assert_array_equal(seg.ghat[t], per.ghat[lead])
    s1 = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=1)
    np.testing.assert_array_equal(s1.topk_id, per.topk_id)
    np.testing.assert_array_equal(s1.ghat, per.ghat)
    # the experts still see each token's own x
    ref = _dense_reference(x, w, spec.top_k, segment_len=S)
    np.testing.assert_allclose(oracle.layer(x, w, seg), ref["y"], rtol=0, atol=1e-12)


def test_compaction_against_python_sort():
    spec = synth.SPECS["tiny"]
    x = synth.make_tokens(spec, 64)
    w = synth.make_layer(spec, keep_rate=0.5)
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    counts, offsets, perm, inv = oracle.compact(r, spec.n_experts)
    K = spec.top_k
    pairs = [(int(r.topk_id[t, k]), t, k) for t in range(64) for k in range(K) if r.keep[t, k]]
    pairs.sort()
    assert list(perm) == [t * K + k for (_, t, k) in pairs]
    assert counts.sum() == r.keep.sum() == offsets[-1]
    assert list(counts) == [sum(1 for p in pairs if p[0] == e) for e in range(spec.n_experts)]
    for pos, i in enumerate(perm):
        assert inv[i] == pos
    assert (inv[r.keep.reshape(-1) == 0] == -1).all()


def test_bf16_inputs_widen_exactly():
    """A bf16 layer and the same values stored as fp32 give bit-identical oracle results."""
    spec = _small_spec(storage="bf16", n_shared=1, d_ff_shared=8)
    x = synth.make_tokens(spec, 24, seed=17)
    w = synth.make_layer(spec, seed=17, keep_rate=0.5)
    w32 = {k: (v.float() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    a = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    b = oracle.route(x.float(), w32["w_router"], w32["w_mask"], spec.top_k)
    np.testing.assert_array_equal(a.g, b.g)
    np.testing.assert_array_equal(oracle.layer(x, w, a), oracle.layer(x.float(), w32, b))


def test_cross_layer_routing_closed_form():
    """Cross-layer routing ('Stepped MoE: Segment-Level Routing with Configurable Inference
    Complexity', core method: one generator pass gives every layer's experts, once per
    segment, from the segment's first position).  Layer l's router reads channel
    1 + (e + l) mod 7 of z for expert e, so its Top-K in rank order are the channels holding
    the K largest values, mapped back through the shift by l.  Its mask router reads the
    constant channel z[:, 0] = 1 with sign + (even l) or - (odd l): every Top-K slot is kept
    in even layers and none in odd ones, with L_reg = sigmoid(+1) or sigmoid(-1)."""
    D, E, K, L, S, T = 8, 7, 3, 4, 2, 9     # the last segment is partial
    rs = np.random.default_rng(5)
    z = np.zeros((T, D), np.float32)
    z[:, 0] = 1.0
    for t in range(T):
        z[t, 1:] = rs.permutation(7).astype(np.float32) * 0.5 - 1.0   # distinct, exact
    wr = np.zeros((L, D, E), np.float32)
    wm = np.zeros((L, D, E), np.float32)
    for l in range(L):
        for e in range(E):
            wr[l, 1 + (e + l) % 7, e] = 1.0
        wm[l, 0, :] = 1.0 if l % 2 == 0 else -1.0
    rl = oracle.route_layers(torch.from_numpy(z), torch.from_numpy(wr), torch.from_numpy(wm), K,
                             segment_len=S)
    assert len(rl) == L
    sig = {1: 1.0 / (1.0 + math.exp(-1.0)), 0: 1.0 / (1.0 + math.exp(1.0))}
    for l, r in enumerate(rl):
        kept = 1 if l % 2 == 0 else 0
        want_act = np.zeros(E, bool)
        for t in range(T):
            lead = (t // S) * S
            channels = sorted(range(7), key=lambda j: -z[lead, 1 + j])[:K]
            want = [(j - l) % 7 for j in channels]
            assert list(r.topk_id[t]) == want
            assert (r.keep[t] == kept).all()
            assert r.nkeep[t] == K * kept
            assert r.lreg[t] == pytest.approx(sig[kept], abs=1e-15)
            if kept:
                want_act[want] = True
        np.testing.assert_array_equal(oracle.active_experts(r, E), want_act)


def test_cross_layer_routing_single_layer_is_layer_routing():
    """With one layer the generator's decision is the layer's own routing of the same input."""
    spec = _small_spec()
    x = synth.make_tokens(spec, 30, seed=21)
    w = synth.make_layer(spec, seed=21, keep_rate=0.5)
    (g,) = oracle.route_layers(x, w["w_router"][None], w["w_mask"][None], spec.top_k, segment_len=4)
    r = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=4)
    for f in ("topk_id", "g", "keep", "ghat", "nkeep", "lreg"):
        np.testing.assert_array_equal(getattr(g, f), getattr(r, f))
