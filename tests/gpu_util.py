"""Helpers for the GPU parity tests: build a layer on both sides from one seeded input set."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from tests import parity


def to_dev(w: dict, device="cuda") -> dict:
    return {k: (v.to(device).contiguous() if isinstance(v, torch.Tensor) else v)
            for k, v in w.items()}


def same_decision_tokens(gr: dict, orr) -> np.ndarray:
    """Tokens whose GPU Top-K set and keep map equal the oracle's (all clean tokens qualify)."""
    T = orr.topk_id.shape[0]
    ok = np.zeros(T, bool)
    for t in range(T):
        gk = {int(e): int(k) for e, k in zip(gr["topk_id"][t], gr["keep"][t])}
        ok_ = {int(e): int(k) for e, k in zip(orr.topk_id[t], orr.keep[t])}
        ok[t] = gk == ok_
    return ok


def run_case(spec: synth.LayerSpec, T: int, seed: int = 0, keep_rate=0.5, mask_off=False,
             path=None, zero_mask=False, mask_bias=None, max_tokens=None, y_tokens=None,
             layer=None, weights=None, x=None, fused=False, case=None):
    """Run the CUDA layer and the oracle on the same inputs; assert parity; return details."""
    from dynamic_expert_routing_b200 import BeamMoE
    big = spec.n_experts * spec.d_ff * spec.d_model * 3 > 50_000_000
    gen = "cuda" if big else "cpu"   # large layers are drawn on the device, then copied
    if weights is None:
        weights = synth.make_layer(spec, seed=seed, keep_rate=keep_rate, zero_mask=zero_mask,
                                   mask_bias=mask_bias, device=gen)
        weights = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in weights.items()}
    if x is None:
        x = synth.make_tokens(spec, T, seed=seed, device=gen).cpu()
    # the launch configuration the bench times: a non-default stream, where the forward is
    # captured as a CUDA graph on the first call and replayed on the second
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        if layer is None:
            layer = BeamMoE(to_dev(weights), spec.top_k, max_tokens or max(T, 1),
                            segment_len=spec.segment_len)
        xd = x.cuda()
        y = torch.empty((T, spec.d_model), dtype=torch.float32, device="cuda")
        layer.forward(xd, mask_off=mask_off, path=path, out=y, fused=fused)
        y.fill_(float("nan"))
        layer.forward(xd, mask_off=mask_off, path=path, out=y, fused=fused)
    torch.cuda.synchronize()
    gr = layer.routing(T)
    st = layer.stats()
    orr = oracle.route(x, weights["w_router"], weights["w_mask"], spec.top_k,
                       segment_len=spec.segment_len, mask_off=mask_off)
    parity.check_structure(gr, T, spec.top_k, spec.n_experts)
    info = parity.compare_routing(gr, orr, spec.n_experts)
    # statistics: exact for Avg-K when every token is clean, otherwise within the unclean share
    avg_k, l_reg, n0 = oracle.stats(orr)
    assert st["tokens"] == T
    assert st["avg_k"] == gr["keep"].sum() / T
    assert abs(st["avg_k"] - avg_k) <= info["unclean"] * spec.top_k / T + 1e-12
    assert abs(st["l_reg"] - l_reg) <= 1e-5 + info["unclean"] / T
    assert st["n_kept"] == int(gr["keep"].sum())
    np.testing.assert_array_equal(st["counts"], np.diff(gr["offsets"]))
    # y on every compared token: the GPU's decision (checked to be valid within the margin;
    # equal to the oracle's on every clean token) through the oracle's Step 4
    same = same_decision_tokens(gr, orr)
    sel = np.arange(T) if y_tokens is None else np.unique(np.asarray(y_tokens, np.int64))
    gdec, near = parity.gpu_decision_routing(gr, x, weights["w_router"], weights["w_mask"],
                                             spec.top_k, spec.segment_len, mask_off)
    y_gpu = y.cpu().numpy()[sel]
    y_ref = oracle.layer(x, weights, gdec, tokens=sel)
    info.update(parity.compare_y(y_gpu, y_ref, spec.storage))
    # reported: the error against the oracle's own decision on every compared token, and the
    # tokens whose decision differs (all inside the margin)
    differ = sel[~same[sel]]
    if differ.size:
        y_own = oracle.layer(x, weights, orr, tokens=sel)
        own = parity.y_report(y_gpu, y_own, spec.storage)
    else:
        own = parity.y_report(y_gpu, y_ref, spec.storage)
    info.update(y_tokens=int(sel.size), differing_tokens=differ.tolist(),
                near_margin_tokens=int(near.sum()), max_abs_own_decision=own["max_abs"],
                rel_l2_own_decision=own["rel_l2"])
    parity.REPORT.append(dict(case=case or f"{spec.name} T={T}", T=T, clean=info["clean"],
                              unclean=info["unclean"], differing=int(differ.size),
                              y_tokens=int(sel.size), max_abs=info["max_abs"],
                              rel_l2=info["rel_l2"], max_abs_own=own["max_abs"],
                              rel_l2_own=own["rel_l2"]))
    info.update(layer=layer, y=y, routing=gr, oracle=orr, stats=st, weights=weights, x=x)
    return info
