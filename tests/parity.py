"""Comparison of the CUDA library's outputs with the fp64 oracle (shared by the GPU tests and
the bench's parity leg, which compares the timed forward's output with the oracle's on the
CPU-baseline token sample).

Acceptance (stated for the BEAM layer; the decision margin 1e-3 is far above the fp32-vs-fp64
logit difference, so clean tokens have one correct answer):
  * a token is clean when its Top-K gap r_(K) - r_(K+1) and every Top-K |mask logit| exceed
    1e-3 (oracle values); unclean tokens are counted and reported;
  * on clean tokens: Top-K ids as a set, in rank order where adjacent Top-K gaps exceed 1e-3,
    keep per expert, per-expert counts, and the (token, expert) sequence of perm are bit-exact;
  * structural checks on every token: perm is the kept pairs sorted by (expert, token), inv
    inverts it, offsets are the prefix sums of the counts;
  * y: bf16 layers max |err| <= 2e-2 and relative L2 <= 5e-3; fp32 layers relative L2 <= 1e-5,
    over every compared token.  A token whose GPU decision differs from the oracle's (possible
    only inside the margin) is checked under the GPU's decision: that decision must be a valid
    one within the margin (`gpu_decision_routing`), and y must match the oracle's Step 4 for it.
    The error against the oracle's own decisions over all tokens is reported alongside.
"""
from __future__ import annotations

import numpy as np

MARGIN = 1e-3
# one dict per GPU parity case of the test run (printed by tests/conftest.py at the end)
REPORT: list = []
TOL_BF16_ABS = 2e-2
TOL_BF16_REL = 5e-3
TOL_F32_REL = 1e-5


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / den) if den > 0 else float(np.linalg.norm(a - b))


def check_structure(gr: dict, T: int, K: int, E: int) -> None:
    """Invariants of the GPU's own routing output (any token, clean or not)."""
    ids, keep, perm, inv, off = gr["topk_id"], gr["keep"], gr["perm"], gr["inv"], gr["offsets"]
    assert ids.shape == (T, K)
    assert ((ids >= 0) & (ids < E)).all()
    for t in range(T):
        assert len(set(ids[t].tolist())) == K, f"token {t} repeats an expert"
    kept = [(int(ids[t, k]), t, k) for t in range(T) for k in range(K) if keep[t, k]]
    kept.sort()
    assert [t * K + k for (_, t, k) in kept] == perm.tolist(), "perm is not sorted by (expert, token)"
    counts = np.bincount(np.array([e for (e, _, _) in kept], np.int64), minlength=E) if kept else np.zeros(E, np.int64)
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    flat_inv = inv.reshape(-1)
    for pos, i in enumerate(perm.tolist()):
        assert flat_inv[i] == pos
    assert (flat_inv[keep.reshape(-1) == 0] == -1).all()


def compare_routing(gr: dict, orr, E: int, margin: float = MARGIN) -> dict:
    """Bit-exact comparison on clean tokens; returns counts of clean / unclean tokens."""
    T, K = orr.topk_id.shape
    clean = orr.clean(margin)
    gid, gkeep = gr["topk_id"], gr["keep"]
    for t in np.nonzero(clean)[0]:
        assert set(gid[t].tolist()) == set(orr.topk_id[t].tolist()), f"Top-K set differs at token {t}"
        if orr.rank_gap[t] > margin:
            np.testing.assert_array_equal(gid[t], orr.topk_id[t], err_msg=f"rank order at token {t}")
        gk = {int(e): int(k) for e, k in zip(gid[t], gkeep[t])}
        ok = {int(e): int(k) for e, k in zip(orr.topk_id[t], orr.keep[t])}
        assert gk == ok, f"keep differs at token {t}"
    # per-expert counts and perm restricted to clean tokens
    def seq(ids, keep, perm):
        out = []
        for i in perm.tolist():
            t, k = divmod(i, K)
            if clean[t]:
                out.append((int(ids[t, k]), t))
        return out

    from oracle import compact
    _, _, operm, _ = compact(orr, E)
    assert seq(gid, gkeep, gr["perm"]) == seq(orr.topk_id, orr.keep, operm), "perm differs on clean tokens"
    return dict(clean=int(clean.sum()), unclean=int((~clean).sum()))


def compare_y(y_gpu, y_ref, storage: str) -> dict:
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    err = float(np.abs(y_gpu - y_ref).max()) if y_ref.size else 0.0
    rl = rel_l2(y_gpu, y_ref) if y_ref.size else 0.0
    if storage == "bf16":
        assert err <= TOL_BF16_ABS, f"max abs error {err:.3e} > {TOL_BF16_ABS}"
        assert rl <= TOL_BF16_REL, f"relative L2 error {rl:.3e} > {TOL_BF16_REL}"
    else:
        assert rl <= TOL_F32_REL, f"relative L2 error {rl:.3e} > {TOL_F32_REL}"
    return dict(max_abs=err, rel_l2=rl)


def fp64_logits(x, w_router, w_mask, segment_len: int = 0):
    """Router and mask logits of the routed rows (segment leaders when segment_len > 1),
    float64 [T][E] each, for the validity check of a decision inside the margin."""
    import torch
    xs = x.double()
    S = segment_len if segment_len > 1 else 1
    lead = torch.arange(0, xs.shape[0], S)
    xl = xs[lead]
    return (xl @ w_router.double()).numpy(), (xl @ w_mask.double()).numpy(), S


def gpu_decision_routing(gr: dict, x, w_router, w_mask, K: int, segment_len: int = 0,
                         mask_off: bool = False, margin: float = MARGIN):
    """The GPU's decision on every token as an oracle.Routing (ids and keep from the GPU, gates
    the fp64 softmax over the chosen K logits, g_hat = g * keep), after checking that it is a
    valid decision within the margin: the chosen set's smallest logit is at least the largest
    unchosen logit minus the margin, and every keep bit agrees with mask logit >= 0 unless that
    logit is within the margin of 0.  Returns (routing, tokens whose decision needed the margin)."""
    import oracle
    r, l, S = fp64_logits(x, w_router, w_mask, segment_len)
    T = gr["topk_id"].shape[0]
    ids = gr["topk_id"].astype(np.int64)
    keep = gr["keep"].astype(np.uint8)
    g = np.zeros((T, K))
    ml = np.zeros((T, K))
    near = np.zeros(T, bool)
    for t in range(T):
        i = t // S
        sel = ids[t]
        rs = r[i, sel]
        others = np.delete(r[i], sel)
        lo = rs.min()
        hi = others.max() if others.size else -np.inf
        assert lo >= hi - margin, f"token {t}: GPU Top-K set is not a Top-K within the margin"
        if lo < hi + margin:
            near[t] = True
        e = np.exp(rs - rs.max())
        g[t] = e / e.sum()
        ml[t] = l[i, sel]
        want = np.ones(K, np.uint8) if mask_off else (ml[t] >= 0).astype(np.uint8)
        bad = keep[t] != want
        if bad.any():
            assert (np.abs(ml[t][bad]) <= margin).all(), f"token {t}: keep differs outside the margin"
            near[t] = True
    ghat = g * keep
    zeros = np.zeros(T)
    out = oracle.Routing(ids.astype(np.int32), g, ml, keep, ghat, zeros, zeros, zeros,
                         keep.sum(axis=1).astype(np.int32), zeros)
    return out, near


def y_report(y_gpu, y_ref, storage: str) -> dict:
    """max |err| and relative L2 of y against a reference, and whether they meet the bars."""
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    err = float(np.abs(y_gpu - y_ref).max()) if y_ref.size else 0.0
    rl = rel_l2(y_gpu, y_ref) if y_ref.size else 0.0
    ok = (err <= TOL_BF16_ABS and rl <= TOL_BF16_REL) if storage == "bf16" else rl <= TOL_F32_REL
    return dict(max_abs=err, rel_l2=rl, ok=bool(ok))
