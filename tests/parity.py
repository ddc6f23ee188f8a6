"""Comparison of the CUDA library's outputs with the fp64 oracle (shared by the GPU tests,
the smoke check and the bench's parity leg).

Acceptance (stated for the BEAM layer; the decision margin 1e-3 is far above the fp32-vs-fp64
logit difference, so clean tokens have one correct answer):
  * a token is clean when its Top-K gap r_(K) - r_(K+1) and every Top-K |mask logit| exceed
    1e-3 (oracle values); unclean tokens are counted and reported;
  * on clean tokens: Top-K ids as a set, in rank order where adjacent Top-K gaps exceed 1e-3,
    keep per expert, per-expert counts, and the (token, expert) sequence of perm are bit-exact;
  * structural checks on every token: perm is the kept pairs sorted by (expert, token), inv
    inverts it, offsets are the prefix sums of the counts;
  * y: bf16 layers max |err| <= 2e-2 and relative L2 <= 5e-3; fp32 layers relative L2 <= 1e-5.
"""
from __future__ import annotations

import numpy as np

MARGIN = 1e-3
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
