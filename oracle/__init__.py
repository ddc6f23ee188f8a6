"""fp64 CPU oracle of the BEAM masked MoE-layer forward (ctypes wrapper over beam_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the test suite, by `__graft_entry__.smoke()` and by the
bench's CPU-baseline leg, never by the library.  It shares no code with the CUDA library.

`build()` compiles beam_oracle.c with gcc (-O2 -fopenmp) into liboracle.so next to it.
Inputs are float32 or bfloat16 torch CPU tensors (or numpy arrays of the same bits); every
element is widened exactly to double inside the C code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "beam_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle shared library if it is missing or older than its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_route.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_stats.argtypes = [I, P, P, P, P, P]
        lib.oracle_compact.argtypes = [I, I, I, P, P, P, P, P, P]
        lib.oracle_layer.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P, I, P, P]
        lib.oracle_expert.argtypes = [I, I, I, P, P, P, P, I, P]
        lib.oracle_route_backward.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, P,
                                              ctypes.c_double, I, P, P, P, P, P, P, P]
        for f in (lib.oracle_route, lib.oracle_stats, lib.oracle_compact, lib.oracle_layer,
                  lib.oracle_expert, lib.oracle_route_backward, lib.oracle_num_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _host(t):
    """(numpy array, dtype code) for a float32/bf16 tensor; bf16 goes as raw uint16 bits."""
    if t is None:
        return None, -1
    if isinstance(t, np.ndarray):
        if t.dtype == np.float32:
            return np.ascontiguousarray(t), 0
        if t.dtype == np.uint16:
            return np.ascontiguousarray(t), 1
        raise TypeError(f"unsupported numpy dtype {t.dtype}")
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy(), 0
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), 1
    raise TypeError(f"unsupported tensor dtype {t.dtype}")


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


@dataclass
class Routing:
    topk_id: np.ndarray    # int32 [T][K], rank order
    g: np.ndarray          # float64 [T][K] softmax over the K kept logits
    mask_logit: np.ndarray  # float64 [T][K]
    keep: np.ndarray       # uint8 [T][K]
    ghat: np.ndarray       # float64 [T][K] = g * keep
    r_gap: np.ndarray      # float64 [T] r_(K) - r_(K+1)
    rank_gap: np.ndarray   # float64 [T] smallest adjacent gap inside the Top-K
    m_margin: np.ndarray   # float64 [T] smallest |mask logit| over the Top-K
    nkeep: np.ndarray      # int32 [T]
    lreg: np.ndarray       # float64 [T]

    def clean(self, margin: float = 1e-3) -> np.ndarray:
        """Tokens whose Top-K gap and mask-logit margin both exceed `margin`."""
        return (self.r_gap > margin) & (self.m_margin > margin)


def route(x, w_router, w_mask, top_k: int, segment_len: int = 0, mask_off: bool = False) -> Routing:
    """Steps 1-3 of the BEAM pipeline (router Top-K, K-way softmax, sigmoid mask) per token."""
    lib = _load()
    xa, dt = _host(x)
    wr, dt2 = _host(w_router)
    wm, dt3 = _host(w_mask)
    if not (dt == dt2 == dt3):
        raise TypeError("x, w_router and w_mask must share one storage type")
    T, D = xa.shape
    E = wr.shape[1]
    K = int(top_k)
    out = Routing(np.zeros((T, K), np.int32), np.zeros((T, K)), np.zeros((T, K)),
                  np.zeros((T, K), np.uint8), np.zeros((T, K)), np.zeros(T), np.zeros(T),
                  np.zeros(T), np.zeros(T, np.int32), np.zeros(T))
    rc = lib.oracle_route(T, D, E, K, dt, int(segment_len), int(bool(mask_off)), _p(xa), _p(wr),
                          _p(wm), _p(out.topk_id), _p(out.g), _p(out.mask_logit), _p(out.keep),
                          _p(out.ghat), _p(out.r_gap), _p(out.rank_gap), _p(out.m_margin),
                          _p(out.nkeep), _p(out.lreg))
    if rc != 0:
        raise RuntimeError(f"oracle_route failed with code {rc}")
    return out


def route_layers(z, w_router, w_mask, top_k: int, segment_len: int = 0,
                 mask_off: bool = False) -> list:
    """Cross-layer routing: the mask generator of "Stepped MoE: Segment-Level Routing with
    Configurable Inference Complexity" (core method) decides every MoE layer's experts at once
    from the dense prefix's output z, one decision per segment taken at its first token.
    Combined with BEAM, layer l's routing is Steps 1-3 of z with layer l's router and
    mask-router matrices.  w_router, w_mask: [L][D][E].  Returns one Routing per layer."""
    if w_router.shape != w_mask.shape or len(w_router.shape) != 3:
        raise ValueError("w_router and w_mask must both be [L][D][E]")
    return [route(z, w_router[l], w_mask[l], top_k, segment_len=segment_len, mask_off=mask_off)
            for l in range(w_router.shape[0])]


def active_experts(routing: Routing, n_experts: int) -> np.ndarray:
    """bool [E]: the experts some token keeps (the experts whose weights the layer reads)."""
    act = np.zeros(int(n_experts), bool)
    act[routing.topk_id[routing.keep.astype(bool)]] = True
    return act


def stats(routing: Routing):
    """(Avg-K, L_reg, tokens with every Top-K slot masked)."""
    lib = _load()
    a = ctypes.c_double()
    l = ctypes.c_double()
    n = ctypes.c_int32()
    T = routing.nkeep.shape[0]
    lib.oracle_stats(T, _p(routing.nkeep), _p(routing.lreg), ctypes.byref(a), ctypes.byref(l),
                     ctypes.byref(n))
    return a.value, l.value, n.value


def compact(routing: Routing, n_experts: int):
    """(counts[E], offsets[E+1], perm[N_kept], inv[T*K]) of the kept (token, slot) pairs."""
    lib = _load()
    T, K = routing.topk_id.shape
    E = int(n_experts)
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(max(1, T * K), np.int32)
    inv = np.zeros(max(1, T * K), np.int32)
    rc = lib.oracle_compact(T, K, E, _p(np.ascontiguousarray(routing.topk_id)),
                            _p(np.ascontiguousarray(routing.keep)), _p(counts), _p(offsets),
                            _p(perm), _p(inv))
    if rc != 0:
        raise RuntimeError(f"oracle_compact failed with code {rc}")
    n = int(offsets[E])
    return counts, offsets, perm[:n].copy(), inv[:T * K].copy()


def layer(x, weights: dict, routing: Routing, tokens=None) -> np.ndarray:
    """Step 4: y (float64 [len(tokens)][D]) for the selected tokens (all when None)."""
    lib = _load()
    xa, dt = _host(x)
    T, D = xa.shape
    wg, _ = _host(weights["w_gate"])
    wu, _ = _host(weights["w_up"])
    wd, _ = _host(weights["w_down"])
    E, F, _ = wg.shape
    K = routing.topk_id.shape[1]
    wsg, _ = _host(weights.get("ws_gate"))
    wsu, _ = _host(weights.get("ws_up"))
    wsd, _ = _host(weights.get("ws_down"))
    S = 0 if wsg is None else wsg.shape[0]
    Fs = 0 if wsg is None else wsg.shape[1]
    sel = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, np.int32)
    y = np.zeros((sel.shape[0], D))
    rc = lib.oracle_layer(T, D, E, K, F, S, Fs, dt, _p(xa), _p(wg), _p(wu), _p(wd), _p(wsg),
                          _p(wsu), _p(wsd), _p(np.ascontiguousarray(routing.topk_id)),
                          _p(np.ascontiguousarray(routing.ghat)),
                          _p(np.ascontiguousarray(routing.keep)), int(sel.shape[0]), _p(sel), _p(y))
    if rc != 0:
        raise RuntimeError(f"oracle_layer failed with code {rc}")
    return y


def expert(x_vec, wg, wu, wd, e: int = 0) -> np.ndarray:
    """One SwiGLU expert (index e of stacked [E][F][D]/[E][D][F] weights) on one float64 vector."""
    lib = _load()
    wga, dt = _host(wg)
    wua, _ = _host(wu)
    wda, _ = _host(wd)
    _, F, D = wga.shape
    xv = np.ascontiguousarray(x_vec, np.float64)
    out = np.zeros(D)
    rc = lib.oracle_expert(D, F, dt, _p(xv), _p(wga), _p(wua), _p(wda), int(e), _p(out))
    if rc != 0:
        raise RuntimeError(f"oracle_expert failed with code {rc}")
    return out


@dataclass
class RouteGrad:
    s: np.ndarray      # float64 [T][K]: <dy_t, E_i(x_t)> of every Top-K slot (= dL/dg_hat)
    d_r: np.ndarray    # float64 [T][K]: dL/d(router logit) of slot k at routed rows, else 0
    d_l: np.ndarray    # float64 [T][K]: dL/d(mask logit) of slot k at routed rows, else 0
    dw_r: np.ndarray   # float64 [D][E] (None when only some rows were asked for)
    dw_m: np.ndarray   # float64 [D][E] (None when only some rows were asked for)
    dx: np.ndarray     # float64 [T][D]: the routing's share of dL/dx (0 off the routed rows)


def route_backward(x, weights: dict, routing: Routing, dy, reg_scale: float = 0.0,
                   segment_len: int = 0, rows=None) -> RouteGrad:
    """Training-side gradient of the router and the mask router under the straight-through
    estimator, plus the L_reg term (BEAM article on aitrends.kr, training paragraph; ai-feeds
    summary, Method, binarisation and straight-through estimator).  dy: float64 [T][D] upstream
    gradient of the output; reg_scale: dL/dL_reg with L_reg the mean over tokens.  The experts
    of every Top-K slot are evaluated (training runs them all; the mask only scales gates).
    `rows` (token indices of routed rows) restricts the work to those rows and skips dW."""
    lib = _load()
    xa, dt = _host(x)
    T, D = xa.shape
    wr, _ = _host(weights["w_router"])
    wm, _ = _host(weights["w_mask"])
    wg, _ = _host(weights["w_gate"])
    wu, _ = _host(weights["w_up"])
    wd, _ = _host(weights["w_down"])
    E, F, _ = wg.shape
    K = routing.topk_id.shape[1]
    dya = np.ascontiguousarray(dy, np.float64)
    if dya.shape != (T, D):
        raise ValueError("dy must be [T][D]")
    sel = None if rows is None else np.ascontiguousarray(rows, np.int32)
    out = RouteGrad(np.zeros((T, K)), np.zeros((T, K)), np.zeros((T, K)),
                    np.zeros((D, E)), np.zeros((D, E)), np.zeros((T, D)))
    rc = lib.oracle_route_backward(
        T, D, E, K, F, dt, int(segment_len), _p(xa), _p(wr), _p(wm), _p(wg), _p(wu), _p(wd),
        _p(np.ascontiguousarray(routing.topk_id)), _p(np.ascontiguousarray(routing.g)),
        _p(np.ascontiguousarray(routing.mask_logit)), _p(dya), float(reg_scale),
        -1 if sel is None else int(sel.shape[0]), _p(sel), _p(out.s), _p(out.d_r), _p(out.d_l),
        _p(out.dw_r), _p(out.dw_m), _p(out.dx))
    if rc != 0:
        raise RuntimeError(f"oracle_route_backward failed with code {rc}")
    if sel is not None:
        out.dw_r = out.dw_m = None
    return out
