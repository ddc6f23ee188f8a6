"""Seeded synthetic MoE layers and token batches shaped like the models the BEAM pages name.

The pages print no layer dimensions, so the shapes below are the stated synthetic stand-ins
for a Mixtral-like, a DeepSeekV2-Lite-like, a Qwen-MoE-like and a fine-grained (212 experts,
Stepped-MoE shape) layer, plus a tiny fp32 layer small enough for a CPU oracle.  No trained
weights or datasets are involved: every tensor is a pure function of (seed, tensor id).

Recipe (all draws from `synth.rng`, float64, rounded once to the storage type):
  x ~ N(0,1) with x[:,0] = 1 (a constant input channel that carries biases through row 0 of
  the router matrices); W_r, W_m ~ N(0, 1/D); W_m[0,:] = c (mask bias); W_g, W_u ~ N(0, 1/D);
  W_d ~ N(0, 1/F).  The DeepSeek-like layer divides x[t,1:] by a per-token temperature
  tau_t ~ U(0.5, 2); the Qwen-like layer adds a Zipf(1.1) log-prior to the router logits via
  W_r[0,e] = log p_e, p_e proportional to (e+1)^-1.1.

The mask bias c is set from the input distribution alone (no routing is evaluated here): the
mask logit of an expert is c + z with z = sum_{d>=1} x_d W_m[d,e], which is close to
N(0, (D-1)/D) (divided by tau_t where a temperature is used) and independent of which experts
the router picks, so P(keep) = Phi(c / sigma_z), or its average over tau.

This module holds no arithmetic of the MoE layer itself.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from statistics import NormalDist

import torch

from . import rng

# Stream ids: one per tensor, fixed forever so stored fixtures stay reproducible.
ID_X, ID_WR, ID_WM, ID_WG, ID_WU, ID_WD, ID_WSG, ID_WSU, ID_WSD, ID_TAU = range(10)


@dataclass(frozen=True)
class LayerSpec:
    name: str
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    n_shared: int = 0
    d_ff_shared: int = 0
    storage: str = "bf16"          # "fp32" or "bf16"
    temperature: bool = False      # per-token temperature tau ~ U(0.5, 2)
    zipf: float = 0.0              # Zipf exponent of the router log-prior (0 = none)
    segment_len: int = 0           # 0/1 = per-token routing; S > 1 = segment routing

    def with_(self, **kw) -> "LayerSpec":
        return replace(self, **kw)


SPECS = {
    "tiny": LayerSpec("tiny", 256, 8, 2, 512, storage="fp32"),
    "mixtral": LayerSpec("mixtral", 4096, 8, 2, 14336),
    "dsv2lite": LayerSpec("dsv2lite", 2048, 64, 6, 1408, n_shared=2, d_ff_shared=1408,
                          temperature=True),
    "qwenmoe": LayerSpec("qwenmoe", 2048, 60, 4, 1408, n_shared=4, d_ff_shared=1408, zipf=1.1),
    "fine": LayerSpec("fine", 1536, 212, 16, 256),
    "fine_seg16": LayerSpec("fine_seg16", 1536, 212, 16, 256, segment_len=16),
}


def _dtype_for(storage: str):
    return torch.float32 if storage == "fp32" else torch.bfloat16


def _tau_grid(n: int = 4000):
    """Midpoints of U(0.5, 2) for averaging over the temperature distribution."""
    return [0.5 + 1.5 * (i + 0.5) / n for i in range(n)]


def mask_bias_for_keep_rate(spec: LayerSpec, keep_rate: float) -> float:
    """Mask bias c giving expected keep rate `keep_rate` among Top-K slots.

    keep_rate must lie in (0, 1); a keep rate of 1 is the plain Top-K layer and is run with the
    mask switched off instead.
    """
    if not 0.0 < keep_rate < 1.0:
        raise ValueError("keep_rate must be in (0, 1); use the mask-off flag for 1.0")
    sigma = math.sqrt((spec.d_model - 1) / spec.d_model)
    nd = NormalDist()
    if not spec.temperature:
        return sigma * nd.inv_cdf(keep_rate)
    taus = _tau_grid()

    def rate(c):
        return sum(nd.cdf(c * t / sigma) for t in taus) / len(taus)

    lo, hi = -20.0, 20.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if rate(mid) < keep_rate:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _fill_storage(shape, key, scale, storage, device):
    """N(0, scale^2) tensor rounded to the storage type chunk by chunk (float64 transient)."""
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=_dtype_for(storage), device=device)
    chunk = 1 << 24
    for start in range(0, n, chunk):
        stop = min(n, start + chunk)
        idx = torch.arange(start, stop, dtype=torch.int64, device=device)
        v = rng.normal(key, idx) * scale
        out[start:stop] = rng.to_storage(v, storage)
    return out.view(*shape)


def make_tokens(spec: LayerSpec, T: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """Token batch x [T][D] in the storage type.  Row t does not depend on T."""
    D = spec.d_model
    x = rng.fill((T, D), rng.stream_key(seed, ID_X), "normal", device=device)
    x[:, 0] = 1.0
    if spec.temperature:
        tau = 0.5 + 1.5 * rng.fill((T,), rng.stream_key(seed, ID_TAU), "uniform", device=device)
        x[:, 1:] = x[:, 1:] / tau[:, None]
    return rng.to_storage(x, spec.storage).contiguous()


def make_router(spec: LayerSpec, seed: int = 0, mask_bias: float | None = 0.0,
                device="cpu"):
    """Router matrices (W_r, W_m), each [D][E] in the storage type.

    mask_bias=None gives W_m = 0 (the mask router's zero initialisation); otherwise W_m is
    drawn and its row 0 set to mask_bias.
    """
    D, E = spec.d_model, spec.n_experts
    s = 1.0 / math.sqrt(D)
    wr = rng.fill((D, E), rng.stream_key(seed, ID_WR), "normal", scale=s, device=device)
    if spec.zipf:
        p = torch.tensor([(e + 1) ** (-spec.zipf) for e in range(E)], dtype=torch.float64)
        p = p / p.sum()
        wr[0, :] = torch.log(p).to(device)
    if mask_bias is None:
        wm = torch.zeros((D, E), dtype=torch.float64, device=device)
    else:
        wm = rng.fill((D, E), rng.stream_key(seed, ID_WM), "normal", scale=s, device=device)
        wm[0, :] = mask_bias
    return rng.to_storage(wr, spec.storage).contiguous(), rng.to_storage(wm, spec.storage).contiguous()


def make_experts(spec: LayerSpec, seed: int = 0, device="cpu"):
    """Routed and shared SwiGLU expert weights in the storage type.

    Returns w_gate [E][F][D], w_up [E][F][D], w_down [E][D][F] and, when the layer has shared
    experts, ws_gate [S][Fs][D], ws_up [S][Fs][D], ws_down [S][D][Fs] (else None for each).
    """
    D, E, F = spec.d_model, spec.n_experts, spec.d_ff
    sd, sf = 1.0 / math.sqrt(D), 1.0 / math.sqrt(F)
    st = spec.storage
    wg = _fill_storage((E, F, D), rng.stream_key(seed, ID_WG), sd, st, device)
    wu = _fill_storage((E, F, D), rng.stream_key(seed, ID_WU), sd, st, device)
    wd = _fill_storage((E, D, F), rng.stream_key(seed, ID_WD), sf, st, device)
    if spec.n_shared:
        S, Fs = spec.n_shared, spec.d_ff_shared
        sfs = 1.0 / math.sqrt(Fs)
        wsg = _fill_storage((S, Fs, D), rng.stream_key(seed, ID_WSG), sd, st, device)
        wsu = _fill_storage((S, Fs, D), rng.stream_key(seed, ID_WSU), sd, st, device)
        wsd = _fill_storage((S, D, Fs), rng.stream_key(seed, ID_WSD), sfs, st, device)
    else:
        wsg = wsu = wsd = None
    return wg, wu, wd, wsg, wsu, wsd


def make_layer(spec: LayerSpec, seed: int = 0, keep_rate: float | None = 0.5,
               mask_bias: float | None = None, zero_mask: bool = False, device="cpu") -> dict:
    """All weights of one layer as a dict of tensors (storage type, on `device`).

    The mask bias is `mask_bias` if given, else derived from `keep_rate`; `zero_mask=True`
    gives W_m = 0.  A keep_rate of None or 1.0 draws W_m with bias 0 (run it with the mask off).
    """
    if zero_mask:
        c = None
    elif mask_bias is not None:
        c = float(mask_bias)
    elif keep_rate is None or keep_rate >= 1.0:
        c = 0.0
    else:
        c = mask_bias_for_keep_rate(spec, keep_rate)
    wr, wm = make_router(spec, seed, c, device)
    wg, wu, wd, wsg, wsu, wsd = make_experts(spec, seed, device)
    return dict(w_router=wr, w_mask=wm, w_gate=wg, w_up=wu, w_down=wd,
                ws_gate=wsg, ws_up=wsu, ws_down=wsd, mask_bias=c)


def make_generator(spec: LayerSpec, n_layers: int, seed: int = 0,
                   keep_rate: float | None = 0.5, mask_bias: float | None = None):
    """Weights of a cross-layer mask generator: (W_r, W_m), each [L][D][E] in the storage type.

    Layer l's pair is `make_router` of the same spec with seed 1000 * (seed + 1) + l, so every
    layer draws its own streams; the mask bias follows `make_layer`'s rule.
    """
    if mask_bias is not None:
        c = float(mask_bias)
    elif keep_rate is None or keep_rate >= 1.0:
        c = 0.0
    else:
        c = mask_bias_for_keep_rate(spec, keep_rate)
    wr, wm = zip(*[make_router(spec, 1000 * (seed + 1) + l, c) for l in range(n_layers)])
    return torch.stack(wr).contiguous(), torch.stack(wm).contiguous()
