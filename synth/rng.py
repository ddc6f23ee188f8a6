"""Counter-based random numbers shared by the oracle tests, the GPU tests and the bench.

Every synthetic tensor is a pure function of (seed, tensor id, element index), so the same
bits can be produced on the host or on a CUDA device, in any chunking.  The construction is
the published SplitMix64 generator (Steele, Lea and Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014), used in counter mode: element i of stream `key` is the SplitMix64
finaliser applied to key + (i + 1) * 0x9E3779B97F4A7C15 (mod 2^64).  Normals come from the
Box-Muller transform (cosine branch only) of two such uniforms, evaluated in float64.

This module holds no arithmetic of the MoE layer itself.
"""
from __future__ import annotations

import math

import torch

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15
_MIX1 = 0xBF58476D1CE4E5B9
_MIX2 = 0x94D049BB133111EB


def _as_i64(v: int) -> int:
    """Two's-complement reinterpretation of an unsigned 64-bit value as int64."""
    v &= _M64
    return v - (1 << 64) if v >= (1 << 63) else v


def splitmix64_scalar(state: int) -> int:
    """Finaliser of SplitMix64 on one unsigned 64-bit integer (pure Python, exact)."""
    z = state & _M64
    z = ((z ^ (z >> 30)) * _MIX1) & _M64
    z = ((z ^ (z >> 27)) * _MIX2) & _M64
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    """Key of the stream that tensor `tensor_id` of run `seed` draws from."""
    return splitmix64_scalar(splitmix64_scalar(seed + _GAMMA) ^ (tensor_id & _M64))


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor holding unsigned 64-bit values."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def raw_u64(key: int, idx: torch.Tensor) -> torch.Tensor:
    """SplitMix64 outputs (as int64 bit patterns) for counters `idx` (int64) of stream `key`."""
    z = idx * _as_i64(_GAMMA) + _as_i64(key + _GAMMA)
    z = (z ^ _srl(z, 30)) * _as_i64(_MIX1)
    z = (z ^ _srl(z, 27)) * _as_i64(_MIX2)
    return z ^ _srl(z, 31)


def raw_u64_scalar(key: int, i: int) -> int:
    """Pure-Python twin of raw_u64 for one counter (used to check the tensor version)."""
    return splitmix64_scalar(key + (i + 1) * _GAMMA)


def uniform_open(key: int, idx: torch.Tensor) -> torch.Tensor:
    """Float64 uniforms in the open interval (0, 1): ((u >> 11) + 0.5) / 2^53."""
    top = _srl(raw_u64(key, idx), 11)
    return (top.to(torch.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(key: int, idx: torch.Tensor) -> torch.Tensor:
    """Float64 standard normals; element i uses uniforms at counters 2i and 2i+1."""
    u1 = uniform_open(key, 2 * idx)
    u2 = uniform_open(key, 2 * idx + 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos((2.0 * math.pi) * u2)


_CHUNK = 1 << 24


def fill(shape, key: int, kind: str, scale: float = 1.0, device="cpu",
         dtype=torch.float64) -> torch.Tensor:
    """A tensor of `shape` whose flat element i is draw(key, i) * scale.

    kind is "normal" or "uniform".  Values are computed in float64 and rounded once to
    `dtype` (float32 or float64) with round-to-nearest-even; bf16 targets go through
    `to_storage`.  Large tensors are produced in chunks so the int64 temporaries stay small.
    """
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(n, dtype=dtype, device=device)
    draw = normal if kind == "normal" else uniform_open
    for start in range(0, n, _CHUNK):
        stop = min(n, start + _CHUNK)
        idx = torch.arange(start, stop, dtype=torch.int64, device=device)
        v = draw(key, idx)
        if scale != 1.0:
            v = v * scale
        out[start:stop] = v.to(dtype)
    return out.view(*shape)


def to_storage(t64: torch.Tensor, storage: str) -> torch.Tensor:
    """Round a float64 tensor to the layer's storage type.

    "fp32": one RNE rounding to float32.  "bf16": RNE to float32, then RNE to bfloat16
    (two roundings, both exact-rule and identical on every platform).
    """
    t32 = t64.to(torch.float32)
    if storage == "fp32":
        return t32
    if storage == "bf16":
        return t32.to(torch.bfloat16)
    raise ValueError(f"unknown storage type {storage!r}")
