"""The seeded generators: exact SplitMix64 counter streams, chunk independence, recipe shape."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import rng


def test_splitmix64_published_first_outputs():
    # SplitMix64 seeded with 0: the first outputs of the reference generator
    # (state advanced by the golden gamma before mixing).
    assert rng.splitmix64_scalar(0x9E3779B97F4A7C15) == 0xE220A8397B1DCDAF
    assert rng.splitmix64_scalar(2 * 0x9E3779B97F4A7C15 & ((1 << 64) - 1)) == 0x6E789E6AA1B965F4


def test_tensor_stream_matches_scalar_twin():
    key = rng.stream_key(0, 3)
    idx = torch.tensor([0, 1, 2, 1000, 123456789, (1 << 40) + 7], dtype=torch.int64)
    got = rng.raw_u64(key, idx)
    for i, v in zip(idx.tolist(), got.tolist()):
        assert (v & ((1 << 64) - 1)) == rng.raw_u64_scalar(key, i)


def test_fill_is_chunk_independent():
    key = rng.stream_key(1, 4)
    a = rng.fill((3, 1000), key, "normal")
    idx = torch.arange(3000, dtype=torch.int64)
    b = rng.normal(key, idx).view(3, 1000)
    assert torch.equal(a, b)
    u = rng.fill((5000,), key, "uniform")
    assert 0.0 < float(u.min()) and float(u.max()) < 1.0


def test_normal_moments():
    v = rng.fill((200000,), rng.stream_key(0, 99), "normal")
    assert abs(float(v.mean())) < 0.01
    assert abs(float(v.std()) - 1.0) < 0.01


def test_tokens_prefix_stable_and_constant_channel():
    spec = synth.SPECS["dsv2lite"].with_(d_model=64)
    a = synth.make_tokens(spec, 5)
    b = synth.make_tokens(spec, 9)
    assert torch.equal(a, b[:5])
    assert (a[:, 0].float() == 1.0).all()


def test_zipf_prior_row():
    spec = synth.SPECS["qwenmoe"].with_(d_model=32)
    wr, _ = synth.make_router(spec)
    p = torch.tensor([(e + 1) ** -1.1 for e in range(60)], dtype=torch.float64)
    want = torch.log(p / p.sum()).float().bfloat16()
    assert torch.equal(wr[0], want)


@pytest.mark.parametrize("name,keep", [("tiny", 0.5), ("mixtral", 0.25), ("dsv2lite", 0.45),
                                       ("dsv2lite", 0.07)])
def test_mask_bias_gives_keep_rate(name, keep):
    """The closed-form mask bias lands near the target keep rate on generated data
    (checked with the oracle's routing on a reduced-width copy of the layer)."""
    spec = synth.SPECS[name].with_(d_model=256, d_ff=128, n_shared=0, storage="fp32")
    c = synth.mask_bias_for_keep_rate(spec, keep)
    T = 2048
    x = synth.make_tokens(spec, T, seed=21)
    wr, wm = synth.make_router(spec, seed=21, mask_bias=c)
    r = oracle.route(x, wr, wm, spec.top_k)
    rate = r.keep.mean()
    sd = math.sqrt(keep * (1 - keep) / (T * spec.top_k))
    assert abs(rate - keep) < 5 * sd + 0.01
