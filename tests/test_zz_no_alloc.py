"""beam_moe_route_noalloc: routing into caller-provided buffers with no device allocation.

Some callers cannot allocate device memory at the point where they route, for instance a
serving engine that has reserved all free device memory for its own pools, so that a later
cudaMalloc would fail.  This entry point keeps its scratch in a fixed array compiled into the
library.  These tests call it through the C ABI and compare it with what beam_moe_forward
produces for the same tokens, twice in a row on different tokens, so the second call runs on
scratch the first one filled.  The two may compute the logits with a different fp32
summation order (large bf16 batches use the tensor cores in the forward), so the comparison
uses the routing tolerance of the parity tests: Top-K ids and keep bits equal wherever the
decision margin exceeds 1e-3, gates and mask logits within 1e-4.  Each call is also compared
with the fp64 oracle's routing: ids (in rank order where the ranks are 1e-3 apart) and keep
bits exact on every clean token, gates and mask logits within 1e-4.

This file is collected last so that a run stopping at the first failure has run every other
test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _route_noalloc(lib, layer, x, flags=0):
    T, K = x.shape[0], layer.top_k
    out = dict(topk_id=torch.full((T, K), -7, dtype=torch.int32, device="cuda"),
               gate=torch.full((T, K), -7.0, device="cuda"),
               mask_logit=torch.full((T, K), -7.0, device="cuda"),
               keep=torch.full((T, K), 7, dtype=torch.uint8, device="cuda"),
               ghat=torch.full((T, K), -7.0, device="cuda"))
    p = {k: ctypes.c_void_p(v.data_ptr()) for k, v in out.items()}
    st = lib.beam_moe_route_noalloc(layer._h, ctypes.c_void_p(x.data_ptr()), T, p["topk_id"],
                                    p["gate"], p["mask_logit"], p["keep"], p["ghat"], flags,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, {k: v.cpu().numpy() for k, v in out.items()}


def _compare_oracle(got, orr, msg, margin=1e-3):
    clean = orr.clean(margin)
    assert clean.mean() >= 0.9, msg
    for t in np.nonzero(clean)[0]:
        assert set(got["topk_id"][t].tolist()) == set(orr.topk_id[t].tolist()), f"{msg}: token {t}"
        if orr.rank_gap[t] > margin:
            np.testing.assert_array_equal(got["topk_id"][t], orr.topk_id[t], err_msg=f"{msg}: token {t}")
            np.testing.assert_array_equal(got["keep"][t], orr.keep[t], err_msg=f"{msg}: token {t}")
            np.testing.assert_allclose(got["gate"][t], orr.g[t], atol=1e-4, err_msg=f"{msg}: token {t}")
            np.testing.assert_allclose(got["mask_logit"][t], orr.mask_logit[t], atol=1e-4,
                                       err_msg=f"{msg}: token {t}")


def _compare(got, ref, msg, margin=1e-3):
    same_ids = (got["topk_id"] == ref["topk_id"]).all(axis=1)
    # a differing Top-K row is only acceptable at a near-tie of two gates
    for t in np.nonzero(~same_ids)[0]:
        g = np.sort(ref["gate"][t])
        assert np.min(np.diff(g)) < margin, f"{msg}: Top-K differs at token {t} without a tie"
    assert same_ids.mean() >= 0.99, msg
    sel = same_ids[:, None] & (np.abs(ref["mask_logit"]) > margin)
    np.testing.assert_array_equal(got["keep"][sel], ref["keep"][sel], err_msg=msg)
    np.testing.assert_allclose(got["gate"][same_ids], ref["gate"][same_ids], atol=1e-4, err_msg=msg)
    np.testing.assert_allclose(got["mask_logit"][same_ids], ref["mask_logit"][same_ids], atol=1e-4,
                               err_msg=msg)
    np.testing.assert_array_equal(got["ghat"], got["gate"] * got["keep"], err_msg=msg)


@pytest.mark.parametrize("spec,T", [
    (synth.SPECS["tiny"], 64),
    (synth.LayerSpec("small", 512, 16, 4, 256, n_shared=1, d_ff_shared=128), 300),
    (synth.LayerSpec("seg", 512, 60, 4, 256, segment_len=16), 16 * 9 + 5),
], ids=["tiny_fp32", "bf16", "bf16_segment"])
def test_route_noalloc_matches_forward_twice(spec, T):
    from dynamic_expert_routing_b200 import BeamMoE, _lib
    lib = _lib.load()
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE({k: v.cuda() for k, v in w.items() if isinstance(v, torch.Tensor)},
                    spec.top_k, max_tokens=T, segment_len=spec.segment_len)
    import oracle
    for call, seed in enumerate((11, 12)):
        xc = synth.make_tokens(spec, T, seed=seed)
        x = xc.cuda()
        layer.forward(x)
        ref = layer.routing(T)
        n0 = layer.launch_count()
        st, got = _route_noalloc(lib, layer, x)
        assert st == _lib.BEAM_OK, lib.beam_moe_last_error()
        assert layer.launch_count() == n0          # the handle's state is left alone
        _compare(got, ref, f"call {call}")
        orr = oracle.route(xc, w["w_router"], w["w_mask"], spec.top_k,
                           segment_len=spec.segment_len)
        _compare_oracle(got, orr, f"call {call} vs oracle")
    # the mask-off flag keeps every Top-K slot
    st, got = _route_noalloc(lib, layer, x, flags=_lib.BEAM_MASK_OFF)
    assert st == _lib.BEAM_OK and got["keep"].all()
    layer.close()


def test_route_noalloc_rejects_sizes_beyond_the_static_buffer():
    from dynamic_expert_routing_b200 import BeamMoE, _lib
    lib = _lib.load()
    spec = synth.LayerSpec("wide", 256, 256, 8, 128)
    w = synth.make_layer(spec, keep_rate=0.5)
    T = 1200   # 1200 * 512 * 4 bytes of logits alone exceed the 2 MiB array
    layer = BeamMoE({k: v.cuda() for k, v in w.items() if isinstance(v, torch.Tensor)},
                    spec.top_k, max_tokens=T)
    x = synth.make_tokens(spec, T).cuda()
    st, _ = _route_noalloc(lib, layer, x)
    assert st == _lib.BEAM_ERR_INVALID_ARG
    assert b"static buffer" in lib.beam_moe_last_error()
    layer.close()
