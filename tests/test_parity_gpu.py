"""CUDA library vs the fp64 oracle, element by element on the same seeded inputs.

Shapes span several tiles and ragged tails of every kernel (token chunks of 32, row blocks of
16/128, 8-token passes), the edge cases of the method (W_m = 0, every slot masked, K = E,
segment routing with a partial last segment, T = 0, T = max_tokens) and the layer shapes the
BEAM pages name (Mixtral-like, DeepSeekV2-Lite-like, Qwen-MoE-like, fine-grained 212 experts).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity
from tests.gpu_util import run_case, to_dev

pytestmark = pytest.mark.gpu


def _small(**kw):
    return synth.LayerSpec("small", 512, 16, 4, 256, storage="bf16").with_(**kw)


# ------------------------------------------------------------------ the tiny fp32 layer
def test_tiny_fp32_parity():
    spec = synth.SPECS["tiny"]
    info = run_case(spec, 64)
    assert info["rel_l2"] <= parity.TOL_F32_REL
    assert 0 < info["stats"]["n_kept"] < 64 * 2


def test_tiny_zero_mask_router_is_plain_topk():
    spec = synth.SPECS["tiny"]
    info = run_case(spec, 64, zero_mask=True)
    assert info["routing"]["keep"].all()
    assert info["stats"]["l_reg"] == 0.5
    assert info["stats"]["avg_k"] == 2.0
    # the mask-off flag on the masked layer reproduces the W_m = 0 layer bit for bit
    w = synth.make_layer(spec, keep_rate=0.5)
    w0 = dict(w, w_mask=torch.zeros_like(w["w_mask"]))
    a = run_case(spec, 64, weights=w, mask_off=True)
    b = run_case(spec, 64, weights=w0)
    assert torch.equal(a["y"], b["y"])
    np.testing.assert_array_equal(a["routing"]["perm"], b["routing"]["perm"])


# ------------------------------------------------------------------ bf16, ragged shapes
@pytest.mark.parametrize("T", [1, 5, 8, 33, 100])
def test_small_bf16_stream_path(T):
    run_case(_small(n_shared=1, d_ff_shared=128), T, seed=T, path="stream")


@pytest.mark.parametrize("E,K", [(212, 16), (60, 4), (64, 6), (8, 2), (32, 32)])
def test_expert_counts_and_topk_widths(E, K):
    spec = _small(n_experts=E, top_k=K, d_ff=128)
    run_case(spec, 70, seed=E + K)


def test_all_slots_masked_gives_shared_only():
    spec = _small(n_shared=2, d_ff_shared=128)
    info = run_case(spec, 40, mask_bias=-1.0e4)
    st = info["stats"]
    assert st["n_kept"] == 0 and st["n_active_experts"] == 0 and st["n_tokens_all_masked"] == 40
    # no shared experts and nothing kept: y is exactly zero
    spec0 = _small()
    info0 = run_case(spec0, 40, mask_bias=-1.0e4)
    assert torch.count_nonzero(info0["y"]) == 0


def test_segment_routing_partial_last_segment():
    spec = _small(segment_len=16, n_shared=1, d_ff_shared=128)
    info = run_case(spec, 16 * 5 + 7)
    ids = info["routing"]["topk_id"]
    for t in range(ids.shape[0]):
        np.testing.assert_array_equal(ids[t], ids[(t // 16) * 16])


def test_zero_tokens_and_max_tokens():
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small()
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=48)
    x0 = torch.empty((0, spec.d_model), dtype=torch.bfloat16, device="cuda")
    y0 = layer.forward(x0)
    assert y0.shape == (0, spec.d_model)
    assert layer.stats()["tokens"] == 0
    run_case(spec, 48, weights=w, layer=layer)
    with pytest.raises(Exception):
        layer.forward(synth.make_tokens(spec, 49).cuda())


def test_deterministic_bits():
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=200)
    x = synth.make_tokens(spec, 200).cuda()
    y1 = layer.forward(x).clone()
    r1 = layer.routing(200)
    y2 = layer.forward(x).clone()
    r2 = layer.routing(200)
    assert torch.equal(y1, y2)
    for k in r1:
        np.testing.assert_array_equal(r1[k], r2[k])


def test_graph_replay_matches_direct_launches():
    """On a non-default stream the forward is captured once and replayed; replays must give
    the same bits as direct launches, also after x's contents change under the same pointer."""
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=96)
        for T, path in ((96, None), (3, None), (96, "stream")):
            x = synth.make_tokens(spec, T, seed=1).cuda()
            y = torch.empty((T, spec.d_model), device="cuda")
            ref = layer.forward(x, path=path, graph=False).clone()
            n0 = layer.launch_count()
            layer.forward(x, path=path, out=y)          # capture + first replay
            layer.forward(x, path=path, out=y)          # replay
            assert layer.launch_count() > n0
            torch.cuda.synchronize()
            assert torch.equal(y, ref)
            x.copy_(synth.make_tokens(spec, T, seed=2).cuda())
            layer.forward(x, path=path, out=y)
            ref2 = layer.forward(x, path=path, graph=False)
            torch.cuda.synchronize()
            assert torch.equal(y, ref2)
            assert not torch.equal(ref, ref2)


def test_bounded_wait_expires_and_the_context_survives():
    """A wait on an mbarrier nothing completes gives up after its limit and reports
    BEAM_ERR_TIMEOUT; the GPU context stays usable (a forward afterwards is still correct)."""
    import time
    from dynamic_expert_routing_b200 import _lib
    lib = _lib.load()
    t0 = time.perf_counter()
    st = lib.beam_moe_wait_selftest(20000, None)
    dt = time.perf_counter() - t0
    assert st == _lib.BEAM_ERR_TIMEOUT, lib.beam_moe_last_error()
    assert b"as designed" in lib.beam_moe_last_error()
    assert 0.015 < dt < 5.0
    run_case(_small(), 40, seed=9)


def test_allocation_failure_frees_everything(monkeypatch):
    """An allocation failing part-way through create returns BEAM_ERR_OOM, releases what was
    already allocated, and leaves the library usable."""
    from dynamic_expert_routing_b200 import BeamMoE, BeamError, _lib
    spec = _small(n_shared=1, d_ff_shared=128)
    w = to_dev(synth.make_layer(spec, keep_rate=0.5))
    wd = {k: v for k, v in w.items() if isinstance(v, torch.Tensor)}
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for n in (1, 7, 20):
        monkeypatch.setenv("BEAM_TEST_FAIL_ALLOC", str(n))
        with pytest.raises(BeamError) as ei:
            BeamMoE(wd, spec.top_k, max_tokens=4096)
        assert ei.value.status == _lib.BEAM_ERR_OOM
    monkeypatch.delenv("BEAM_TEST_FAIL_ALLOC")
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert abs(free0 - free1) < 64 << 20      # nothing of the failed creates is left behind
    run_case(spec, 50, seed=4)


def test_host_buffer_entry_point():
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=64)
    x = synth.make_tokens(spec, 64)
    y_dev = layer.forward(x.cuda()).cpu()
    y_host = torch.empty((64, spec.d_model), dtype=torch.float32).pin_memory()
    layer.forward_host(x.pin_memory(), y_host)
    assert torch.equal(y_dev, y_host)


# ------------------------------------------------------------------ tensor-core path
@pytest.mark.parametrize("T", [1, 17, 128, 129, 700])
def test_small_bf16_tensor_path(T):
    run_case(_small(n_shared=1, d_ff_shared=128), T, seed=100 + T, path="tensor")


@pytest.mark.parametrize("E,K,T", [(212, 16, 300), (60, 4, 1000), (8, 2, 2000)])
def test_tensor_path_group_shapes(E, K, T):
    spec = _small(n_experts=E, top_k=K, d_ff=384, n_shared=2, d_ff_shared=256)
    run_case(spec, T, seed=E, path="tensor")


@pytest.mark.parametrize("T", [1, 2, 3, 9, 64])
def test_tensor_path_split_k(T):
    """Small batches split K: gate/up partials finished by the SwiGLU kernel, down partials
    added by the combine; the shared group (smaller K) gets its own split count."""
    spec = _small(d_ff=1024, n_shared=1, d_ff_shared=512)
    run_case(spec, T, seed=200 + T, path="tensor")


def test_tensor_and_stream_paths_agree():
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=64)
    x = synth.make_tokens(spec, 64).cuda()
    ys = layer.forward(x, path="stream").cpu().double().numpy()
    r1 = layer.routing(64)
    yt = layer.forward(x, path="tensor").cpu().double().numpy()
    r2 = layer.routing(64)
    for k in r1:
        np.testing.assert_array_equal(r1[k], r2[k])
    assert parity.rel_l2(yt, ys) < 1e-3


def test_tensor_path_segment_and_mask_off():
    spec = _small(segment_len=16, n_shared=1, d_ff_shared=128)
    run_case(spec, 16 * 20 + 3, path="tensor")
    run_case(_small(), 200, path="tensor", mask_off=True)


# ------------------------------------------------------------------ the pages' layer shapes
@pytest.mark.parametrize("name,T,keep", [
    ("mixtral", 1, 0.5), ("mixtral", 8, 0.25), ("dsv2lite", 1, 0.07), ("dsv2lite", 64, 0.45),
    ("qwenmoe", 8, 0.14), ("fine", 32, 0.5),
])
def test_model_shapes_decode(name, T, keep):
    spec = synth.SPECS[name]
    run_case(spec, T, keep_rate=keep)


@pytest.mark.parametrize("name,T,keep,mask_off", [
    ("mixtral", 4096, 0.5, False), ("mixtral", 4096, 0.25, False), ("mixtral", 64, 0.5, False),
    ("dsv2lite", 8192, 0.45, False), ("dsv2lite", 8192, 0.07, False),
    ("qwenmoe", 16384, 0.14, False), ("fine", 8192, 0.25, False), ("fine", 8192, 0.5, True),
    ("fine_seg16", 8192, 0.5, False),
])
def test_model_shapes_prefill(name, T, keep, mask_off):
    """Full-size prefill on the path the bench times: routing on every token, y on 256 tokens
    spread evenly over the batch (first and last included)."""
    spec = synth.SPECS[name]
    sample = np.unique(np.linspace(0, T - 1, 256).round().astype(np.int64))
    info = run_case(spec, T, keep_rate=keep, mask_off=mask_off, y_tokens=sample)
    # with segment routing an unclean leader makes its whole segment unclean
    assert info["unclean"] <= 0.05 * T * max(1, spec.segment_len)


# ------------------------------------------------------------------ configuration limits
@pytest.mark.parametrize("spec,T", [
    (synth.LayerSpec("wide_d", 8192, 8, 2, 256, n_shared=1, d_ff_shared=128), 40),      # D = 8192
    (synth.LayerSpec("e256", 512, 256, 32, 128), 33),                                    # E = 256, K = 32
    (synth.LayerSpec("k1", 256, 4, 1, 128), 70),                                         # K = 1
    (synth.LayerSpec("fp32_shared_seg", 256, 8, 3, 256, n_shared=2, d_ff_shared=128,
                     storage="fp32", segment_len=8), 61),                                # fp32 path
], ids=["d8192", "e256_k32", "k1", "fp32_shared_segment"])
def test_configuration_limits(spec, T):
    run_case(spec, T, seed=77)


def test_large_max_tokens_small_forward():
    """A handle sized for a long prefill serves a one-token decode (split-K workspaces are
    sized independently of max_tokens)."""
    spec = _small(n_shared=1, d_ff_shared=128)
    run_case(spec, 1, seed=5, max_tokens=20000)
    run_case(spec, 3000, seed=6, max_tokens=20000)


@pytest.mark.parametrize("T", [4, 300])
def test_profiling_stages_count_every_launch(T):
    """Per-stage timing: every stage launches once per forward and the launches per stage add
    up to the handle's launch counter (so a roofline that divides a stage's time by its
    launches is consistent).  T = 300 runs the shared experts on the second stream, timed
    under stages of their own; T = 4 splits K and runs them inside the routed launches (as
    separate kernels: fused=False, not the one-launch decode path), with SwiGLU finished inside
    the split gate/up launch."""
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=256)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=T)
    x = synth.make_tokens(spec, T, seed=5).cuda()
    y = torch.empty((T, spec.d_model), device="cuda")
    layer.forward(x, path="tensor", out=y, fused=False)
    n = 3
    n0 = layer.launch_count()
    layer.profile_begin(n)
    for _ in range(n):
        layer.forward(x, path="tensor", out=y, fused=False)
    prof = layer.profile_end()
    assert prof["forwards"] == n
    stages = {k: v for k, v in prof.items() if k != "forwards"}
    assert sum(c for _, c in stages.values()) == layer.launch_count() - n0
    split = T <= 64
    # split K: SwiGLU is finished inside the gate/up launch (no finishing kernel)
    expect = ["tc_gateup", "tc_down"] + ([] if split else ["tc_shared_gateup", "tc_shared_down"])
    for s_ in expect:
        assert stages[s_][1] == n, (s_, stages[s_])
        assert stages[s_][0] > 0
    absent = ["tc_shared_gateup", "tc_shared_down"] if split else []
    for s_ in absent:
        assert s_ not in stages, (s_, stages)
    layer.close()


# ------------------------------------------------------------------ tail-wave K pieces
def _tail_pieces(rem, ksteps, G):
    """K pieces per tile of the last, partial wave, as the grouped GEMM chooses them: at most
    8 pieces of at least 8 k steps each in at most two sub-waves, minimising the estimated
    tail makespan sub_waves * (ceil(ksteps / s) + 4 + 3 s), and only when that is at most
    three quarters of ksteps (the unsplit tail)."""
    if rem <= 0:
        return 1
    best, best_cost = 1, ksteps
    for s in range(2, 9):
        if ksteps < 8 * s:
            break
        sub = -(-rem * s // G)
        if sub > 2:
            break
        cost = sub * (-(-ksteps // s) + 4 + 3 * s)
        if cost < best_cost:
            best, best_cost = s, cost
    return best if 4 * best_cost <= 3 * ksteps else 1


def _k_splits(G, tiles, ksteps):
    """Split-K factor of a forward of at most 64 tokens (the host's makespan rule: 4 % per
    extra split, at least 4 k steps per slice, no empty slice)."""
    best, best_cost = 1, float("inf")
    for s in range(1, 17):
        cost = (-(-tiles * s // G)) / s * (1.0 + 0.04 * (s - 1))
        if cost < best_cost - 1e-9:
            best, best_cost = s, cost
    s = max(1, min(best, max(1, ksteps // 4)))
    per = -(-ksteps // s)
    return -(-ksteps // per)


def _routed_tail_pieces(spec, T, counts):
    """K pieces of the tail tiles of the routed gate/up and down launches of a forward with
    these kept rows per expert (1 = no tail split: also whenever the launch splits K, for
    launches of fewer than 40 k steps, and for forwards with T*K <= 64 E, which run the
    swapped form for small groups instead)."""
    G = torch.cuda.get_device_properties(0).multi_processor_count
    D, F, K, E = spec.d_model, spec.d_ff, spec.top_k, spec.n_experts
    if T * K <= 64 * E:
        return {"gateup": 1, "down": 1}
    M = int(sum(-(-int(c) // 128) for c in counts))
    out = {}
    for name, nt, ks in (("gateup", 2 * F // 256, D // 64), ("down", D // 256, F // 64)):
        if T <= 64:
            groups = min(E, max(1, (T * K + 1) // 2))
            if _k_splits(G, -(-T // 128) * groups * nt, ks) > 1:
                out[name] = 1
                continue
        out[name] = _tail_pieces(M * nt % G, ks, G) if ks >= 40 else 1
    return out


@pytest.mark.parametrize("spec,T,expect", [
    (synth.LayerSpec("tail_a", 4096, 2, 1, 4096), 130, ("gateup", "down")),
    (synth.LayerSpec("tail_b", 4096, 4, 1, 512), 300, ("gateup",)),
    (synth.LayerSpec("tail_c", 1024, 4, 1, 4096), 300, ("down",)),
    (synth.LayerSpec("tail_d", 4096, 8, 2, 512), 4400, ("gateup",)),
    (synth.LayerSpec("tail_e", 3072, 2, 1, 3072, n_shared=1, d_ff_shared=512), 256, ("gateup", "down")),
], ids=["both_gemms", "deep_k_gateup", "deep_k_down", "full_wave_then_pieces",
        "with_shared_problem"])
def test_tail_wave_k_pieces(spec, T, expect):
    """Whole-K launches of the routed problem cut the tiles of their last, partial wave into K
    pieces whose f32 partials the last-arriving epilogue warp adds in piece order.  These
    shapes make the launches named in `expect` take that path (checked from the routing the
    GPU produced).  y is compared with the oracle on every token (or a spread sample for the
    larger layers); run_case runs two forwards (the second on counters the first used, which
    the compaction clears), and a direct launch gives the same bits as the graph replay."""
    big = spec.d_model * spec.d_ff * T > 2_000_000_000 or spec.d_ff_shared * spec.d_model * T > 1_000_000_000
    sample = np.unique(np.concatenate([np.arange(0, T, 13), [T - 1]])) if big else None
    info = run_case(spec, T, seed=31, y_tokens=sample)
    pieces = _routed_tail_pieces(spec, T, info["stats"]["counts"])
    for name in expect:
        assert pieces[name] > 1, (name, pieces)
    layer = info["layer"]
    y2 = layer.forward(info["x"].cuda(), graph=False)
    torch.cuda.synchronize()
    assert torch.equal(y2, info["y"])
    layer.close()


# ------------------------------------------------------------------ swapped small groups
@pytest.mark.parametrize("spec,T", [
    (synth.LayerSpec("swap", 4096, 8, 8, 2048), 16),      # groups of 16 rows: N = 32
    (synth.LayerSpec("swap", 4096, 8, 8, 2048), 32),      # 32 rows: N = 32
    (synth.LayerSpec("swap", 4096, 8, 8, 2048), 33),      # 33 rows: N = 64
    (synth.LayerSpec("swap", 4096, 8, 8, 2048), 64),      # 64 rows: N = 64
], ids=["rows16", "rows32", "rows33", "rows64"])
def test_swapped_small_groups(spec, T):
    """A group of at most 64 rows in a whole-K launch runs with the weights as the M operand
    and its rows as N = 32 or 64.  With K = E and the mask off every expert gets exactly T rows
    (these sizes keep K unsplit: 128 gate/up and 128 down tiles).  T <= 32 routes through the
    fused small-batch kernel, T = 33 and 64 through the multi-kernel path."""
    sample = np.unique(np.concatenate([np.arange(0, T, 4), [T - 1]]))
    info = run_case(spec, T, seed=41, mask_off=True, y_tokens=sample)
    np.testing.assert_array_equal(info["stats"]["counts"], np.full(spec.n_experts, T))
    layer = info["layer"]
    y2 = layer.forward(info["x"].cuda(), mask_off=True, graph=False)
    torch.cuda.synchronize()
    assert torch.equal(y2, info["y"])
    layer.close()


def test_swapped_many_small_groups():
    """Many small groups (64 experts, K = 2, 1000 tokens: 15 to 44 rows each, T*K <= 64 E) in
    whole-K launches with several waves of tiles: every group runs swapped."""
    spec = synth.LayerSpec("swap_many", 4096, 64, 2, 1280)
    T = 1000
    sample = np.unique(np.concatenate([np.arange(0, T, 16), [T - 1]]))
    info = run_case(spec, T, seed=43, mask_off=True, y_tokens=sample)
    counts = info["stats"]["counts"]
    assert (counts <= 64).all() and (counts > 0).all()
    layer = info["layer"]
    y2 = layer.forward(info["x"].cuda(), mask_off=True, graph=False)
    torch.cuda.synchronize()
    assert torch.equal(y2, info["y"])
    layer.close()


# ------------------------------------------------------------------ fused decode launch
@pytest.mark.parametrize("spec,T,mask_off", [
    (_small(), 1, False),
    (_small(n_shared=1, d_ff_shared=256), 7, False),
    (_small(segment_len=16, n_shared=1, d_ff_shared=128), 32, False),
    (_small(), 32, True),
    (synth.LayerSpec("e256", 512, 256, 32, 128), 3, False),
    (synth.SPECS["dsv2lite"], 1, False),
    (synth.SPECS["mixtral"], 8, False),
], ids=["t1", "shared_t7", "segments_t32", "mask_off_t32", "e256_k32", "dsv2lite_t1", "mixtral_t8"])
def test_fused_decode_matches_oracle_and_separate_kernels(spec, T, mask_off):
    """BEAM_FUSED_DECODE runs a batch of <= 32 tokens as one cooperative launch (router,
    routing, compaction, both GEMMs, SwiGLU, combine, separated by grid barriers).  It must meet
    the oracle like every path, repeat its own bits, and agree with the separate-kernel path,
    which sums the router logits in another order: routing equal away from near-ties, y within
    the tolerance."""
    info = run_case(spec, T, seed=61, mask_off=mask_off, fused=True)
    layer = info["layer"]
    x = info["x"].cuda()
    n0 = layer.launch_count()
    y1 = layer.forward(x, mask_off=mask_off, fused=True).clone()
    assert layer.launch_count() == n0 + 1          # one kernel
    assert torch.equal(y1, info["y"])
    r_fused = layer.routing(T)
    y2 = layer.forward(x, mask_off=mask_off, fused=False)
    r_sep = layer.routing(T)
    torch.cuda.synchronize()
    assert layer.launch_count() > n0 + 2
    same = (r_fused["topk_id"] == r_sep["topk_id"]).all(axis=1)
    assert same.mean() >= 0.9
    assert parity.rel_l2(y1.cpu().double().numpy()[same], y2.cpu().double().numpy()[same]) < 2e-3
    layer.close()


def test_fused_decode_is_one_profiled_stage():
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=256)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=8)
    x = synth.make_tokens(spec, 8, seed=3).cuda()
    layer.forward(x, fused=True)
    layer.profile_begin(2)
    layer.forward(x, fused=True)
    layer.forward(x, fused=True)
    prof = layer.profile_end()
    stages = {k: v for k, v in prof.items() if k != "forwards"}
    assert list(stages) == ["fused_decode"] and stages["fused_decode"][1] == 2
    layer.close()


# ------------------------------------------------------------------ exact ties in Top-K
@pytest.mark.parametrize("T,path", [(1, "tensor"), (24, "tensor"), (300, "tensor"), (40, "stream")])
def test_exact_ties_go_to_the_lower_expert(T, path):
    """Experts with identical router columns get bit-identical logits (every column of a
    router launch is summed in the same order), so they tie exactly.  Top-K must then take the
    lower expert first: whenever the higher one of a tied pair is selected, the lower one is
    selected too and ranks before it.  Covers the GEMV router with the fused small-batch
    routing (T <= 32), the GEMV router with the separate selection, and the tensor-core router
    (>= 64 routed rows)."""
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small()
    w = synth.make_layer(spec, keep_rate=0.5)
    wr = w["w_router"].clone()
    ties = [(0, 1), (4, 9), (4, 15), (9, 15), (7, 8)]
    wr[:, 1] = wr[:, 0]
    wr[:, 9] = wr[:, 4]
    wr[:, 15] = wr[:, 4]
    wr[:, 8] = wr[:, 7]
    w["w_router"] = wr
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=T)
    x = synth.make_tokens(spec, T, seed=19).cuda()
    layer.forward(x, path=path)
    ids = layer.routing(T)["topk_id"]
    seen = 0
    for t in range(T):
        rank = {int(e): r for r, e in enumerate(ids[t])}
        for lo, hi in ties:
            if hi in rank:
                assert lo in rank and rank[lo] < rank[hi], (t, lo, hi, ids[t])
                seen += 1
    assert seen > 0 or T == 1
    # and the same decisions as the oracle, which breaks exact ties the same way
    orr = oracle.route(x.cpu(), wr, w["w_mask"], spec.top_k)
    agree = (np.sort(ids, axis=1) == np.sort(orr.topk_id, axis=1)).all(axis=1)
    assert agree.mean() >= 0.95
    layer.close()


# ------------------------------------------------------------------ fp16 range of intermediates
@pytest.mark.parametrize("T,path,fused", [(300, "tensor", False), (5, "tensor", False),
                                          (5, "tensor", True), (40, "stream", False)],
                         ids=["tensor_whole_k", "tensor_split_k", "fused_decode", "stream"])
def test_fp16_overflow_of_h_is_reported(T, path, fused):
    """bf16 layers store H = silu(W_g x) * (W_u x) (and the unsplit expert outputs) in fp16.
    One token scaled by 1000 drives its shared expert's H far past 65504 (gate and up grow with
    the scale, H with its square); the forward must then report BEAM_ERR_RANGE from
    beam_moe_stats, on every expert path, while ordinary inputs before and after give BEAM_OK
    (the error word is cleared by every forward)."""
    from dynamic_expert_routing_b200 import BeamMoE, BeamError, _lib
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=T)
    x = synth.make_tokens(spec, T, seed=3)
    xs = x.clone()
    xs[T // 2] *= 1000.0
    layer.forward(x.cuda(), path=path, fused=fused)
    assert layer.stats()["tokens"] == T
    layer.forward(xs.cuda(), path=path, fused=fused)
    with pytest.raises(BeamError) as ei:
        layer.stats()
    assert ei.value.status == _lib.BEAM_ERR_RANGE
    layer.forward(x.cuda(), path=path, fused=fused)
    assert layer.stats()["tokens"] == T
    layer.close()


# ------------------------------------------------------------------ short-K down projection
@pytest.mark.parametrize("F,T,E,K", [(256, 1600, 8, 2), (128, 900, 16, 4), (256, 3000, 60, 4),
                                     (128, 600, 8, 1), (256, 2000, 212, 16)],
                         ids=["f256_e8", "f128_e16", "f256_e60", "f128_k1", "f256_e212"])
def test_short_k_down_projection(F, T, E, K):
    """Routed down projections with F <= 256 (at most 4 k-steps per tile) run the kernel that
    keeps a unit's H rows in shared memory for all of its N-tiles (groups of more than 64 rows on
    average: T*K > 64 E).  Groups span one to many 128-row M-tiles; y against the oracle on a
    spread sample, and a direct launch repeats the graph replay's bits."""
    spec = synth.LayerSpec("astat", 512, E, K, F, n_shared=1, d_ff_shared=128)
    assert T * K > 64 * E
    sample = np.unique(np.linspace(0, T - 1, 200).round().astype(np.int64))
    info = run_case(spec, T, seed=F + T, path="tensor", y_tokens=sample)
    if T * K / (2 * E) > 150:
        assert info["stats"]["counts"].max() > 128      # groups span several M-tiles
    layer = info["layer"]
    y2 = layer.forward(info["x"].cuda(), path="tensor", graph=False)
    torch.cuda.synchronize()
    assert torch.equal(y2, info["y"])
    layer.close()


# ------------------------------------------------------------------ pipelined host call
@pytest.mark.parametrize("T,seg", [(3000, 0), (2500, 16), (1100, 0)], ids=["t3000", "segments", "two_chunks"])
def test_pipelined_host_call(T, seg):
    """BEAM_HOST_PIPELINE: the batch runs as chunks whose copies overlap the other chunks'
    forwards.  y against the oracle on a spread sample; the routing of every token (clean tokens
    bit-exact); the statistics describe the whole call (added over the chunks on the device)
    and agree with the returned routing exactly; offsets / perm / inv are refused."""
    from dynamic_expert_routing_b200 import BeamMoE, BeamError, _lib
    spec = _small(n_shared=1, d_ff_shared=128, segment_len=seg)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=T, segment_len=seg)
    x = synth.make_tokens(spec, T, seed=17)
    yh = torch.full((T, spec.d_model), float("nan"), dtype=torch.float32).pin_memory()
    layer.forward_host(x.pin_memory(), yh, pipeline=True)
    gr = layer.routing(T, compaction=False)
    orr = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k, segment_len=seg)
    clean = orr.clean()
    for t in np.nonzero(clean)[0]:
        assert set(gr["topk_id"][t].tolist()) == set(orr.topk_id[t].tolist())
    same = clean & np.array([{int(e): int(k) for e, k in zip(gr["topk_id"][t], gr["keep"][t])} ==
                             {int(e): int(k) for e, k in zip(orr.topk_id[t], orr.keep[t])} for t in range(T)])
    sel = np.nonzero(same)[0][::7]
    y_ref = oracle.layer(x, w, orr, tokens=sel)
    parity.compare_y(yh.numpy()[sel], y_ref, spec.storage)
    st = layer.stats()
    assert st["tokens"] == T
    keep = gr["keep"].astype(bool)
    assert st["n_kept"] == int(keep.sum())
    assert st["avg_k"] == keep.sum() / T
    counts = np.bincount(gr["topk_id"][keep], minlength=spec.n_experts)
    np.testing.assert_array_equal(st["counts"], counts)
    assert st["n_active_experts"] == int((counts > 0).sum())
    assert st["n_tokens_all_masked"] == int((keep.sum(axis=1) == 0).sum())
    with pytest.raises(BeamError) as ei:
        layer.routing(T)
    assert ei.value.status == _lib.BEAM_ERR_UNSUPPORTED
    # a second call on the same buffers gives the same bits; an ordinary forward afterwards
    # restores the full routing
    y1 = yh.clone()
    layer.forward_host(x.pin_memory(), yh, pipeline=True)
    assert torch.equal(y1, yh)
    layer.forward(x.cuda())
    layer.routing(T)
    layer.close()


@pytest.mark.parametrize("T,y_dtype", [(700, torch.float32), (700, torch.bfloat16), (5, torch.float32)],
                         ids=["f32", "bf16", "decode"])
def test_host_async_calls(T, y_dtype):
    """BEAM_HOST_ASYNC: consecutive calls on alternating staging sets, queued without waits and
    finished by host_wait, give the bits of the same synchronous calls (four calls, so each
    staging set is reused with a new input); statistics describe the last call; a synchronous
    call afterwards waits for the queued copies and is itself unchanged."""
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=T)
    xs = [synth.make_tokens(spec, T, seed=40 + i).pin_memory() for i in range(3)]
    order = [0, 1, 2, 0]
    ref = []
    for i in order:
        y = torch.empty((T, spec.d_model), dtype=y_dtype).pin_memory()
        layer.forward_host(xs[i], y)
        ref.append(y)
    st_ref = layer.stats()
    ys = [torch.full((T, spec.d_model), float("nan"), dtype=y_dtype).pin_memory() for _ in order]
    for i, y in zip(order, ys):
        layer.forward_host(xs[i], y, asynchronous=True)
    layer.host_wait()
    for a, b in zip(ys, ref):
        assert torch.equal(a, b)
    st = layer.stats()
    for k in ("avg_k", "n_kept", "n_active_experts", "tokens"):
        assert st[k] == st_ref[k], k
    y2 = torch.empty((T, spec.d_model), dtype=y_dtype).pin_memory()
    layer.forward_host(xs[1], y2)
    assert torch.equal(y2, ref[1])
    layer.close()

@pytest.mark.parametrize("T", [1, 40, 700], ids=["decode", "small", "prefill"])
def test_bf16_y_is_the_rounded_float32_y(T):
    """BEAM_Y_BF16 (a bfloat16 `out`): the combine writes the float32 sum rounded to nearest
    even, so y equals the float32 forward's y converted by torch, bit for bit; the same through
    forward_routed; and the flag is refused with the fused decode launch and on host calls."""
    from dynamic_expert_routing_b200 import BeamMoE, BeamGenerator, BeamError, _lib
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    wd = to_dev(w)
    layer = BeamMoE(wd, spec.top_k, max_tokens=T)
    x = synth.make_tokens(spec, T, seed=71).cuda()
    y32 = layer.forward(x)
    y16 = layer.forward(x, out=torch.empty((T, spec.d_model), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(y16, y32.to(torch.bfloat16))
    gen = BeamGenerator(wd["w_router"][None].contiguous(), wd["w_mask"][None].contiguous(),
                        spec.top_k, max_tokens=T)
    one = gen.layer(gen.route(x), 0)
    r32 = layer.forward_routed(x, one)
    r16 = layer.forward_routed(x, one, out=torch.empty((T, spec.d_model), dtype=torch.bfloat16,
                                                        device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(r16, r32.to(torch.bfloat16))
    lib = _lib.load()
    import ctypes
    yb = torch.empty((T, spec.d_model), dtype=torch.bfloat16, device="cuda")
    assert lib.beam_moe_forward(layer._h, ctypes.c_void_p(x.data_ptr()), T, ctypes.c_void_p(yb.data_ptr()),
                                _lib.BEAM_Y_BF16 | _lib.BEAM_FUSED_DECODE, None) == _lib.BEAM_ERR_INVALID_ARG
    xh = x.cpu().pin_memory()
    with pytest.raises(BeamError):
        _lib.check(lib.beam_moe_forward_host(layer._h, ctypes.c_void_p(xh.data_ptr()), T,
                                             ctypes.c_void_p(yb.cpu().pin_memory().data_ptr()),
                                             _lib.BEAM_Y_BF16, None))
    torch.cuda.synchronize()
    gen.close()
    layer.close()

def test_host_call_forms_interleaved():
    """Host calls of every form on one handle, interleaved: asynchronous calls of different
    batch sizes and mask settings, a pipelined synchronous call between them, and asynchronous
    calls again; each result equals the synchronous plain call of the same input."""
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    Tmax = 1200
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=Tmax)
    plan = [(1200, False, "async"), (300, True, "async"), (1200, False, "pipeline"),
            (7, False, "async"), (1200, True, "async"), (1100, False, "async")]
    xs = [synth.make_tokens(spec, T, seed=60 + i).pin_memory() for i, (T, _, _) in enumerate(plan)]
    ref = []
    for (T, mo, _), x in zip(plan, xs):
        y = torch.empty((T, spec.d_model), dtype=torch.float32).pin_memory()
        layer.forward_host(x, y, mask_off=mo)
        ref.append(y)
    out = [torch.full((T, spec.d_model), float("nan")).pin_memory() for T, _, _ in plan]
    for (T, mo, form), x, y in zip(plan, xs, out):
        layer.forward_host(x, y, mask_off=mo, pipeline=form == "pipeline",
                           asynchronous=form == "async")
    layer.host_wait()
    for i, (a, b) in enumerate(zip(out, ref)):
        if plan[i][2] == "pipeline":
            # chunks run as forwards of their own (their own K splits and tail pieces, and a
            # token near a Top-K or mask tie may route differently): close on almost every row
            assert torch.isfinite(a).all()
            close = ((a - b).abs().max(dim=1).values <= 1e-2 * (1 + b.abs().max(dim=1).values))
            assert close.float().mean() > 0.95, i
        else:
            assert torch.equal(a, b), i
    with pytest.raises(ValueError):
        layer.forward_host(xs[0], out[0], pipeline=True, asynchronous=True)
    layer.close()

@pytest.mark.parametrize("T,form", [(1500, "pipeline"), (1500, "plain"), (3, "plain"), (1500, "async")],
                         ids=["pipelined", "plain", "decode", "async"])
def test_host_bf16_output(T, form):
    """BEAM_HOST_Y_BF16: the host receives y rounded to bf16 by the combine.  The bits are the
    float32 y of the same call form, rounded to nearest even (torch's conversion), so the
    output loses nothing beyond that rounding; the fused decode launch is refused with it."""
    from dynamic_expert_routing_b200 import BeamMoE
    spec = _small(n_shared=1, d_ff_shared=128)
    w = synth.make_layer(spec, keep_rate=0.5)
    layer = BeamMoE(to_dev(w), spec.top_k, max_tokens=T)
    x = synth.make_tokens(spec, T, seed=23).pin_memory()
    y32 = torch.full((T, spec.d_model), float("nan"), dtype=torch.float32).pin_memory()
    y16 = torch.full((T, spec.d_model), float("nan"), dtype=torch.bfloat16).pin_memory()
    pipeline, asynchronous = form == "pipeline", form == "async"
    layer.forward_host(x, y32, pipeline=pipeline, asynchronous=asynchronous)
    layer.forward_host(x, y16, pipeline=pipeline, asynchronous=asynchronous)
    layer.host_wait()
    assert torch.equal(y16, y32.to(torch.bfloat16))
    with pytest.raises(ValueError):
        layer.forward_host(x, torch.empty((T, spec.d_model), dtype=torch.float16), pipeline=pipeline)
    if form == "plain":
        from dynamic_expert_routing_b200 import BeamError, _lib
        import ctypes
        with pytest.raises(BeamError):
            _lib.check(_lib.load().beam_moe_forward_host(
                layer._h, ctypes.c_void_p(x.data_ptr()), T, ctypes.c_void_p(y16.data_ptr()),
                _lib.BEAM_HOST_Y_BF16 | _lib.BEAM_FUSED_DECODE, None))
    layer.close()
