"""Expert parallelism on one GPU, through the C ABI, against the fp64 oracle.

* one rank (P = 1): ExpertParallelMoE over a real NCCL process group of one rank, with the
  library's compute steps (LibraryBackend): dispatch, the count and row all-to-alls, the expert
  handle's routed forward on the received rows, the return all-to-all and the combine;
* two and three ranks emulated in one process: every rank's LibraryBackend holds only its block
  of experts; the test moves the rows between the ranks itself, by the same ExchangePlan the
  distributed forward uses, so the library's receive-side routing (rows from several sources,
  source-major) and the combine of returned rows are exercised with real multi-rank layouts.
  (No kernels wait on each other: the ranks' steps run one after another.)

Bars: the routing is each rank's own (compared with the oracle on clean tokens, as the layer
tests do); y within the bf16 bars of the layer (max abs 2e-2, relative L2 5e-3) on tokens whose
decision equals the oracle's; every token counted.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shard(w, first, count):
    out = {k: v for k, v in w.items() if k in ("w_router", "w_mask", "ws_gate", "ws_up", "ws_down")}
    for k in ("w_gate", "w_up", "w_down"):
        out[k] = w[k][first:first + count].contiguous()
    return {k: v.cuda().contiguous() for k, v in out.items() if isinstance(v, torch.Tensor)}


def _check(x, y, w, spec):
    orr = oracle.route(x, w["w_router"], w["w_mask"], spec.top_k)
    clean = orr.clean()
    assert clean.mean() > 0.8
    sel = np.nonzero(clean)[0]
    y_ref = oracle.layer(x, w, orr, tokens=sel)
    return parity.compare_y(y.cpu().numpy()[sel], y_ref, spec.storage)


@pytest.mark.parametrize("spec,T", [
    (synth.LayerSpec("ep", 512, 8, 2, 256, n_shared=1, d_ff_shared=128), 70),
    (synth.LayerSpec("ep_small", 512, 16, 4, 256), 5),
], ids=["shared_t70", "t5"])
def test_ep_one_rank_over_nccl(spec, T):
    import torch.distributed as dist
    from dynamic_expert_routing_b200.ep import ExpertParallelMoE, LibraryBackend
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        w = synth.make_layer(spec, keep_rate=0.5)
        be = LibraryBackend(_shard(w, 0, spec.n_experts), spec.top_k, T, world=1)
        ep = ExpertParallelMoE(be, spec.n_experts)
        x = synth.make_tokens(spec, T, seed=3)
        y = ep(x.cuda())
        torch.cuda.synchronize()
        _check(x, y, w, spec)
        be.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("spec,P,Ts", [
    (synth.LayerSpec("ep2", 512, 8, 2, 256, n_shared=1, d_ff_shared=128), 2, (70, 33)),
    (synth.LayerSpec("ep3", 512, 7, 3, 256), 3, (9, 130, 1)),
    (synth.LayerSpec("ep_dsv2", 2048, 64, 6, 1408, n_shared=2, d_ff_shared=1408), 2, (200, 16)),
], ids=["two_ranks_shared", "three_ranks_uneven", "two_ranks_dsv2_shape"])
def test_ep_emulated_ranks(spec, P, Ts):
    from dynamic_expert_routing_b200.ep import ExchangePlan, LibraryBackend, expert_range
    w = synth.make_layer(spec, keep_rate=0.5)
    ranges = [expert_range(spec.n_experts, P, q) for q in range(P)]
    bes = [LibraryBackend(_shard(w, f, c), spec.top_k, max(Ts), world=P) for f, c in ranges]
    xs = [synth.make_tokens(spec, T, seed=10 + q) for q, T in enumerate(Ts)]
    # 1. every rank dispatches its own tokens
    disp = [be.dispatch(x.cuda()) for be, x in zip(bes, xs)]
    counts = [c.cpu().tolist() for _, c in disp]
    # 2. counts of each rank's experts, as the count all-to-all delivers them
    recv_counts = [[counts[s][f:f + c] for s in range(P)] for f, c in ranges]
    plans = [ExchangePlan(counts[q], recv_counts[q], ranges) for q in range(P)]
    # 3. rows: rank q receives, from each source s in order, s's rows of q's experts
    offs = [np.concatenate([[0], np.cumsum(p.send_rows)]) for p in plans]
    recv = [torch.cat([disp[s][0][offs[s][q]:offs[s][q + 1]] for s in range(P)]) for q in range(P)]
    # 4. every rank's experts on what it received
    y_recv = [bes[q].experts(recv[q], torch.tensor(recv_counts[q], dtype=torch.int32,
                                                   device="cuda").view(P, -1)) for q in range(P)]
    # 5. outputs back: rank s gets, from each expert rank q in order, the rows it sent to q
    roffs = [np.concatenate([[0], np.cumsum(p.recv_rows)]) for p in plans]
    y_perm = [torch.cat([y_recv[q][roffs[q][s]:roffs[q][s + 1]] for q in range(P)]) for s in range(P)]
    # 6. combine on every rank
    ys = [bes[s].combine(y_perm[s]) for s in range(P)]
    torch.cuda.synchronize()
    for s in range(P):
        assert y_perm[s].shape[0] == plans[s].n_kept
        _check(xs[s], ys[s], w, spec)
    for be in bes:
        be.close()


def test_routing_only_handle_rejects_forward_and_receive_routing_layout():
    from dynamic_expert_routing_b200 import BeamError, _lib
    from dynamic_expert_routing_b200.ep import LibraryBackend
    spec = synth.LayerSpec("ep_r", 512, 8, 2, 256)
    w = synth.make_layer(spec, keep_rate=0.5)
    be = LibraryBackend(_shard(w, 0, 4), spec.top_k, 16, world=2)
    lib = _lib.load()
    import ctypes
    x = synth.make_tokens(spec, 16).cuda()
    y = torch.empty((16, 512), device="cuda")
    st = lib.beam_moe_forward(be._h, ctypes.c_void_p(x.data_ptr()), 16, ctypes.c_void_p(y.data_ptr()),
                              0, None)
    assert st == _lib.BEAM_ERR_UNSUPPORTED
    # receive-side routing: 3 sources x 4 local experts, source-major / expert-minor
    rc = torch.tensor([[2, 0, 1, 0], [0, 0, 0, 3], [1, 1, 0, 0]], dtype=torch.int32, device="cuda")
    n = int(rc.sum())
    r = {k: v[:n] for k, v in be.route.items()}
    assert lib.beam_ep_recv_routing(ctypes.c_void_p(rc.data_ptr()), 3, 4, n,
                                    *[ctypes.c_void_p(r[k].data_ptr()) for k in
                                      ("topk_id", "keep", "ghat", "n_keep", "lreg")], None) == 0
    torch.cuda.synchronize()
    assert r["topk_id"].view(-1).tolist() == [0, 0, 2, 3, 3, 3, 0, 1]
    assert (r["keep"] == 1).all() and (r["ghat"] == 1).all() and (r["n_keep"] == 1).all()
    be.close()
