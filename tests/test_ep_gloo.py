"""Expert parallelism on the CPU: two gloo ranks run the exchange logic of
dynamic_expert_routing_b200/ep.py (ExpertParallelMoE: the count and row all-to-alls, the plan of
send / receive rows, the return of the outputs in X_perm order) with a CPU stand-in for the
compute steps written from the fp64 oracle, and every rank's y must equal the single-process
oracle's layer on that rank's tokens.  The expert partition is the library's own
(beam_ep_expert_range, a host-only C call).  The GPU compute steps are tested in
tests/test_ep_gpu.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBackend:
    """The compute steps of one rank, in float64 on the CPU from the oracle: routing and
    compaction of the rank's tokens, its experts on the rows it receives, and the combine."""

    def __init__(self, w, top_k, first, count):
        self.w, self.K, self.first, self.count = w, top_k, first, count

    def dispatch(self, x):
        import oracle
        self.x = x
        self.r = oracle.route(x, self.w["w_router"], self.w["w_mask"], self.K)
        counts, offsets, perm, inv = oracle.compact(self.r, self.w["w_router"].shape[1])
        self.inv = inv.reshape(-1, self.K)
        rows = x[torch.from_numpy(perm // self.K).long()].double()
        return rows, torch.from_numpy(counts.astype(np.int32))

    def experts(self, rows, recv_counts):
        import oracle
        out = torch.zeros((rows.shape[0], rows.shape[1]), dtype=torch.float64)
        j = 0
        for s in range(recv_counts.shape[0]):            # source-major
            for e in range(recv_counts.shape[1]):        # then this rank's experts in order
                for _ in range(int(recv_counts[s, e])):
                    ge = self.first + e
                    out[j] = torch.from_numpy(oracle.expert(rows[j].numpy(), self.w["w_gate"],
                                                            self.w["w_up"], self.w["w_down"], ge))
                    j += 1
        assert j == rows.shape[0]
        return out

    def combine(self, y_perm):
        import oracle
        T = self.x.shape[0]
        none = oracle.Routing(self.r.topk_id, self.r.g, self.r.mask_logit,
                              np.zeros_like(self.r.keep), np.zeros_like(self.r.ghat),
                              self.r.r_gap, self.r.rank_gap, self.r.m_margin, self.r.nkeep, self.r.lreg)
        y = torch.from_numpy(oracle.layer(self.x, self.w, none))   # the shared experts alone
        yp = y_perm.numpy()
        for t in range(T):
            for k in range(self.K):
                p = self.inv[t, k]
                if p >= 0:
                    y[t] += self.r.ghat[t, k] * torch.from_numpy(yp[p])
        return y


def _worker(rank, world, port, spec_args, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import oracle
    import synth
    from dynamic_expert_routing_b200.ep import ExpertParallelMoE, expert_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = synth.LayerSpec(*spec_args[0], **spec_args[1])
        w = synth.make_layer(spec, keep_rate=0.5)
        first, count = expert_range(spec.n_experts, world, rank)
        ep = ExpertParallelMoE(OracleBackend(w, spec.top_k, first, count), spec.n_experts)
        T = [37, 50, 21, 8][rank]                            # ranks hold different batches
        x = synth.make_tokens(spec, T, seed=100 + rank)
        y = ep(x)
        ref = oracle.layer(x, w, oracle.route(x, w["w_router"], w["w_mask"], spec.top_k))
        out[rank] = float(np.abs(y.numpy() - ref).max() / max(1e-30, np.abs(ref).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,spec_args", [
    (2, (("ep", 64, 8, 2, 32), dict(storage="fp32"))),
    (2, (("ep_shared", 64, 6, 3, 32), dict(storage="fp32", n_shared=1, d_ff_shared=32))),
    (3, (("ep_uneven", 64, 7, 2, 32), dict(storage="bf16"))),
], ids=["two_ranks", "two_ranks_shared", "three_ranks_uneven_blocks"])
def test_expert_parallel_exchange_matches_single_process_oracle(world, spec_args):
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, spec_args, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r] < 1e-12, (r, out[r])


def test_expert_ranges_partition_the_experts():
    sys.path.insert(0, ROOT)
    from dynamic_expert_routing_b200.ep import ExchangePlan, expert_range
    for E, P in ((8, 2), (60, 8), (212, 8), (7, 3), (3, 4), (1, 1)):
        ranges = [expert_range(E, P, q) for q in range(P)]
        assert ranges[0][0] == 0
        for (f0, c0), (f1, _) in zip(ranges, ranges[1:]):
            assert f0 + c0 == f1
        assert sum(c for _, c in ranges) == E
        assert max(c for _, c in ranges) - min(c for _, c in ranges) <= 1
    plan = ExchangePlan([3, 0, 2, 5], [[1, 2], [0, 4]], [(0, 2), (2, 2)])
    assert plan.send_rows == [3, 7] and plan.recv_rows == [3, 4]
    assert plan.n_kept == 10 and plan.n_recv == 7
    from dynamic_expert_routing_b200 import BeamError
    with pytest.raises(BeamError):
        expert_range(8, 2, 2)
