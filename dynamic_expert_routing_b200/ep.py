"""Expert parallelism for the BEAM layer: the routed experts split over P ranks, tokens
exchanged with all-to-all (the BEAM article on aitrends.kr leaves multi-GPU interaction to future
work, limitation (D)).

Rank q holds the experts [floor(qE/P), floor((q+1)E/P)) (beam_ep_expert_range), the router and
mask router of all E experts, and the shared experts.  A forward of a rank's own tokens x:

  1. dispatch: routing over all E experts and the compaction (library kernels).  X_perm holds
     the kept rows sorted by expert, then token, so the rows for rank r's experts are one
     contiguous range of it, and the per-expert counts give the ranges;
  2. the counts of each rank's experts go to that rank (all-to-all of E int32);
  3. the rows go to the ranks holding their experts (all-to-all of rows);
  4. experts: the received rows (source-major, expert-minor) run through the rank's experts
     (library kernels: one-slot routing of each row, grouping by expert, the grouped SwiGLU
     GEMMs, and the output row written back in received order);
  5. the outputs go back (the reverse all-to-all): each rank gets its rows' expert outputs in
     X_perm order;
  6. combine: the fixed-order weighted sum with the gates, plus the shared experts (library).

The exchanges run with torch.distributed (NCCL on GPUs); every rank makes the same collective
calls in the same order.  The compute steps are behind a small backend interface, so that the
exchange logic can also be driven by a CPU stand-in (the gloo tests); on a GPU the backend is
`LibraryBackend`, whose every step runs in the CUDA library.  No peer GPU memory is given to any
kernel: rows cross between GPUs only inside the collectives.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import check


def expert_range(n_experts: int, world: int, rank: int) -> tuple[int, int]:
    """(first, count) of rank `rank`'s experts, by the library's own partition (host call)."""
    first, count = ctypes.c_int32(), ctypes.c_int32()
    check(_lib.load().beam_ep_expert_range(int(n_experts), int(world), int(rank),
                                           ctypes.byref(first), ctypes.byref(count)))
    return first.value, count.value


class ExchangePlan:
    """Row counts of one forward's exchange, from this rank's per-expert counts and the counts
    it received: send_rows[r] rows go to rank r (its experts' range of X_perm) and recv_rows[s]
    rows come from rank s (the sum of what s holds for this rank's experts)."""

    def __init__(self, counts: list[int], recv_counts: list[list[int]], ranges: list[tuple[int, int]]):
        self.send_rows = [sum(counts[f:f + c]) for f, c in ranges]
        self.recv_rows = [sum(row) for row in recv_counts]
        self.n_kept = sum(counts)
        self.n_recv = sum(self.recv_rows)


class ExpertParallelMoE:
    """One rank of an expert-parallel BEAM layer.

    backend: the compute steps (LibraryBackend on a GPU); group: the torch.distributed process
    group of the P ranks (default: the world)."""

    def __init__(self, backend, n_experts: int, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.P = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E = int(n_experts)
        self.ranges = [expert_range(self.E, self.P, r) for r in range(self.P)]
        self.first, self.E_local = self.ranges[self.rank]
        self.backend = backend

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        dist, g = self.dist, self.group
        rows, counts = self.backend.dispatch(x)
        # 2. counts of each destination's experts (its contiguous slice of counts[E])
        recv_counts = torch.empty(self.P * self.E_local, dtype=torch.int32, device=counts.device)
        dist.all_to_all_single(recv_counts, counts, output_split_sizes=[self.E_local] * self.P,
                               input_split_sizes=[c for _, c in self.ranges], group=g)
        plan = ExchangePlan(counts.cpu().tolist(), recv_counts.view(self.P, self.E_local).cpu().tolist(),
                            self.ranges)
        # 3. rows to the ranks holding their experts
        recv = torch.empty((plan.n_recv, rows.shape[1]), dtype=rows.dtype, device=rows.device)
        dist.all_to_all_single(recv, rows[:plan.n_kept], output_split_sizes=plan.recv_rows,
                               input_split_sizes=plan.send_rows, group=g)
        # 4. this rank's experts on the rows it received
        y_recv = self.backend.experts(recv, recv_counts.view(self.P, self.E_local))
        # 5. outputs back, in this rank's X_perm order
        y_perm = torch.empty((plan.n_kept, y_recv.shape[1]), dtype=y_recv.dtype, device=y_recv.device)
        dist.all_to_all_single(y_perm, y_recv, output_split_sizes=plan.send_rows,
                               input_split_sizes=plan.recv_rows, group=g)
        # 6. fixed-order combine with the shared experts
        return self.backend.combine(y_perm)

    __call__ = forward


class LibraryBackend:
    """The compute steps of one expert-parallel rank in the CUDA library: a routing-only handle
    (all E experts' router and mask router, the shared experts) and an expert handle over the
    rank's own E_local experts (top_k = 1, no shared experts), both built from `weights`:
    w_router, w_mask [D][E], optional ws_gate/ws_up/ws_down, and w_gate/w_up [E_local][F][D],
    w_down [E_local][D][F] for this rank's block of experts.  max_recv_rows bounds the rows one
    forward can receive (default: P * max_tokens * min(top_k, E_local))."""

    def __init__(self, weights: dict, top_k: int, max_tokens: int, world: int,
                 segment_len: int = 0, max_recv_rows: int | None = None, stream=None):
        from .layer import _DTYPES, _ptr, _stream_handle, BeamMoE
        from ._lib import BeamConfig, BeamWeights
        lib = _lib.load()
        wr = weights["w_router"]
        D, E = wr.shape
        wsg = weights.get("ws_gate")
        S = 0 if wsg is None else wsg.shape[0]
        Fs = 0 if wsg is None else wsg.shape[1]
        F = weights["w_gate"].shape[1]
        E_local = weights["w_gate"].shape[0]
        self.cfg = BeamConfig(D, E, top_k, F, S, Fs, _DTYPES[wr.dtype], segment_len, max_tokens)
        w = BeamWeights(_ptr(wr), _ptr(weights["w_mask"]), None, None, None, _ptr(wsg),
                        _ptr(weights.get("ws_up")), _ptr(weights.get("ws_down")))
        h = ctypes.c_void_p()
        check(lib.beam_moe_create_ep(ctypes.byref(self.cfg), ctypes.byref(w),
                                     ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(h)))
        self._h = h
        self.D, self.E, self.K, self.E_local, self.T_max = D, E, top_k, E_local, max_tokens
        self.dtype = wr.dtype
        self.max_recv = max_recv_rows or max(1, world * max_tokens * min(top_k, max(1, E_local)))
        self.experts_layer = None
        if E_local > 0:
            zeros = torch.zeros((D, E_local), dtype=wr.dtype, device=wr.device)
            ew = dict(w_router=zeros, w_mask=zeros, w_gate=weights["w_gate"],
                      w_up=weights["w_up"], w_down=weights["w_down"])
            self.experts_layer = BeamMoE(ew, 1, self.max_recv, stream=stream)
        dev = wr.device
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.rows = torch.empty((max_tokens * top_k, D), dtype=wr.dtype, device=dev)
        n = self.max_recv
        self.route = dict(topk_id=torch.empty((n, 1), dtype=torch.int32, device=dev),
                          keep=torch.empty((n, 1), dtype=torch.uint8, device=dev),
                          ghat=torch.empty((n, 1), dtype=torch.float32, device=dev),
                          n_keep=torch.empty((n,), dtype=torch.int32, device=dev),
                          lreg=torch.empty((n,), dtype=torch.float32, device=dev))
        self._T = 0

    def dispatch(self, x: torch.Tensor, mask_off: bool = False, stream=None):
        """(X_perm rows [T*K][D] in the storage type, of which the first n_kept are the kept
        rows by expert then token; per-expert counts [E] int32), both on the device."""
        from .layer import _ptr, _stream_handle
        from ._lib import BEAM_MASK_OFF
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.dtype):
            raise ValueError("x must be a contiguous CUDA tensor of the layer's storage dtype")
        T = x.shape[0]
        check(_lib.load().beam_moe_ep_dispatch(self._h, _ptr(x), T, BEAM_MASK_OFF if mask_off else 0,
                                               _ptr(self.rows), _ptr(self.counts),
                                               ctypes.c_void_p(_stream_handle(stream))))
        self._T = T
        return self.rows[:T * self.K], self.counts

    def experts(self, rows: torch.Tensor, recv_counts: torch.Tensor, stream=None) -> torch.Tensor:
        from .layer import _ptr, _stream_handle
        n = rows.shape[0]
        out = torch.empty((n, self.D), dtype=torch.float32, device=rows.device)
        if n == 0:
            return out
        if n > self.max_recv:
            raise ValueError(f"{n} rows received; the expert handle holds {self.max_recv}")
        r = {k: v[:n] for k, v in self.route.items()}
        P, El = recv_counts.shape
        check(_lib.load().beam_ep_recv_routing(_ptr(recv_counts.contiguous()), P, El, n,
                                               _ptr(r["topk_id"]), _ptr(r["keep"]), _ptr(r["ghat"]),
                                               _ptr(r["n_keep"]), _ptr(r["lreg"]),
                                               ctypes.c_void_p(_stream_handle(stream))))
        return self.experts_layer.forward_routed(rows.contiguous(), r, out=out, stream=stream,
                                                 graph=False)

    def combine(self, y_perm: torch.Tensor, stream=None) -> torch.Tensor:
        from .layer import _ptr, _stream_handle
        y = torch.empty((self._T, self.D), dtype=torch.float32, device=y_perm.device)
        check(_lib.load().beam_moe_ep_combine(self._h, _ptr(y_perm.contiguous()), _ptr(y),
                                              ctypes.c_void_p(_stream_handle(stream))))
        return y

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.load().beam_moe_destroy(self._h)
            self._h = None
        if self.experts_layer is not None:
            self.experts_layer.close()
            self.experts_layer = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

