"""Python handle over the C ABI: torch tensors in, pointers to the CUDA library out.

Every step of the layer runs in the library's kernels; this module only marshals arguments.
PyTorch provides device memory and the current CUDA stream.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from ._lib import (BEAM_DTYPE_BF16, BEAM_DTYPE_F32, BEAM_MASK_OFF, BEAM_FUSED_DECODE, BEAM_NO_GRAPH,
                   BEAM_PATH_STREAM, BEAM_PATH_TENSOR, BEAM_TRAIN, BeamConfig, BeamGenConfig,
                   BeamRouting, BeamStats, BeamWeights, check)

_DTYPES = {torch.float32: BEAM_DTYPE_F32, torch.bfloat16: BEAM_DTYPE_BF16}
_PATHS = {None: 0, "auto": 0, "stream": BEAM_PATH_STREAM, "tensor": BEAM_PATH_TENSOR}


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _y_flag(out: torch.Tensor, T: int, D: int) -> int:
    """BEAM_Y_BF16 for a bfloat16 output tensor; the output must be a contiguous CUDA tensor
    of float32 or bfloat16 with room for [T][D]."""
    if not (out.is_cuda and out.is_contiguous() and out.numel() >= T * D
            and out.dtype in (torch.float32, torch.bfloat16)):
        raise ValueError("out must be a contiguous CUDA float32 or bfloat16 tensor of at least T*D values")
    return _lib.BEAM_Y_BF16 if out.dtype == torch.bfloat16 else 0


class BeamMoE:
    """A BEAM masked MoE layer held by the CUDA library.

    weights: dict with w_router [D][E], w_mask [D][E], w_gate/w_up [E][F][D], w_down [E][D][F]
    and, with shared experts, ws_gate/ws_up [S][Fs][D], ws_down [S][D][Fs]; CUDA tensors of one
    storage type (float32 or bfloat16).  The library copies them at construction.
    """

    def __init__(self, weights: dict, top_k: int, max_tokens: int, segment_len: int = 0,
                 stream=None):
        lib = _lib.load()
        wr = weights["w_router"]
        dt = _DTYPES.get(wr.dtype)
        if dt is None:
            raise TypeError(f"unsupported storage dtype {wr.dtype}")
        for k in ("w_router", "w_mask", "w_gate", "w_up", "w_down"):
            t = weights[k]
            if not (t.is_cuda and t.is_contiguous() and t.dtype == wr.dtype):
                raise ValueError(f"{k} must be a contiguous CUDA tensor of dtype {wr.dtype}")
        D, E = wr.shape
        F = weights["w_gate"].shape[1]
        wsg = weights.get("ws_gate")
        S = 0 if wsg is None else wsg.shape[0]
        Fs = 0 if wsg is None else wsg.shape[1]
        self.cfg = BeamConfig(D, E, top_k, F, S, Fs, dt, segment_len, max_tokens)
        w = BeamWeights(*[_ptr(weights.get(k)) for k in ("w_router", "w_mask", "w_gate", "w_up",
                                                         "w_down", "ws_gate", "ws_up", "ws_down")])
        h = ctypes.c_void_p()
        check(lib.beam_moe_create(ctypes.byref(self.cfg), ctypes.byref(w),
                                  ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(h)))
        self._h = h
        self.dtype = wr.dtype
        self.d_model, self.n_experts, self.top_k = D, E, top_k
        self.max_tokens = max_tokens

    # -------------------------------------------------------------- forward
    @staticmethod
    def flags(mask_off: bool = False, path: str | None = None, graph: bool = True,
              fused: bool = False, train: bool = False) -> int:
        return ((BEAM_MASK_OFF if mask_off else 0) | _PATHS[path] | (0 if graph else BEAM_NO_GRAPH)
                | (BEAM_FUSED_DECODE if fused else 0) | (BEAM_TRAIN if train else 0))

    def forward(self, x: torch.Tensor, mask_off: bool = False, path: str | None = None,
                out: torch.Tensor | None = None, stream=None, graph: bool = True,
                fused: bool = False, train: bool = False) -> torch.Tensor:
        """y [T][D] float32 of x [T][D] (storage dtype, CUDA), enqueued on the current stream.
        graph=False launches the kernels directly instead of replaying a captured graph;
        fused=True runs a bf16 batch of <= 32 tokens as one cooperative launch (opt-in);
        train=True evaluates every Top-K slot's expert (the mask only scales the gates) so
        that backward_router can follow.  A bfloat16 `out` receives y rounded to bf16
        (BEAM_Y_BF16)."""
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.dtype):
            raise ValueError("x must be a contiguous CUDA tensor of the layer's storage dtype")
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.d_model), dtype=torch.float32, device=x.device)
        check(_lib.load().beam_moe_forward(self._h, _ptr(x), T, _ptr(out),
                                           self.flags(mask_off, path, graph, fused, train) |
                                           _y_flag(out, T, self.d_model),
                                           ctypes.c_void_p(_stream_handle(stream))))
        return out

    __call__ = forward

    def backward_router(self, x: torch.Tensor, dy: torch.Tensor, reg_scale: float = 0.0,
                        slots: bool = False, stream=None) -> dict:
        """Gradient of the routing after a forward(train=True) of the same x: dW_router,
        dW_mask [D][E] and the routing's share of dx [T][D] (float32), for the upstream
        gradient dy [T][D] (float32) and reg_scale = dL/dL_reg.  slots=True also returns the
        per-slot d_gate_logit, d_mask_logit and dghat [T][K]."""
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.dtype):
            raise ValueError("x must be a contiguous CUDA tensor of the layer's storage dtype")
        T = x.shape[0]
        if not (dy.is_cuda and dy.is_contiguous() and dy.dtype == torch.float32
                and tuple(dy.shape) == (T, self.d_model)):
            raise ValueError("dy must be a contiguous CUDA float32 tensor of shape [T][D]")
        D, E, K = self.d_model, self.n_experts, self.top_k
        f32 = dict(dtype=torch.float32, device=x.device)
        out = dict(dw_router=torch.empty((D, E), **f32), dw_mask=torch.empty((D, E), **f32),
                   dx=torch.empty((T, D), **f32))
        if slots:
            for k in ("d_gate_logit", "d_mask_logit", "dghat"):
                out[k] = torch.empty((T, K), **f32)
        check(_lib.load().beam_moe_backward_router(
            self._h, _ptr(x), _ptr(dy), T, ctypes.c_float(reg_scale), _ptr(out["dw_router"]),
            _ptr(out["dw_mask"]), _ptr(out["dx"]), _ptr(out.get("d_gate_logit")),
            _ptr(out.get("d_mask_logit")), _ptr(out.get("dghat")),
            ctypes.c_void_p(_stream_handle(stream))))
        return out

    def forward_routed(self, x: torch.Tensor, routing: dict, path: str | None = None,
                       out: torch.Tensor | None = None, stream=None, graph: bool = True) -> torch.Tensor:
        """y [T][D] float32 of x [T][D] with the routing given (one layer's slice of
        BeamGenerator.route, see BeamGenerator.layer): the router and the Top-K/mask step are
        skipped, the compaction, experts and combine run as in forward."""
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.dtype):
            raise ValueError("x must be a contiguous CUDA tensor of the layer's storage dtype")
        T = x.shape[0]
        for k, dt in (("topk_id", torch.int32), ("keep", torch.uint8), ("ghat", torch.float32),
                      ("n_keep", torch.int32), ("lreg", torch.float32)):
            t = routing[k]
            if not (t.is_cuda and t.is_contiguous() and t.dtype == dt and t.shape[0] == T):
                raise ValueError(f"routing[{k!r}] must be a contiguous CUDA {dt} tensor of {T} rows")
        if out is None:
            out = torch.empty((T, self.d_model), dtype=torch.float32, device=x.device)
        r = _routing_struct(routing)
        check(_lib.load().beam_moe_forward_routed(self._h, _ptr(x), T, ctypes.byref(r), _ptr(out),
                                                  self.flags(False, path, graph) |
                                                  _y_flag(out, T, self.d_model),
                                                  ctypes.c_void_p(_stream_handle(stream))))
        return out

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, mask_off: bool = False,
                     path: str | None = None, stream=None, pipeline: bool = False,
                     asynchronous: bool = False) -> torch.Tensor:
        """Host-buffer variant: copies x in, runs the layer, copies y out, synchronises.
        pipeline=True (batches of >= 1024 tokens) runs chunks whose copies overlap the
        forwards of the others (see BEAM_HOST_PIPELINE).  asynchronous=True returns once the
        copies and the forward are queued (BEAM_HOST_ASYNC): consecutive calls overlap one
        call's forward with the neighbours' copies; call host_wait() before reading y_host or
        reusing x_host.  A bfloat16 y_host receives y rounded to bf16 on the device
        (BEAM_HOST_Y_BF16); otherwise y_host is float32."""
        T = x_host.shape[0]
        if y_host.dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("y_host must be float32 or bfloat16")
        if pipeline and asynchronous:
            raise ValueError("pipeline and asynchronous are exclusive")
        flags = self.flags(mask_off, path) | (_lib.BEAM_HOST_PIPELINE if pipeline else 0) | \
            (_lib.BEAM_HOST_ASYNC if asynchronous else 0) | \
            (_lib.BEAM_HOST_Y_BF16 if y_host.dtype == torch.bfloat16 else 0)
        check(_lib.load().beam_moe_forward_host(self._h, _ptr(x_host), T, _ptr(y_host), flags,
                                                ctypes.c_void_p(_stream_handle(stream))))
        return y_host

    def host_wait(self) -> None:
        """Wait for every queued host call's copies and the last forward (BEAM_HOST_ASYNC)."""
        check(_lib.load().beam_moe_host_wait(self._h))

    # -------------------------------------------------------------- inspection
    def stats(self) -> dict:
        s = BeamStats()
        counts = np.zeros(self.n_experts, np.int32)
        check(_lib.load().beam_moe_stats(self._h, ctypes.byref(s),
                                         counts.ctypes.data_as(ctypes.c_void_p)))
        return dict(avg_k=s.avg_k, l_reg=s.l_reg, n_active_experts=s.n_active_experts,
                    n_tokens_all_masked=s.n_tokens_all_masked, tokens=s.tokens,
                    n_kept=s.n_kept, counts=counts)

    def routing(self, T: int, compaction: bool = True) -> dict:
        """Routing of the last forward (T must be that forward's token count); compaction=False
        leaves out offsets, perm and inv (not kept by a pipelined host call)."""
        K, E = self.top_k, self.n_experts
        out = dict(topk_id=np.zeros((T, K), np.int32), gate=np.zeros((T, K), np.float32),
                   mask_logit=np.zeros((T, K), np.float32), keep=np.zeros((T, K), np.uint8))
        if compaction:
            out.update(offsets=np.zeros(E + 1, np.int32), perm=np.zeros(max(1, T * K), np.int32),
                       inv=np.zeros((T, K), np.int32))
        p = {k: v.ctypes.data_as(ctypes.c_void_p) for k, v in out.items()}
        check(_lib.load().beam_moe_get_routing(self._h, p["topk_id"], p["gate"], p["mask_logit"],
                                               p["keep"], p.get("offsets"), p.get("perm"), p.get("inv")))
        if compaction:
            out["perm"] = out["perm"][: int(out["offsets"][E])].copy()
        return out

    def profile_begin(self, max_forwards: int) -> None:
        """Time every kernel of the next `max_forwards` forwards with CUDA events."""
        check(_lib.load().beam_moe_profile_begin(self._h, int(max_forwards)))

    def profile_end(self) -> dict:
        """{stage name: (total ms, launches)} over the profiled forwards, plus 'forwards'."""
        n = _lib.BEAM_N_STAGES
        ms = (ctypes.c_float * n)()
        cnt = (ctypes.c_int32 * n)()
        nf = ctypes.c_int32()
        lib = _lib.load()
        check(lib.beam_moe_profile_end(self._h, ms, cnt, ctypes.byref(nf)))
        out = {lib.beam_moe_stage_name(i).decode(): (float(ms[i]), int(cnt[i]))
               for i in range(n) if cnt[i] > 0}
        out["forwards"] = int(nf.value)
        return out

    def launch_count(self) -> int:
        """Kernels launched by this layer's forwards so far."""
        return int(_lib.load().beam_moe_launch_count(self._h))

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.load().beam_moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


_ROUTING_FIELDS = ("topk_id", "gate", "mask_logit", "keep", "ghat", "n_keep", "lreg", "active")


def _routing_struct(routing: dict) -> BeamRouting:
    return BeamRouting(*[_ptr(routing.get(k)) for k in _ROUTING_FIELDS])


class BeamGenerator:
    """Cross-layer mask generator held by the CUDA library.

    w_router, w_mask: [L][D][E] CUDA tensors of one storage type (float32 or bfloat16), layer
    l's router and mask-router matrices.  route(z) gives every layer's routing of the token
    batch z [T][D] at once (one decision per segment of `segment_len` tokens, taken at the
    segment's first token, when segment_len > 1).
    """

    def __init__(self, w_router: torch.Tensor, w_mask: torch.Tensor, top_k: int, max_tokens: int,
                 segment_len: int = 0, stream=None):
        lib = _lib.load()
        dt = _DTYPES.get(w_router.dtype)
        if dt is None:
            raise TypeError(f"unsupported storage dtype {w_router.dtype}")
        for name, t in (("w_router", w_router), ("w_mask", w_mask)):
            if not (t.is_cuda and t.is_contiguous() and t.dtype == w_router.dtype and t.dim() == 3
                    and t.shape == w_router.shape):
                raise ValueError(f"{name} must be a contiguous [L][D][E] CUDA tensor of dtype {w_router.dtype}")
        L, D, E = w_router.shape
        self.cfg = BeamGenConfig(D, L, E, top_k, dt, segment_len, max_tokens)
        h = ctypes.c_void_p()
        check(lib.beam_gen_create(ctypes.byref(self.cfg), _ptr(w_router), _ptr(w_mask),
                                  ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(h)))
        self._h = h
        self.dtype = w_router.dtype
        self.n_layers, self.d_model, self.n_experts, self.top_k = L, D, E, top_k
        self.max_tokens = max_tokens

    def route(self, z: torch.Tensor, mask_off: bool = False, out: dict | None = None,
              stream=None) -> dict:
        """Every layer's routing of z [T][D]: topk_id [L][T][K] int32, gate, mask_logit, ghat
        [L][T][K] float32, keep [L][T][K] uint8, n_keep [L][T] int32, lreg [L][T] float32 and
        active [L][(E+31)/32] int32 (bit e%32 of word e/32: expert e kept in that layer)."""
        if not (z.is_cuda and z.is_contiguous() and z.dtype == self.dtype):
            raise ValueError("z must be a contiguous CUDA tensor of the generator's storage dtype")
        T = z.shape[0]
        L, K, nw = self.n_layers, self.top_k, (self.n_experts + 31) // 32
        if out is None:
            dev = z.device
            out = dict(topk_id=torch.empty((L, T, K), dtype=torch.int32, device=dev),
                       gate=torch.empty((L, T, K), dtype=torch.float32, device=dev),
                       mask_logit=torch.empty((L, T, K), dtype=torch.float32, device=dev),
                       keep=torch.empty((L, T, K), dtype=torch.uint8, device=dev),
                       ghat=torch.empty((L, T, K), dtype=torch.float32, device=dev),
                       n_keep=torch.empty((L, T), dtype=torch.int32, device=dev),
                       lreg=torch.empty((L, T), dtype=torch.float32, device=dev),
                       active=torch.empty((L, nw), dtype=torch.int32, device=dev))
        r = _routing_struct(out)
        check(_lib.load().beam_gen_route(self._h, _ptr(z), T, ctypes.byref(r),
                                         BEAM_MASK_OFF if mask_off else 0,
                                         ctypes.c_void_p(_stream_handle(stream))))
        return out

    @staticmethod
    def layer(routing: dict, l: int) -> dict:
        """Layer l's slice of a route() result (views), as BeamMoE.forward_routed takes it."""
        return {k: v[l] for k, v in routing.items()}

    def sync(self) -> None:
        """Wait for the last route(); raises if one of its bounded device waits ran out."""
        check(_lib.load().beam_gen_sync(self._h))

    def close(self) -> None:
        if getattr(self, "_h", None):
            _lib.load().beam_gen_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def softtopk(logits: torch.Tensor, top_k: int, tau: float, mask: bool = True, nu: bool = False,
             stream=None) -> dict:
    """SoftTopK of routing logits [T][E] (float32, CUDA): the relaxed mask y [T][E] float32,
    y_i = sigmoid((r_i - nu) / tau) with sum_i y_i = top_k, plus (mask=True) the hard Top-K
    indicator [T][E] uint8 and (nu=True) nu [T] float32.  See beam_softtopk_forward."""
    if not (logits.is_cuda and logits.is_contiguous() and logits.dtype == torch.float32
            and logits.dim() == 2):
        raise ValueError("logits must be a contiguous [T][E] CUDA float32 tensor")
    T, E = logits.shape
    out = dict(y=torch.empty((T, E), dtype=torch.float32, device=logits.device))
    if mask:
        out["mask"] = torch.empty((T, E), dtype=torch.uint8, device=logits.device)
    if nu:
        out["nu"] = torch.empty((T,), dtype=torch.float32, device=logits.device)
    check(_lib.load().beam_softtopk_forward(_ptr(logits), T, E, int(top_k), ctypes.c_float(tau),
                                            _ptr(out["y"]), _ptr(out.get("mask")),
                                            _ptr(out.get("nu")),
                                            ctypes.c_void_p(_stream_handle(stream))))
    return out


def softtopk_backward(y: torch.Tensor, dy: torch.Tensor, tau: float, stream=None) -> torch.Tensor:
    """d logits [T][E] float32 for the upstream gradient dy [T][E] of SoftTopK's y (the
    relaxation's Jacobian through nu).  See beam_softtopk_backward."""
    for name, t in (("y", y), ("dy", dy)):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.float32 and t.dim() == 2
                and t.shape == y.shape):
            raise ValueError(f"{name} must be a contiguous [T][E] CUDA float32 tensor")
    T, E = y.shape
    dr = torch.empty_like(y)
    check(_lib.load().beam_softtopk_backward(_ptr(y), _ptr(dy), T, E, ctypes.c_float(tau),
                                             _ptr(dr), ctypes.c_void_p(_stream_handle(stream))))
    return dr
