"""ctypes declarations of the C ABI in include/beam_moe.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libbeam_moe.so")

BEAM_OK = 0
BEAM_ERR_INVALID_ARG = 1
BEAM_ERR_OOM = 2
BEAM_ERR_CUDA = 3
BEAM_ERR_UNSUPPORTED = 4
BEAM_ERR_TIMEOUT = 5
BEAM_ERR_NO_FORWARD = 6
BEAM_ERR_RANGE = 7

BEAM_DTYPE_F32 = 0
BEAM_DTYPE_BF16 = 1

BEAM_MASK_OFF = 0x1
BEAM_PATH_STREAM = 0x2
BEAM_PATH_TENSOR = 0x4
BEAM_NO_GRAPH = 0x8
BEAM_FUSED_DECODE = 0x10
BEAM_TRAIN = 0x20
BEAM_HOST_PIPELINE = 0x40
BEAM_HOST_Y_BF16 = 0x80
BEAM_HOST_ASYNC = 0x100
BEAM_Y_BF16 = 0x200

BEAM_N_STAGES = 17
BEAM_ROUTE_NOALLOC_SCRATCH_BYTES = 2 << 20

STATUS_NAMES = {0: "BEAM_OK", 1: "BEAM_ERR_INVALID_ARG", 2: "BEAM_ERR_OOM", 3: "BEAM_ERR_CUDA",
                4: "BEAM_ERR_UNSUPPORTED", 5: "BEAM_ERR_TIMEOUT", 6: "BEAM_ERR_NO_FORWARD",
                7: "BEAM_ERR_RANGE"}


class BeamConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("segment_len", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32)]


class BeamWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_router", "w_mask", "w_gate", "w_up", "w_down",
                                               "ws_gate", "ws_up", "ws_down")]


class BeamStats(ctypes.Structure):
    _fields_ = [("avg_k", ctypes.c_double), ("l_reg", ctypes.c_double),
                ("n_active_experts", ctypes.c_int32), ("n_tokens_all_masked", ctypes.c_int32),
                ("tokens", ctypes.c_int32), ("n_kept", ctypes.c_int32)]


class BeamGenConfig(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("n_layers", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("segment_len", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32)]


class BeamRouting(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("topk_id", "gate", "mask_logit", "keep", "ghat",
                                               "n_keep", "lreg", "active")]


class BeamError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library; there is no fallback, a missing build is an error."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m dynamic_expert_routing_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    P, I, U = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32
    lib.beam_moe_create.argtypes = [ctypes.POINTER(BeamConfig), ctypes.POINTER(BeamWeights), P,
                                    ctypes.POINTER(P)]
    lib.beam_moe_forward.argtypes = [P, P, I, P, U, P]
    lib.beam_moe_forward_host.argtypes = [P, P, I, P, U, P]
    lib.beam_moe_stats.argtypes = [P, ctypes.POINTER(BeamStats), P]
    lib.beam_moe_host_wait.argtypes = [P]
    lib.beam_moe_host_wait.restype = ctypes.c_int
    lib.beam_moe_get_routing.argtypes = [P, P, P, P, P, P, P, P]
    lib.beam_moe_route_noalloc.argtypes = [P, P, I, P, P, P, P, P, U, P]
    lib.beam_moe_route_noalloc.restype = ctypes.c_int
    lib.beam_moe_wait_selftest.argtypes = [I, P]
    lib.beam_moe_wait_selftest.restype = ctypes.c_int
    lib.beam_moe_profile_begin.argtypes = [P, I]
    lib.beam_moe_profile_end.argtypes = [P, P, P, P]
    lib.beam_moe_stage_name.argtypes = [I]
    lib.beam_moe_stage_name.restype = ctypes.c_char_p
    lib.beam_moe_launch_count.argtypes = [P]
    lib.beam_moe_launch_count.restype = ctypes.c_int64
    lib.beam_gen_create.argtypes = [ctypes.POINTER(BeamGenConfig), P, P, P, ctypes.POINTER(P)]
    lib.beam_gen_route.argtypes = [P, P, I, ctypes.POINTER(BeamRouting), U, P]
    lib.beam_gen_sync.argtypes = [P]
    lib.beam_gen_destroy.argtypes = [P]
    lib.beam_gen_destroy.restype = None
    lib.beam_moe_forward_routed.argtypes = [P, P, I, ctypes.POINTER(BeamRouting), P, U, P]
    lib.beam_moe_backward_router.argtypes = [P, P, P, I, ctypes.c_float, P, P, P, P, P, P, P]
    lib.beam_softtopk_forward.argtypes = [P, I, I, I, ctypes.c_float, P, P, P, P]
    lib.beam_softtopk_backward.argtypes = [P, P, I, I, ctypes.c_float, P, P]
    lib.beam_softtopk_forward.restype = ctypes.c_int
    lib.beam_softtopk_backward.restype = ctypes.c_int
    lib.beam_moe_create_ep.argtypes = [ctypes.POINTER(BeamConfig), ctypes.POINTER(BeamWeights), P,
                                       ctypes.POINTER(P)]
    lib.beam_moe_ep_dispatch.argtypes = [P, P, I, U, P, P, P]
    lib.beam_moe_ep_combine.argtypes = [P, P, P, P]
    lib.beam_ep_expert_range.argtypes = [I, I, I, ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.beam_ep_recv_routing.argtypes = [P, I, I, I, P, P, P, P, P, P]
    for f in (lib.beam_moe_create_ep, lib.beam_moe_ep_dispatch, lib.beam_moe_ep_combine,
              lib.beam_ep_expert_range, lib.beam_ep_recv_routing):
        f.restype = ctypes.c_int
    lib.beam_moe_destroy.argtypes = [P]
    lib.beam_moe_destroy.restype = None
    lib.beam_moe_last_error.restype = ctypes.c_char_p
    lib.beam_moe_version.restype = ctypes.c_char_p
    for f in (lib.beam_moe_create, lib.beam_moe_forward, lib.beam_moe_forward_host,
              lib.beam_moe_stats, lib.beam_moe_get_routing, lib.beam_moe_profile_begin,
              lib.beam_moe_profile_end, lib.beam_gen_create, lib.beam_gen_route,
              lib.beam_gen_sync, lib.beam_moe_forward_routed, lib.beam_moe_backward_router):
        f.restype = ctypes.c_int
    _lib = lib
    return lib


def check(status: int) -> None:
    if status != BEAM_OK:
        msg = load().beam_moe_last_error().decode(errors="replace")
        raise BeamError(status, msg)
