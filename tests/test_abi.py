"""The C ABI on a machine without a GPU: the library loads, exports every declared entry point,
and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "beam_moe.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(beam_(?:moe|gen)_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from dynamic_expert_routing_b200 import build, _lib
    build.build()
    return _lib.load()


def test_header_declares_the_named_calls():
    names = _declared_functions()
    for n in ("beam_moe_create", "beam_moe_forward", "beam_moe_stats", "beam_gen_create",
              "beam_gen_route", "beam_moe_forward_routed"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), f"{n} not exported"


def test_invalid_config_is_rejected_without_cuda(lib):
    from dynamic_expert_routing_b200._lib import BeamConfig, BeamWeights, BEAM_ERR_INVALID_ARG
    w = BeamWeights(*([ctypes.c_void_p(16)] * 5 + [None] * 3))
    h = ctypes.c_void_p()
    bad = [
        BeamConfig(100, 8, 2, 512, 0, 0, 1, 0, 64),     # d_model not a multiple of 64 (bf16)
        BeamConfig(256, 0, 2, 512, 0, 0, 1, 0, 64),     # no experts
        BeamConfig(256, 8, 9, 512, 0, 0, 1, 0, 64),     # K > E
        BeamConfig(256, 8, 2, 500, 0, 0, 1, 0, 64),     # F not a multiple of 128
        BeamConfig(256, 8, 2, 512, 1, 0, 1, 0, 64),     # shared expert without a size
        BeamConfig(256, 8, 2, 512, 0, 0, 7, 0, 64),     # unknown dtype
        BeamConfig(256, 8, 2, 512, 0, 0, 1, 0, 0),      # max_tokens 0
        BeamConfig(256, 300, 2, 512, 0, 0, 1, 0, 64),   # too many experts
    ]
    for cfg in bad:
        st = lib.beam_moe_create(ctypes.byref(cfg), ctypes.byref(w), None, ctypes.byref(h))
        assert st == BEAM_ERR_INVALID_ARG
        assert lib.beam_moe_last_error()
        assert not h.value


def test_null_handle_calls(lib):
    from dynamic_expert_routing_b200._lib import BeamStats, BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_forward(None, None, 1, None, 0, None) == BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_forward_host(None, None, 1, None, 0, None) == BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_host_wait(None) == BEAM_ERR_INVALID_ARG
    s = BeamStats()
    assert lib.beam_moe_stats(None, ctypes.byref(s), None) == BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_get_routing(None, None, None, None, None, None, None, None) == BEAM_ERR_INVALID_ARG
    lib.beam_moe_destroy(None)
    assert lib.beam_moe_wait_selftest(0, None) == BEAM_ERR_INVALID_ARG
    assert b"sm_100a" in lib.beam_moe_version()


def test_invalid_generator_config_is_rejected_without_cuda(lib):
    from dynamic_expert_routing_b200._lib import BeamGenConfig, BEAM_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    w = ctypes.c_void_p(16)
    bad = [
        BeamGenConfig(100, 4, 8, 2, 1, 0, 64),     # d_model not a multiple of 64 (bf16)
        BeamGenConfig(256, 0, 8, 2, 1, 0, 64),     # no layers
        BeamGenConfig(256, 513, 8, 2, 1, 0, 64),   # too many layers
        BeamGenConfig(256, 4, 0, 2, 1, 0, 64),     # no experts
        BeamGenConfig(256, 4, 8, 9, 1, 0, 64),     # K > E
        BeamGenConfig(256, 4, 8, 2, 7, 0, 64),     # unknown dtype
        BeamGenConfig(256, 4, 8, 2, 1, -1, 64),    # negative segment length
        BeamGenConfig(256, 4, 8, 2, 1, 0, 0),      # max_tokens 0
    ]
    for cfg in bad:
        assert lib.beam_gen_create(ctypes.byref(cfg), w, w, None, ctypes.byref(h)) == BEAM_ERR_INVALID_ARG
        assert lib.beam_moe_last_error()
        assert not h.value
    good = BeamGenConfig(256, 4, 8, 2, 1, 0, 64)
    assert lib.beam_gen_create(ctypes.byref(good), None, w, None, ctypes.byref(h)) == BEAM_ERR_INVALID_ARG
    assert lib.beam_gen_create(ctypes.byref(good), w, w, None, None) == BEAM_ERR_INVALID_ARG


def test_generator_and_routed_forward_null_handles(lib):
    from dynamic_expert_routing_b200._lib import BeamRouting, BEAM_ERR_INVALID_ARG
    r = BeamRouting()
    assert lib.beam_gen_route(None, None, 1, ctypes.byref(r), 0, None) == BEAM_ERR_INVALID_ARG
    assert lib.beam_gen_sync(None) == BEAM_ERR_INVALID_ARG
    lib.beam_gen_destroy(None)
    assert lib.beam_moe_forward_routed(None, None, 1, ctypes.byref(r), None, 0, None) == BEAM_ERR_INVALID_ARG


def test_routing_gradient_null_handle(lib):
    from dynamic_expert_routing_b200._lib import BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_backward_router(None, None, None, 1, ctypes.c_float(0.0), None, None,
                                        None, None, None, None, None) == BEAM_ERR_INVALID_ARG
    assert lib.beam_moe_last_error()


def test_stage_table_matches_the_header(lib):
    from dynamic_expert_routing_b200 import _lib
    names = [lib.beam_moe_stage_name(i).decode() for i in range(_lib.BEAM_N_STAGES)]
    assert all(names) and len(set(names)) == len(names)
    assert lib.beam_moe_stage_name(_lib.BEAM_N_STAGES) == b""
    assert names[-4:] == ["fused_decode", "route_grad", "route_dw", "chunk_stats"]
    assert "swiglu_finish" not in names and "shared_swiglu_finish" not in names


def test_missing_library_fails_loudly(tmp_path):
    from dynamic_expert_routing_b200 import _lib
    with pytest.raises(RuntimeError):
        _lib._lib = None
        try:
            _lib.load(str(tmp_path / "nope.so"))
        finally:
            _lib._lib = None


def test_binding_constants_match_the_header():
    """Every flag, status code, dtype and size the header defines has the same value in the
    binding, so a flag added on one side only fails here."""
    from dynamic_expert_routing_b200 import _lib
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    found = {}
    for name, val, shift in re.findall(r"#define\s+(BEAM_[A-Z0-9_]+)\s+\(?(0x[0-9a-fA-F]+|\d+)u?(?:\s*<<\s*(\d+))?", text):
        found[name] = int(val, 0) << (int(shift) if shift else 0)
    for name, val in re.findall(r"\b(BEAM_[A-Z0-9_]+)\s*=\s*(\d+)", text):
        found[name] = int(val)
    found.pop("BEAM_MOE_H", None)
    assert len(found) >= 20
    for name, val in found.items():
        assert getattr(_lib, name) == val, name


def test_output_dtype_flag_of_the_binding():
    """forward(out=...) takes a CUDA float32 or bfloat16 tensor of at least T*D values and sets
    BEAM_Y_BF16 for bfloat16; anything else is refused before the library is called."""
    import torch
    from dynamic_expert_routing_b200.layer import _y_flag
    with pytest.raises(ValueError):
        _y_flag(torch.empty((4, 8)), 4, 8)                       # host memory
    with pytest.raises(ValueError):
        _y_flag(torch.empty((4, 8), dtype=torch.float16), 4, 8)  # neither float32 nor bf16
