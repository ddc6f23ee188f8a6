"""BEAM masked MoE-layer forward for NVIDIA B200 (sm_100a).

The compute path is the CUDA library libbeam_moe.so (C ABI in include/beam_moe.h); this package
is its Python binding.  There is no CPU fallback: importing `BeamMoE` and creating a layer
requires the built library and a CUDA device.
"""
from ._lib import (BEAM_MASK_OFF, BEAM_PATH_STREAM, BEAM_PATH_TENSOR, BeamError, LIB_PATH, load)
from .layer import BeamGenerator, BeamMoE, softtopk, softtopk_backward

__all__ = ["BeamMoE", "BeamGenerator", "softtopk", "softtopk_backward", "BeamError", "load", "LIB_PATH", "BEAM_MASK_OFF", "BEAM_PATH_STREAM",
           "BEAM_PATH_TENSOR"]
