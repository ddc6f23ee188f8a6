"""Seeded synthetic inputs (token batches and layer weights) for tests and the bench.

Shared by both sides of every parity check: the CPU oracle and the CUDA library receive the
same tensors from here.  Nothing in this package computes any part of the MoE layer.
"""
from .layers import (LayerSpec, SPECS, make_layer, make_tokens, make_router, make_experts,
                     make_generator, mask_bias_for_keep_rate)

__all__ = ["LayerSpec", "SPECS", "make_layer", "make_tokens", "make_router", "make_experts",
           "make_generator", "mask_bias_for_keep_rate"]
