"""Seeded synthetic inputs for the MoE-layer forward.

This package only draws input tensors (activations, router weights, expert
weights, the per-expert logit offset that skews the routing) for the named
workloads.  It holds none of the layer's arithmetic, so both the CUDA path and
the fp64 oracle can be fed from it without sharing any computation.
"""
from .gen import CONFIGS, MoEShape, make_inputs, make_router_logits, shape_of  # noqa: F401
