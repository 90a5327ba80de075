"""Seeded synthetic DiT attention-layer inputs.

This package only draws numbers: Q/K/V tensors of a video / 3D diffusion
transformer attention layer, their per-step drift, and the workload shapes.
It holds none of the sparse-attention method's arithmetic, so that both the
fp64 oracle and the CUDA path can take their inputs from it without sharing
any other code.
"""
from .workloads import WORKLOADS, Workload, workload, sweep_points
from .dit_inputs import (
    bf16_round,
    head_tensors,
    layer_tensors,
    drift_head,
    drift_layer,
    random_blocks_head,
    random_metadata_head,
    random_qkv,
    rising_qkv,
)

__all__ = [
    "WORKLOADS", "Workload", "workload", "sweep_points",
    "bf16_round", "head_tensors", "layer_tensors", "drift_head", "drift_layer",
    "random_blocks_head", "random_metadata_head", "random_qkv", "rising_qkv",
]
