"""Seeded synthetic inputs for the Dust estimator workloads.

This module generates inputs only (activations, weights, targets) and holds
none of the estimator's arithmetic. Both the CPU oracle tests and the CUDA
path read the same arrays from here; the noise the method draws is not
generated here (each side has its own counter-based generator).
"""
from .workloads import (  # noqa: F401
    CONFIGS,
    Workload,
    bf16_round,
    make_head_inputs,
    make_attn_inputs,
    make_mlp_inputs,
    zipf_targets,
)
