"""Seeded synthetic inputs shared by the tests, the bench and the oracle.

This package only draws random numbers and describes workload shapes.  It
holds none of the method's arithmetic (no rotation, no norm, no
quantisation), so importing it from both the CUDA side and the CPU oracle
does not couple the two.
"""
from .synthetic import (  # noqa: F401
    WORKLOADS,
    Workload,
    Linear,
    activations,
    weight,
    norm_weight,
    outlier_channels,
    workload_inputs,
    mlp_weights,
)
