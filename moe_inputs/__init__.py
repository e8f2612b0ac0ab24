"""Seeded synthetic inputs for the intra-expert sparse MoE layer.

This package only draws numbers: it holds none of the layer's arithmetic
(no routing, no SwiGLU, no threshold, no projection). Both the CUDA path
(through its tests and the benchmark) and the CPU oracle read what it
produces, so that the two sides see bit-identical inputs.
"""

from .generate import (  # noqa: F401
    LayerShape,
    LayerWeights,
    make_weights,
    make_tokens,
    round_to_storage,
    widen_f64,
)
from .workloads import WORKLOADS, Workload, get_workload  # noqa: F401
