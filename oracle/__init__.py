"""CPU oracle for the intra-expert sparse MoE layer (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the C-ABI library
and its Python binding) never imports, links or calls it, and it imports
nothing from the product package.
"""

from .moe_oracle import (  # noqa: F401
    RouterResult,
    LayerResult,
    route,
    swiglu,
    active_mask,
    down_projection,
    layer_forward,
    calibrate_tau,
)
