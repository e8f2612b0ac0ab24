"""B200 (sm_100a) Mixture-of-Experts feed-forward layer that skips the
computation of inactive neurons inside each routed expert.

The layer is the C-ABI library ``libmoe_sparse.so`` (include/moe_sparse.h);
this package holds its CUDA sources (``csrc/``), the build step and a thin
Python binding.
"""

from ._lib import LIB_PATH, PATHS, STAGES, MoEError, load  # noqa: F401
from .layer import MoESparseLayer  # noqa: F401
from .sharded import DffShardedLayer, shard_rows  # noqa: F401
