"""d_ff (tensor-parallel) sharding of the layer over a torch.distributed group.

Every expert's neurons are split evenly across the n ranks of the group:
rank r holds rows [r F/n, (r+1) F/n) of W_gate, W_up and W_down of every
routed expert (and the same share of each shared expert), and the router is
replicated. The activation threshold is applied per neuron and the combine is
linear in the neurons' contributions, so the layer run over a rank's own
neurons gives an exact partial output, and one sum all-reduce over the group
gives the layer's output. The routing is computed identically on every rank
from the replicated router. (The pages state only that the method keeps the
serving system's parallelism working [gist.science EN "Uncovering
Intra-expert Activation Sparsity for Efficient Mixture-of-Expert Model
Execution", Technical Summary > Methodology > System Implementation in
vLLM]; this split is the standard tensor-parallel split of an FFN.)

The per-rank layer is the C-ABI library's; the all-reduce is the process
group's (NCCL over NVLink on GPUs). With the default fp32 reduction each
rank's layer writes its partial output in fp32 straight from the combine's
sums (desc.out_f32, no rounding), the all-reduce adds the partials in fp32,
and the sum is rounded to the layer's dtype once. With another reduce_dtype
the partials are written in the layer's dtype and reduced in reduce_dtype:
two roundings.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist

from .layer import MoESparseLayer


def shard_rows(W: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Rank `rank`'s rows of a [n_experts][d_ff][d_model] weight, contiguous."""
    if W.dim() != 3:
        raise ValueError("expected a [n_experts][d_ff][d_model] weight")
    F = W.shape[1]
    if F % world:
        raise ValueError(f"d_ff = {F} is not divisible by the group size {world}")
    f = F // world
    return W[:, rank * f:(rank + 1) * f, :].contiguous()


class DffShardedLayer:
    """The layer with each expert's d_ff split over a process group.

    Construct on every rank of `group` (default: the world); give `forward`
    this rank's weight shards (`shard`) and the replicated router. Returns
    the full [T][d_model] output on every rank.
    """

    def __init__(self, d_model: int, d_ff: int, n_experts: int, top_k_max: int,
                 max_tokens: int, *, n_shared: int = 0, d_ff_shared: int = 0, group=None,
                 reduce_dtype: torch.dtype = torch.float32,
                 layer_factory: Optional[Callable[..., object]] = None, **layer_kw):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if d_ff % self.world or (n_shared and d_ff_shared % self.world):
            raise ValueError("d_ff (and d_ff_shared) must be divisible by the group size")
        self.reduce_dtype = reduce_dtype
        if reduce_dtype == torch.float32:
            layer_kw.setdefault("out_f32", True)  # partials leave the layer unrounded
        factory = layer_factory or MoESparseLayer
        self.layer = factory(d_model, d_ff // self.world, n_experts, top_k_max, max_tokens,
                             n_shared=n_shared,
                             d_ff_shared=d_ff_shared // self.world if n_shared else 0,
                             **layer_kw)
        # the dtype of the returned output: the layer's own (bf16 / fp32), or
        # that of the partials for a layer without one
        self.result_dtype = getattr(self.layer, "torch_dtype", None)

    def shard(self, W: torch.Tensor) -> torch.Tensor:
        """This rank's rows of a full [experts][d_ff][d_model] weight."""
        return shard_rows(W, self.rank, self.world)

    def set_shared(self, Wg_s: torch.Tensor, Wu_s: torch.Tensor, Wd_s: torch.Tensor,
                   tau_shared: float) -> None:
        """This rank's shards of the shared experts' weights."""
        self.layer.set_shared(Wg_s, Wu_s, Wd_s, tau_shared)

    def forward(self, x: torch.Tensor, W_router: torch.Tensor, W_gate: torch.Tensor,
                W_up: torch.Tensor, W_down: torch.Tensor, tau: float, top_k: int,
                router_bias: Optional[torch.Tensor] = None) -> torch.Tensor:
        part = self.layer.forward(x, W_router, W_gate, W_up, W_down, tau, top_k,
                                  router_bias=router_bias)
        final = self.result_dtype or part.dtype
        if self.world == 1:
            return part.to(final)
        acc = part.to(self.reduce_dtype)
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=self.group)
        return acc.to(final)
