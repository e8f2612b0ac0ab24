"""The synthetic workloads the layer is tested and measured on.

Each entry fixes the layer shape, the seeds, the token counts and the
target sparsities at which the threshold ``tau`` is calibrated. The taus
themselves are computed by the CPU oracle and stored as data next to the
tests (``tests/golden/tau_calibration.json``); this module only names the
workloads.

The pages measured trained MoE models on public accuracy benchmarks; no
weights or datasets are available here, so i.i.d. Gaussian layers of the
named shapes stand in for them and reproduce only the shapes and the
target sparsities.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

from .generate import LayerShape


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    weight_seed: int
    token_seed: int
    tokens: Tuple[int, ...]          # batch sizes T run on this layer
    sparsities: Tuple[float, ...]    # target fractions of inactive neurons
    calib_seed: int                  # seed of the calibration batch
    calib_tokens: int                # size of the calibration batch
    description: str


WORKLOADS: Dict[str, Workload] = {
    "tiny_f32": Workload(
        name="tiny_f32",
        shape=LayerShape(d_model=256, n_experts=8, top_k=2, d_ff=512, renormalize=True,
                         dtype="f32"),
        weight_seed=0, token_seed=0, tokens=(16,), sparsities=(0.7,),
        calib_seed=0, calib_tokens=16,
        description="tiny fp32 layer: T=16, d=256, E=8, top-2 renormalised, d_ff=512; "
                    "tau = 0.7 quantile of |h| over the batch's routed pairs",
    ),
    "mixtral_decode": Workload(
        name="mixtral_decode",
        shape=LayerShape(d_model=4096, n_experts=8, top_k=2, d_ff=14336, renormalize=True,
                         dtype="bf16"),
        weight_seed=1, token_seed=1, tokens=(1, 8, 32, 64), sparsities=(0.7,),
        calib_seed=0, calib_tokens=256,
        description="Mixtral-8x7B-shaped layer, bf16: d=4096, E=8, top-2 renormalised, "
                    "d_ff=14336, decode T in {1,8,32,64}; tau from a 256-token seed-0 "
                    "calibration batch at 70% sparsity",
    ),
    "many_small_experts": Workload(
        name="many_small_experts",
        shape=LayerShape(d_model=2048, n_experts=128, top_k=8, d_ff=768, renormalize=True,
                         dtype="bf16", router_bias_var=0.5),
        weight_seed=2, token_seed=2, tokens=(256,), sparsities=(0.8,),
        calib_seed=2, calib_tokens=256,
        description="128 experts top-8 renormalised, d=2048, d_ff=768, T=256, bf16; "
                    "router bias ~N(0, var 0.5) for skewed load; 80% sparsity",
    ),
    "shared_routed_prefill": Workload(
        name="shared_routed_prefill",
        shape=LayerShape(d_model=2048, n_experts=64, top_k=6, d_ff=1408, renormalize=False,
                         n_shared=2, d_ff_shared=1408, dtype="bf16"),
        weight_seed=3, token_seed=3, tokens=(4096,), sparsities=(0.6,),
        calib_seed=3, calib_tokens=4096,
        description="64 routed experts top-6 (softmax weights, no renormalisation) plus 2 "
                    "always-on shared experts, d=2048, d_ff=1408, prefill T=4096, bf16; "
                    "separate taus for routed and shared experts at 60% sparsity",
    ),
    "mixtral_sweep": Workload(
        name="mixtral_sweep",
        shape=LayerShape(d_model=4096, n_experts=8, top_k=2, d_ff=14336, renormalize=True,
                         dtype="bf16"),
        weight_seed=4, token_seed=4, tokens=(1, 16, 128, 512), sparsities=(0.0, 0.5, 0.7, 0.9),
        calib_seed=4, calib_tokens=512,
        description="sparsity sweep on the Mixtral-8x7B shape, bf16: tau at "
                    "{0,50,70,90}% calibrated on the T=512 batch, run at T in {1,16,128,512} "
                    "(prefixes of that batch)",
    ),
}


def get_workload(name: str) -> Workload:
    return WORKLOADS[name]
