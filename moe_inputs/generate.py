"""Counter-keyed Gaussian draws for MoE layer weights and tokens.

Recipe (stated once, used by every test, the benchmark and the oracle):

* Every tensor is drawn from its own numpy ``PCG64`` stream keyed by
  ``SeedSequence([seed, tag, index])``: ``tag`` names the tensor and
  ``index`` the expert (0 for tensors without an expert axis). Streams
  are independent, so experts are generated in parallel threads and a
  tensor does not depend on the draw order of the others.
* Values are ``standard_normal(dtype=float32)`` scaled by the tensor's
  standard deviation in float32. ``N(0, v)`` in a workload recipe means
  variance ``v``, so the scale is ``sqrt(v)`` rounded to float32.
* For bf16 workloads the float32 values are rounded to bf16 with
  round-to-nearest-even (``torch`` cast). The oracle reads those rounded
  values widened exactly to float64, so both sides see the same numbers.
* Tokens ``x`` come from the stream ``[seed, TAG_X, 0]`` drawn row-major,
  so a batch of ``T`` tokens is the first ``T`` rows of any longer batch
  with the same seed.
"""

from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np
import torch

TAG_ROUTER = 1
TAG_GATE = 2
TAG_UP = 3
TAG_DOWN = 4
TAG_BIAS = 5
TAG_SHARED_GATE = 6
TAG_SHARED_UP = 7
TAG_SHARED_DOWN = 8
TAG_X = 9

_STORAGE = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape and routing options of one MoE feed-forward layer."""

    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    renormalize: bool = True
    n_shared: int = 0
    d_ff_shared: int = 0
    dtype: str = "bf16"  # storage and arithmetic type of x / weights / out
    router_bias_var: float = 0.0  # 0: no router bias


@dataclasses.dataclass
class LayerWeights:
    """Weights in storage layout (CPU torch tensors, storage dtype).

    W_router [E][d]     logits = x @ W_router^T
    W_gate   [E][F][d]  row j: input weights of neuron j
    W_up     [E][F][d]
    W_down   [E][F][d]  row j: output vector of neuron j
    router_bias [E] float32 or None
    Ws_gate / Ws_up / Ws_down [S][Fs][d] for always-on shared experts, or None
    """

    shape: LayerShape
    W_router: torch.Tensor
    W_gate: torch.Tensor
    W_up: torch.Tensor
    W_down: torch.Tensor
    router_bias: Optional[torch.Tensor] = None
    Ws_gate: Optional[torch.Tensor] = None
    Ws_up: Optional[torch.Tensor] = None
    Ws_down: Optional[torch.Tensor] = None


def _stream(seed: int, tag: int, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tag, index])))


def _normal(seed: int, tag: int, index: int, shape, std: float) -> np.ndarray:
    a = _stream(seed, tag, index).standard_normal(shape, dtype=np.float32)
    a *= np.float32(std)
    return a


def round_to_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    """float32 array -> CPU tensor in the storage dtype (RNE for bf16)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(_STORAGE[dtype])


def widen_f64(t: torch.Tensor) -> np.ndarray:
    """Storage tensor -> float64 numpy array (exact widening)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def _per_expert(seed: int, tag: int, n: int, rows: int, cols: int, std: float,
                dtype: str, threads: int) -> torch.Tensor:
    out = torch.empty((n, rows, cols), dtype=_STORAGE[dtype])

    def one(e: int) -> None:
        out[e].copy_(round_to_storage(_normal(seed, tag, e, (rows, cols), std), dtype))

    if n == 0:
        return out
    with ThreadPoolExecutor(max_workers=max(1, min(threads, n))) as pool:
        list(pool.map(one, range(n)))
    return out


def make_weights(shape: LayerShape, seed: int, threads: int = 8) -> LayerWeights:
    """Draw all weights of a layer; W_router, W_gate, W_up ~ N(0, 1/d_model),
    W_down ~ N(0, 1/d_ff) (shared experts: N(0, 1/d_ff_shared)),
    router bias ~ N(0, router_bias_var)."""
    d, E, F = shape.d_model, shape.n_experts, shape.d_ff
    s_in = 1.0 / math.sqrt(d)
    Wr = round_to_storage(_normal(seed, TAG_ROUTER, 0, (E, d), s_in), shape.dtype)
    Wg = _per_expert(seed, TAG_GATE, E, F, d, s_in, shape.dtype, threads)
    Wu = _per_expert(seed, TAG_UP, E, F, d, s_in, shape.dtype, threads)
    Wd = _per_expert(seed, TAG_DOWN, E, F, d, 1.0 / math.sqrt(F), shape.dtype, threads)
    bias = None
    if shape.router_bias_var > 0:
        bias = torch.from_numpy(_normal(seed, TAG_BIAS, 0, (E,), math.sqrt(shape.router_bias_var)))
    w = LayerWeights(shape, Wr, Wg, Wu, Wd, bias)
    if shape.n_shared > 0:
        S, Fs = shape.n_shared, shape.d_ff_shared
        w.Ws_gate = _per_expert(seed, TAG_SHARED_GATE, S, Fs, d, s_in, shape.dtype, threads)
        w.Ws_up = _per_expert(seed, TAG_SHARED_UP, S, Fs, d, s_in, shape.dtype, threads)
        w.Ws_down = _per_expert(seed, TAG_SHARED_DOWN, S, Fs, d, 1.0 / math.sqrt(Fs),
                                shape.dtype, threads)
    return w


def make_tokens(d_model: int, T: int, seed: int, dtype: str) -> torch.Tensor:
    """x ~ N(0, 1), [T][d_model]; the first rows do not depend on T."""
    return round_to_storage(_normal(seed, TAG_X, 0, (T, d_model), 1.0), dtype)
