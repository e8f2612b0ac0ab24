"""Plain fp64 CPU oracle of one MoE feed-forward layer with intra-expert
activation sparsity (TEST INFRASTRUCTURE: only tests/, the smoke check and
the benchmark's CPU-baseline leg use it; the product path never does).

What it computes, step by step, in float64 on the exact values the CUDA
path reads (bf16/fp32 storage values widened exactly):

1. Router [gist.science EN "Uncovering Intra-expert Activation Sparsity for
   Efficient Mixture-of-Expert Model Execution", Technical Summary >
   Methodology > System Implementation in vLLM: the router logic is kept
   as in the dense model]. Logits ``L = x W_router^T (+ bias)``, softmax
   over all experts, the top-k experts by probability (ties to the lower
   expert index), weights ``p_sel / sum(p_sel)`` when renormalising, else
   ``p_sel``.
2. SwiGLU intermediate per routed (token, expert) pair
   [mlsanity.com page, "Builds on": GLU Variants Improve Transformer]:
   ``g = x W_gate[e]^T``, ``u = x W_up[e]^T``, ``h = SiLU(g) * u`` with
   ``SiLU(g) = g / (1 + exp(-g))``.
3. Threshold mask [gist.science EN, Technical Summary > Methodology >
   System Implementation in vLLM > "Activation Masking": one pass, a
   threshold test per value, no sort]: neuron j is active iff its score
   exceeds tau, at or below tau is inactive. Two scores:
   ``score="h"``: the SwiGLU value, active iff ``|h_j| > tau``;
   ``score="gate"``: the pages' own system, where the dense gate projection
   alone produces the scores [same list, "Gate Projection"] and only the
   active neurons' up and down weights are read afterwards ["Fused Up-Down
   Projection"]: active iff ``|SiLU(g_j)| > tau``. In both modes an active
   neuron contributes its full ``h_j = SiLU(g_j) u_j``.
4. Down projection over the active neurons only [same list,
   "Fused Up-Down Projection"]: ``y = sum_{j active} h_j W_down[e][j, :]``,
   written as the product of the masked ``h`` with ``W_down[e]``: the
   inactive terms are exact zeros, so this is the same sum.
5. Combine: ``out[t] = sum_i w[t, i] y[t, i] + sum_s y_shared[s, t]``;
   shared experts are always active with weight 1 and their own threshold
   [gist.science EN, Technical Summary > Methodology > "Empirical
   Analysis": routed vs always-active shared experts].

Batching the tokens routed to one expert into one matrix product is the
same per-pair arithmetic done by a library matmul; no other reordering or
blocking is done.
"""

from __future__ import annotations

import dataclasses
import math
from fractions import Fraction
from typing import List, Optional

import numpy as np

try:  # weights may arrive as torch tensors (bf16 has no numpy dtype)
    import torch
except Exception:  # pragma: no cover
    torch = None


def _f64(a) -> np.ndarray:
    if torch is not None and isinstance(a, torch.Tensor):
        return a.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(a, dtype=np.float64)


@dataclasses.dataclass
class RouterResult:
    logits: np.ndarray     # [T][E] float64
    probs: np.ndarray      # [T][E] float64 softmax over all experts
    topk_idx: np.ndarray   # [T][k] int64, by decreasing probability
    topk_w: np.ndarray     # [T][k] float64 combine weights
    gap: np.ndarray        # [T] logit gap between k-th and (k+1)-th choice (inf if k == E)


@dataclasses.dataclass
class LayerResult:
    out: np.ndarray                  # [T][d] float64
    router: RouterResult
    h: np.ndarray                    # [T][k][F] float64 SwiGLU values of routed pairs
    active: np.ndarray               # [T][k][F] bool, score > tau
    h_shared: Optional[np.ndarray]   # [S][T][Fs] or None
    active_shared: Optional[np.ndarray]
    gate_abs: Optional[np.ndarray] = None         # [T][k][F] |SiLU(g)| of routed pairs
    gate_abs_shared: Optional[np.ndarray] = None  # [S][T][Fs]


def route(x, W_router, top_k: int, renormalize: bool, bias=None) -> RouterResult:
    """Step 1: logits, softmax over all experts, top-k, combine weights."""
    x = _f64(x)
    Wr = _f64(W_router)
    L = x @ Wr.T
    if bias is not None:
        L = L + _f64(bias)[None, :]
    m = L.max(axis=1, keepdims=True)
    ex = np.exp(L - m)
    p = ex / ex.sum(axis=1, keepdims=True)
    T, E = L.shape
    # stable sort of -p: equal probabilities keep increasing expert index
    order = np.argsort(-p, axis=1, kind="stable")
    idx = order[:, :top_k]
    p_sel = np.take_along_axis(p, idx, axis=1)
    w = p_sel / p_sel.sum(axis=1, keepdims=True) if renormalize else p_sel.copy()
    if top_k < E:
        Ls = np.take_along_axis(L, order, axis=1)
        gap = Ls[:, top_k - 1] - Ls[:, top_k]
    else:
        gap = np.full(T, np.inf)
    return RouterResult(L, p, idx.astype(np.int64), w, gap)


def swiglu_parts(x_rows, W_gate_e, W_up_e):
    """Step 2 in its two factors for rows of x, one expert:
    ``SiLU(x W_gate^T)`` and ``x W_up^T``."""
    xr = _f64(x_rows)
    g = xr @ _f64(W_gate_e).T
    u = xr @ _f64(W_up_e).T
    with np.errstate(over="ignore"):
        silu = g / (1.0 + np.exp(-g))
    return silu, u


def swiglu(x_rows, W_gate_e, W_up_e) -> np.ndarray:
    """Step 2: h = SiLU(x W_gate^T) * (x W_up^T) for rows of x, one expert."""
    silu, u = swiglu_parts(x_rows, W_gate_e, W_up_e)
    return silu * u


def active_mask(score: np.ndarray, tau: float) -> np.ndarray:
    """Step 3: active iff |score| > tau (at or below tau is inactive)."""
    return np.abs(score) > tau


def score_of(silu_g: np.ndarray, h: np.ndarray, score: str) -> np.ndarray:
    """The value whose magnitude step 3 compares with tau."""
    if score == "gate":
        return silu_g
    if score == "h":
        return h
    raise ValueError(f"score must be 'h' or 'gate', not {score!r}")


def down_projection(h: np.ndarray, active: np.ndarray, W_down_e) -> np.ndarray:
    """Step 4: sum over active neurons of h_j * W_down[j, :]."""
    return np.where(active, h, 0.0) @ _f64(W_down_e)


def layer_forward(x, W_router, W_gate, W_up, W_down, tau: float, top_k: int,
                  renormalize: bool, router_bias=None, Ws_gate=None, Ws_up=None,
                  Ws_down=None, tau_shared: float = 0.0, dense: bool = False,
                  score: str = "h") -> LayerResult:
    """Steps 1-5 for a batch x [T][d]. ``dense=True`` skips the threshold
    (every neuron active), the layer's dense reference; ``score`` picks the
    value compared with tau (step 3)."""
    x64 = _f64(x)
    T, d = x64.shape
    r = route(x64, W_router, top_k, renormalize, router_bias)
    E = r.logits.shape[1]
    F = W_gate.shape[1]
    h = np.zeros((T, top_k, F))
    gabs = np.zeros((T, top_k, F))
    act = np.zeros((T, top_k, F), dtype=bool)
    y = np.zeros((T, top_k, d))
    for e in range(E):
        tt, ii = np.nonzero(r.topk_idx == e)
        if tt.size == 0:
            continue
        sg, u = swiglu_parts(x64[tt], W_gate[e], W_up[e])
        he = sg * u
        ae = np.ones_like(he, dtype=bool) if dense else active_mask(score_of(sg, he, score), tau)
        h[tt, ii] = he
        gabs[tt, ii] = np.abs(sg)
        act[tt, ii] = ae
        y[tt, ii] = down_projection(he, ae, W_down[e])
    out = np.einsum("tk,tkd->td", r.topk_w, y)
    hs = acts = gs = None
    if Ws_gate is not None and Ws_gate.shape[0] > 0:
        S, Fs = Ws_gate.shape[0], Ws_gate.shape[1]
        hs = np.zeros((S, T, Fs))
        gs = np.zeros((S, T, Fs))
        acts = np.zeros((S, T, Fs), dtype=bool)
        for s in range(S):
            sg, u = swiglu_parts(x64, Ws_gate[s], Ws_up[s])
            hs[s] = sg * u
            gs[s] = np.abs(sg)
            acts[s] = np.ones_like(hs[s], dtype=bool) if dense else \
                active_mask(score_of(sg, hs[s], score), tau_shared)
            out = out + down_projection(hs[s], acts[s], Ws_down[s])
    return LayerResult(out, r, h, act, hs, acts, gabs, gs)


def calibrate_tau(abs_h, q: float, round_f32: bool = True) -> float:
    """Nearest-rank quantile of a pool of |h| values for target sparsity q.

    The pages speak of target sparsities without saying how the threshold
    is chosen [gist.science EN, Technical Summary > Results > "Accuracy
    Preservation"]; the plainest reading: sort the pool ascending into
    a[0..n-1] and take tau = a[ceil(q n) - 1], so that at least a fraction
    q of the values is at or below tau. q = 0 gives tau = 0. The result is
    rounded to float32, the precision the CUDA path compares in.
    """
    if q <= 0.0:
        return 0.0
    a = np.sort(np.asarray(abs_h, dtype=np.float64).ravel())
    n = a.size
    # exact rank: q is a decimal fraction, so q*n is taken in rationals
    # (0.7 * 10 in binary floating point is 7.000000000000001)
    qn = Fraction(str(q)) * n
    r = int(math.ceil(qn))
    r = min(max(r, 1), n)
    return float(np.float32(a[r - 1])) if round_f32 else float(a[r - 1])


def routed_abs_h(layer: LayerResult) -> np.ndarray:
    """The calibration pool: |h| over all routed (token, expert) pairs."""
    return np.abs(layer.h).ravel()


def shared_abs_h(layer: LayerResult) -> np.ndarray:
    return np.abs(layer.h_shared).ravel()


def routed_abs_gate(layer: LayerResult) -> np.ndarray:
    """The calibration pool of the gate score: |SiLU(g)| over routed pairs."""
    return layer.gate_abs.ravel()


def shared_abs_gate(layer: LayerResult) -> np.ndarray:
    return layer.gate_abs_shared.ravel()


def measured_sparsity(abs_h: np.ndarray, tau: float) -> float:
    a = np.asarray(abs_h).ravel()
    return float(np.count_nonzero(a <= tau)) / a.size


def pair_list(topk_idx: np.ndarray) -> List[tuple]:
    """Routed pairs in (token, choice) order."""
    T, k = topk_idx.shape
    return [(t, i) for t in range(T) for i in range(k)]
