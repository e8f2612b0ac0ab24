"""Shared parity machinery for the GPU tests: run the layer through the C ABI
and the CPU oracle on the same seeded inputs and compare.

Criteria (fixed by the layer's specification, written here once):
  * routing indices bit-exact, except tokens whose k-th / (k+1)-th logit gap
    is within 1e-6 of the token's largest |logit| (fp32 vs fp64 may order
    them differently; such tokens are reported and left out);
  * active-neuron sets bit-exact, except neurons with ||h_ref| - tau| <=
    1e-3 tau (the comparison runs on fp32 h on the GPU, fp64 in the oracle);
  * relative Frobenius error of the output <= 1e-5 (fp32) or 2e-2 (bf16).
"""

from __future__ import annotations

import json
import os
from typing import Optional

import numpy as np
import torch

from moe_inputs import LayerShape, LayerWeights, make_tokens, make_weights
from oracle import moe_oracle as om
from intra_expert_activation_b200 import MoESparseLayer

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = {"f32": 1e-5, "bf16": 2e-2}
GAP_REL = 1e-6
BAND_REL = 1e-3

with open(os.path.join(GOLDEN, "tau_calibration.json")) as _f:
    TAUS = json.load(_f)


def tau_of(workload: str, q: float, score: str = "h"):
    e = TAUS[workload]["taus_gate" if score == "gate" else "taus"][f"{q:.2f}"]
    return e["tau"], e.get("tau_shared", 0.0)


class DeviceWeights:
    def __init__(self, w: LayerWeights, device="cuda"):
        self.host = w
        self.shape = w.shape
        mv = lambda t: None if t is None else t.to(device).contiguous()
        self.W_router = mv(w.W_router)
        self.W_gate = mv(w.W_gate)
        self.W_up = mv(w.W_up)
        self.W_down = mv(w.W_down)
        self.bias = mv(w.router_bias)
        self.Ws_gate = mv(w.Ws_gate)
        self.Ws_up = mv(w.Ws_up)
        self.Ws_down = mv(w.Ws_down)


def make_layer(shape: LayerShape, max_tokens: int, path="auto", debug=True, **kw):
    return MoESparseLayer(shape.d_model, shape.d_ff, shape.n_experts, shape.top_k, max_tokens,
                          renormalize=shape.renormalize, n_shared=shape.n_shared,
                          d_ff_shared=shape.d_ff_shared, dtype=shape.dtype, path=path,
                          debug=debug, **kw)


def run_gpu(layer: MoESparseLayer, dw: DeviceWeights, x: torch.Tensor, tau: float,
            tau_shared: float = 0.0, top_k: Optional[int] = None):
    sh = dw.shape
    if sh.n_shared:
        layer.set_shared(dw.Ws_gate, dw.Ws_up, dw.Ws_down, tau_shared)
    xd = x.to("cuda").contiguous()
    out = layer.forward(xd, dw.W_router, dw.W_gate, dw.W_up, dw.W_down, tau,
                        top_k or sh.top_k, router_bias=dw.bias)
    dbg = layer.debug()
    torch.cuda.synchronize()
    res = {"out": out.to(torch.float64).cpu().numpy()}
    for k, v in dbg.items():
        res[k] = v.cpu().numpy()
    res["stats"] = layer.stats()
    return res


def unpack_bits(words: np.ndarray, F: int) -> np.ndarray:
    w = words.astype(np.uint32)
    bits = (w[..., None] >> np.arange(32, dtype=np.uint32)) & 1
    return bits.reshape(*w.shape[:-1], -1)[..., :F].astype(bool)


def oracle_forward(dw: DeviceWeights, x: torch.Tensor, tau: float, tau_shared: float = 0.0,
                   dense: bool = False, top_k: Optional[int] = None, score: str = "h"):
    w = dw.host
    sh = dw.shape
    return om.layer_forward(x, w.W_router, w.W_gate, w.W_up, w.W_down, tau, top_k or sh.top_k,
                            sh.renormalize, router_bias=w.router_bias, Ws_gate=w.Ws_gate,
                            Ws_up=w.Ws_up, Ws_down=w.Ws_down, tau_shared=tau_shared,
                            dense=dense, score=score)


def _band_corrected(ref, dw, gpu_act, gpu_act_shared, tau, tau_shared, ok_tok):
    """The oracle output with the GPU's decisions for neurons inside the band.

    Inside the band both decisions are correct; the reference output is the
    oracle's sum with each such neuron's term added or removed as the GPU
    decided: delta = (gpu_active - ref_active) * w * h_j * W_down[e][j, :].
    """
    out = ref.out.copy()
    w = dw.host
    r = ref.router
    T, k, F = ref.h.shape
    if gpu_act is not None:
        flips = np.argwhere((gpu_act != ref.active) & ok_tok[:, None, None])
        for t, i, j in flips:
            e = int(r.topk_idx[t, i])
            sign = 1.0 if gpu_act[t, i, j] else -1.0
            row = w.W_down[e, j].to(torch.float64).numpy()
            out[t] += sign * r.topk_w[t, i] * ref.h[t, i, j] * row
    if gpu_act_shared is not None and ref.h_shared is not None:
        for s, t, j in np.argwhere(gpu_act_shared != ref.active_shared):
            sign = 1.0 if gpu_act_shared[s, t, j] else -1.0
            row = w.Ws_down[s, j].to(torch.float64).numpy()
            out[t] += sign * ref.h_shared[s, t, j] * row
    return out


def compare(gpu: dict, ref, tau: float, tau_shared: float, dtype: str, dw=None,
            check_active=True, dense=False, score: str = "h") -> dict:
    """Assert the parity criteria; return the measured errors. The band is
    taken on the score the mask used: |h|, or |SiLU(g)| for the gate score."""
    r = ref.router
    T, k = r.topk_idx.shape
    Lmax = np.abs(r.logits).max(axis=1)
    ambiguous = r.gap <= GAP_REL * np.maximum(Lmax, 1e-30)
    ok_tok = ~ambiguous
    gi = gpu["topk_idx"].astype(np.int64)
    assert np.array_equal(gi[ok_tok], r.topk_idx[ok_tok]), "routing indices differ"
    np.testing.assert_allclose(gpu["topk_w"][ok_tok], r.topk_w[ok_tok], rtol=2e-5, atol=1e-7)
    info = {"tokens": T, "ambiguous_tokens": int(ambiguous.sum())}
    assert ambiguous.mean() <= 0.01

    ga = gs = None
    if check_active and "active_bits" in gpu:
        F = ref.h.shape[2]
        ga = unpack_bits(gpu["active_bits"], F).reshape(T, k, F)
        diff = ga[ok_tok] != ref.active[ok_tok]
        if dense:
            assert ga[ok_tok].all(), "dense path must keep every neuron"
        else:
            sc = ref.gate_abs if score == "gate" else np.abs(ref.h)
            band = np.abs(sc[ok_tok] - tau) <= BAND_REL * tau
            bad = diff & ~band
            assert not bad.any(), f"{int(bad.sum())} active-set mismatches outside the band"
        info["active_mismatch_in_band"] = int(diff.sum())
        if ref.h_shared is not None and "active_bits_shared" in gpu:
            Fs = ref.h_shared.shape[2]
            gs = unpack_bits(gpu["active_bits_shared"], Fs)
            ds = gs != ref.active_shared
            if dense:
                assert gs.all(), "dense path must keep every shared neuron"
            else:
                scs = ref.gate_abs_shared if score == "gate" else np.abs(ref.h_shared)
                bs = np.abs(scs - tau_shared) <= BAND_REL * tau_shared
                assert not (ds & ~bs).any(), "shared active-set mismatch outside the band"
            info["shared_mismatch_in_band"] = int(ds.sum())

    out_ref = ref.out
    if dw is not None and (info.get("active_mismatch_in_band", 0) or
                           info.get("shared_mismatch_in_band", 0)):
        out_ref = _band_corrected(ref, dw, ga, gs, tau, tau_shared, ok_tok)
    out_ref = out_ref[ok_tok]
    err = np.linalg.norm(gpu["out"][ok_tok] - out_ref) / max(np.linalg.norm(out_ref), 1e-300)
    info["rel_frobenius"] = float(err)
    assert err <= TOL[dtype], f"relative Frobenius error {err:.3e} > {TOL[dtype]:.0e} ({info})"
    return info


def workload_weights(name: str):
    from moe_inputs import WORKLOADS
    wl = WORKLOADS[name]
    return wl, DeviceWeights(make_weights(wl.shape, wl.weight_seed))


def workload_tokens(wl, T: int) -> torch.Tensor:
    return make_tokens(wl.shape.d_model, T, wl.token_seed, wl.shape.dtype)
