"""Pins of the CPU oracle against facts that do not come from the oracle.

The pages print no worked numbers for the layer, so the oracle is pinned by
closed forms (tests/golden/*.json), by independent formulations (a dense
einsum over all experts, pure-Python scalar loops) and by invariances. Each
is chosen so that a plausible slip in the oracle (a sign in SiLU, gate and
up swapped, a transposed W_down, >= instead of >, a dropped
renormalisation, a wrong tie-break, an off-by-one quantile) fails at least
one of them; ``test_planted_mistakes_are_caught`` checks that on the CPU.
"""

import json
import math
import os
import random

import numpy as np
import pytest

import oracle.moe_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_layer(rng, T, d, E, F, S=0, Fs=0):
    x = rng.standard_normal((T, d))
    Wr = rng.standard_normal((E, d)) / math.sqrt(d)
    Wg = rng.standard_normal((E, F, d)) / math.sqrt(d)
    Wu = rng.standard_normal((E, F, d)) / math.sqrt(d)
    Wd = rng.standard_normal((E, F, d)) / math.sqrt(F)
    sh = {}
    if S:
        sh = dict(Ws_gate=rng.standard_normal((S, Fs, d)) / math.sqrt(d),
                  Ws_up=rng.standard_normal((S, Fs, d)) / math.sqrt(d),
                  Ws_down=rng.standard_normal((S, Fs, d)) / math.sqrt(Fs))
    return x, Wr, Wg, Wu, Wd, sh


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------- closed forms

def test_swiglu_closed_form():
    g = _load("swiglu_closed_form.json")
    ln3 = math.log(3.0)
    x = np.array(g["x"])
    Wr = np.array(g["W_router"])
    Wg = np.array(g["W_gate_ln3"]) * ln3
    Wu = np.array(g["W_up"])
    Wd = np.array(g["W_down"])
    h = om.swiglu(x, Wg[0], Wu[0])
    np.testing.assert_allclose(h[0], np.array(g["h_over_ln3"]) * ln3, rtol=1e-15, atol=1e-15)
    for case in g["cases"]:
        tau = case["tau_over_ln3"] * ln3
        res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, top_k=1, renormalize=True)
        assert res.active[0, 0].tolist() == case["active"]
        np.testing.assert_allclose(res.out[0], np.array(case["out_over_ln3"]) * ln3,
                                   rtol=1e-14, atol=1e-15)
        assert res.router.topk_w[0, 0] == 1.0


def test_router_closed_form():
    g = _load("router_closed_form.json")
    L = np.log(np.array(g["logits_ln"]))[None, :]
    E = L.shape[1]
    x = np.ones((1, 1))
    for case in g["cases"]:
        r = om.route(x, L.T.copy(), case["top_k"], case["renormalize"])
        assert r.topk_idx[0].tolist() == case["idx"]
        np.testing.assert_allclose(r.topk_w[0], case["w"], rtol=1e-14)
    ties = g["ties"]
    Lt = np.array(ties["logits"])[:, None]
    for k, key in ((1, "top1"), (2, "top2"), (3, "top3")):
        r = om.route(x, Lt, k, True)
        assert r.topk_idx[0].tolist() == ties[key]
    assert E == 4


def test_calibration_nearest_rank_hand_values():
    pool = np.array([0.5, 0.1, 0.4, 0.2, 0.3])
    # ceil(0.7*5) = 4 -> 4th smallest = 0.4 ; ceil(0.2*5) = 1 -> 0.1 ; ceil(0.9*5)=5 -> 0.5
    assert om.calibrate_tau(pool, 0.7) == float(np.float32(0.4))
    assert om.calibrate_tau(pool, 0.2) == float(np.float32(0.1))
    assert om.calibrate_tau(pool, 0.9) == float(np.float32(0.5))
    assert om.calibrate_tau(pool, 0.0) == 0.0
    # q*n exactly integral in decimal but not in binary floating point
    pool10 = np.arange(1, 11) / 10.0
    assert om.calibrate_tau(pool10, 0.7, round_f32=False) == 0.7


def test_calibration_hits_count():
    rng = np.random.default_rng(5)
    pool = np.abs(rng.standard_normal(10007))
    for q in (0.3, 0.5, 0.7, 0.8, 0.9):
        tau = om.calibrate_tau(pool, q, round_f32=False)
        assert np.count_nonzero(pool <= tau) == math.ceil(q * 10007 - 1e-9)
        tau32 = om.calibrate_tau(pool, q)
        assert abs(om.measured_sparsity(pool, tau32) - q) <= 3.0 / pool.size


# ------------------------------------------------------- router invariants

def test_renormalised_weights_sum_to_one():
    rng = np.random.default_rng(1)
    x, Wr, *_ = _rand_layer(rng, 64, 32, 16, 8)
    r = om.route(x, Wr, 4, True)
    s = r.topk_w.sum(axis=1)
    assert np.all(np.abs(s - 1.0) <= 4 * np.finfo(np.float64).eps)


def test_unrenormalised_weights_are_top_probabilities():
    rng = np.random.default_rng(2)
    x, Wr, *_ = _rand_layer(rng, 64, 32, 16, 8)
    r = om.route(x, Wr, 6, False)
    full = np.sort(r.probs, axis=1)[:, ::-1][:, :6]
    np.testing.assert_allclose(np.sort(r.topk_w, axis=1)[:, ::-1], full, rtol=1e-15)
    assert np.all(r.topk_w.sum(axis=1) <= 1.0 + 1e-15)
    # independent softmax: exp / sum exp with no max shift
    p = np.exp(x @ Wr.T)
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(np.take_along_axis(p, r.topk_idx, 1), r.topk_w, rtol=1e-13)


def test_renormalised_equals_softmax_of_selected_logits():
    rng = np.random.default_rng(3)
    x, Wr, *_ = _rand_layer(rng, 50, 24, 12, 8)
    r = om.route(x, Wr, 3, True)
    Lsel = np.take_along_axis(x @ Wr.T, r.topk_idx, 1)
    sm = np.exp(Lsel - Lsel.max(1, keepdims=True))
    sm /= sm.sum(1, keepdims=True)
    np.testing.assert_allclose(r.topk_w, sm, rtol=1e-14, atol=1e-15)


def test_router_bias_shift_invariance_and_effect():
    rng = np.random.default_rng(4)
    x, Wr, *_ = _rand_layer(rng, 40, 16, 8, 8)
    b = rng.standard_normal(8) * math.sqrt(0.5)
    r1 = om.route(x, Wr, 2, True, b)
    r2 = om.route(x, Wr, 2, True, b + 7.0)
    assert np.array_equal(r1.topk_idx, r2.topk_idx)
    np.testing.assert_allclose(r1.topk_w, r2.topk_w, rtol=1e-12)
    big = np.zeros(8)
    big[5] = 100.0
    r3 = om.route(x, Wr, 2, True, big)
    assert np.all(r3.topk_idx[:, 0] == 5)


# ------------------------------------------------- independent formulations

def _dense_moe_einsum(x, Wr, Wg, Wu, Wd, k, renorm, bias=None, mask_tau=None):
    """All E experts evaluated densely, unselected experts weighted 0."""
    L = x @ Wr.T + (0 if bias is None else bias)
    p = np.exp(L - L.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    T, E = p.shape
    W = np.zeros((T, E))
    for t in range(T):
        sel = sorted(range(E), key=lambda e: (-p[t, e], e))[:k]
        s = sum(p[t, e] for e in sel)
        for e in sel:
            W[t, e] = p[t, e] / s if renorm else p[t, e]
    G = np.einsum("td,efd->tef", x, Wg)
    U = np.einsum("td,efd->tef", x, Wu)
    H = G * U / (1.0 + np.exp(-G))
    if mask_tau is not None:
        H = H * (np.abs(H) > mask_tau)
    Y = np.einsum("tef,efd->ted", H, Wd)
    return np.einsum("te,ted->td", W, Y)


def test_tau0_equals_dense_brute_force():
    rng = np.random.default_rng(6)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 9, 16, 5, 24)
    for k, renorm in ((2, True), (3, False), (1, True)):
        res = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, k, renorm)
        ref = _dense_moe_einsum(x, Wr, Wg, Wu, Wd, k, renorm)
        assert _rel(res.out, ref) <= 1e-12
        dense = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, k, renorm, dense=True)
        assert _rel(dense.out, ref) <= 1e-12


def test_masked_dense_equals_einsum_with_mask():
    rng = np.random.default_rng(7)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 7, 16, 4, 32)
    b = rng.standard_normal(4)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, router_bias=b)
    tau = float(np.median(np.abs(res.h)))
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 2, True, router_bias=b)
    ref = _dense_moe_einsum(x, Wr, Wg, Wu, Wd, 2, True, bias=b, mask_tau=tau)
    assert _rel(res.out, ref) <= 1e-12


def _scalar_brute_force(x, Wr, Wg, Wu, Wd, k, renorm, tau, score="h"):
    """Pure-Python scalar loops: each neuron enumerated, inactive rows skipped
    (score "gate": the neuron's up and down rows are read only when
    |SiLU(g)| > tau)."""
    T, d = len(x), len(x[0])
    E, F = len(Wg), len(Wg[0])
    out = [[0.0] * d for _ in range(T)]
    for t in range(T):
        L = [sum(x[t][i] * Wr[e][i] for i in range(d)) for e in range(E)]
        mx = max(L)
        ex = [math.exp(v - mx) for v in L]
        Z = sum(ex)
        p = [v / Z for v in ex]
        sel = sorted(range(E), key=lambda e: (-p[e], e))[:k]
        tot = sum(p[e] for e in sel)
        for e in sel:
            w = p[e] / tot if renorm else p[e]
            for j in range(F):
                g = sum(x[t][i] * Wg[e][j][i] for i in range(d))
                silu = g / (1.0 + math.exp(-g))
                if score == "gate" and abs(silu) <= tau:
                    continue  # inactive by the gate score: up and down rows never read
                u = sum(x[t][i] * Wu[e][j][i] for i in range(d))
                h = silu * u
                if score == "h" and abs(h) <= tau:
                    continue  # inactive neuron: its W_down row is never read
                for c in range(d):
                    out[t][c] += w * h * Wd[e][j][c]
    return np.array(out)


def test_micro_shape_scalar_brute_force():
    rng = np.random.default_rng(8)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 3, 4, 3, 6)
    base = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True)
    for q in (0.0, 0.5, 0.8):
        tau = om.calibrate_tau(np.abs(base.h), q)
        res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 2, True)
        ref = _scalar_brute_force(x.tolist(), Wr.tolist(), Wg.tolist(), Wu.tolist(),
                                  Wd.tolist(), 2, True, tau)
        assert _rel(res.out, ref) <= 1e-12 or np.linalg.norm(ref) == 0.0


def test_single_expert_is_textbook_swiglu_ffn():
    rng = np.random.default_rng(9)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 5, 8, 1, 12)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 1, True)
    g = x @ Wg[0].T
    ffn = (g * (1.0 / (1.0 + np.exp(-g))) * (x @ Wu[0].T)) @ Wd[0]
    assert _rel(res.out, ffn) <= 1e-13


def test_k_equals_E_is_full_soft_mixture():
    rng = np.random.default_rng(10)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 6, 8, 4, 10)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 4, True)
    p = np.exp(x @ Wr.T)
    p /= p.sum(1, keepdims=True)
    y = np.stack([om.swiglu(x, Wg[e], Wu[e]) @ Wd[e] for e in range(4)], 1)
    assert _rel(res.out, np.einsum("te,ted->td", p, y)) <= 1e-13


def test_tau_infinity_leaves_only_shared_experts():
    rng = np.random.default_rng(11)
    x, Wr, Wg, Wu, Wd, sh = _rand_layer(rng, 6, 8, 4, 10, S=2, Fs=12)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, np.inf, 2, True)
    assert np.all(res.out == 0.0)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, np.inf, 2, False, tau_shared=0.0, **sh)
    G = np.einsum("td,sfd->stf", x, sh["Ws_gate"])
    H = G / (1 + np.exp(-G)) * np.einsum("td,sfd->stf", x, sh["Ws_up"])
    ref = np.einsum("stf,sfd->td", H, sh["Ws_down"])
    assert _rel(res.out, ref) <= 1e-13


def test_shared_threshold_is_separate():
    rng = np.random.default_rng(12)
    x, Wr, Wg, Wu, Wd, sh = _rand_layer(rng, 8, 8, 4, 10, S=1, Fs=16)
    r0 = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, tau_shared=0.0, **sh)
    ts = float(np.quantile(np.abs(r0.h_shared), 0.6))
    r1 = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, tau_shared=ts, **sh)
    assert np.array_equal(r1.active, r0.active)
    assert np.array_equal(r1.active_shared, np.abs(r0.h_shared) > ts)
    Hm = np.where(np.abs(r0.h_shared[0]) > ts, r0.h_shared[0], 0.0)
    delta = (np.where(r0.active_shared[0], r0.h_shared[0], 0) - Hm) @ sh["Ws_down"][0]
    assert _rel(r0.out - r1.out, delta) <= 1e-10


def test_negative_shared_threshold_runs_shared_experts_dense():
    # the pages' system keeps shared experts dense and sparsifies only the
    # routed ones: with tau_shared < 0 every shared neuron is active, and the
    # output is the sparse routed part plus the textbook shared SwiGLU FFNs
    rng = np.random.default_rng(41)
    x, Wr, Wg, Wu, Wd, sh = _rand_layer(rng, 7, 8, 4, 10, S=2, Fs=12)
    base = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True)
    tau = float(np.quantile(np.abs(base.h), 0.7))
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 2, True, tau_shared=-1.0, **sh)
    assert res.active_shared.all()
    routed = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 2, True)
    G = np.einsum("td,sfd->stf", x, sh["Ws_gate"])
    H = G / (1 + np.exp(-G)) * np.einsum("td,sfd->stf", x, sh["Ws_up"])
    shared = np.einsum("stf,sfd->td", H, sh["Ws_down"])
    assert np.array_equal(res.active, routed.active)
    assert _rel(res.out, routed.out + shared) <= 1e-13


# ------------------------------------------------------------- invariances

def test_token_permutation():
    rng = np.random.default_rng(13)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 10, 8, 4, 16)
    perm = rng.permutation(10)
    a = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.3, 2, True)
    b = om.layer_forward(x[perm], Wr, Wg, Wu, Wd, 0.3, 2, True)
    assert _rel(b.out, a.out[perm]) <= 1e-13
    assert np.array_equal(b.active, a.active[perm])


def test_neuron_permutation():
    rng = np.random.default_rng(14)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 10, 8, 4, 16)
    perm = rng.permutation(16)
    a = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.3, 2, True)
    b = om.layer_forward(x, Wr, Wg[:, perm], Wu[:, perm], Wd[:, perm], 0.3, 2, True)
    assert _rel(b.out, a.out) <= 1e-13
    assert np.array_equal(b.active, a.active[:, :, perm])


def test_expert_permutation():
    rng = np.random.default_rng(15)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 10, 8, 5, 16)
    perm = rng.permutation(5)
    inv = np.argsort(perm)
    a = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.2, 2, True)
    b = om.layer_forward(x, Wr[perm], Wg[perm], Wu[perm], Wd[perm], 0.2, 2, True)
    assert _rel(b.out, a.out) <= 1e-13
    assert np.array_equal(perm[b.router.topk_idx], a.router.topk_idx)
    assert np.array_equal(inv[a.router.topk_idx], b.router.topk_idx)


def test_down_scaling_is_exact():
    rng = np.random.default_rng(16)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 10, 8, 4, 16)
    a = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.3, 2, True)
    b = om.layer_forward(x, Wr, Wg, Wu, 2.0 * Wd, 0.3, 2, True)
    assert np.array_equal(b.out, 2.0 * a.out)


def test_threshold_is_strict():
    h = np.array([[0.0, 0.5, -0.5, 0.50000001, -1.0]])
    assert om.active_mask(h, 0.5).tolist() == [[False, False, False, True, True]]
    assert om.active_mask(h, 0.0).tolist() == [[False, True, True, True, True]]


# ------------------------------------------------------- gate-score variant

def test_gate_score_closed_form():
    gs = _load("gate_score_closed_form.json")
    g = _load("swiglu_closed_form.json")
    ln3 = math.log(3.0)
    x = np.array(g["x"])
    Wr = np.array(g["W_router"])
    Wg = np.array(g["W_gate_ln3"]) * ln3
    Wu = np.array(g["W_up"])
    Wd = np.array(g["W_down"])
    base = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 1, True, score="gate")
    np.testing.assert_allclose(base.gate_abs[0, 0], np.array(gs["score_over_ln3"]) * ln3,
                               rtol=1e-15, atol=1e-15)
    for case in gs["cases"]:
        tau = case["tau_over_ln3"] * ln3
        for mode, key in (("gate", "gate"), ("h", "h")):
            res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 1, True, score=mode)
            assert res.active[0, 0].tolist() == case[f"active_{key}"], (mode, case)
            np.testing.assert_allclose(res.out[0], np.array(case[f"out_{key}_over_ln3"]) * ln3,
                                       rtol=1e-14, atol=1e-14)


def test_gate_mode_micro_scalar_brute_force():
    rng = np.random.default_rng(18)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 3, 4, 3, 6)
    base = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, score="gate")
    for q in (0.0, 0.5, 0.8):
        tau = om.calibrate_tau(om.routed_abs_gate(base), q)
        res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 2, True, score="gate")
        ref = _scalar_brute_force(x.tolist(), Wr.tolist(), Wg.tolist(), Wu.tolist(),
                                  Wd.tolist(), 2, True, tau, score="gate")
        assert _rel(res.out, ref) <= 1e-12 or np.linalg.norm(ref) == 0.0


def test_gate_mode_tau0_equals_dense():
    rng = np.random.default_rng(19)
    x, Wr, Wg, Wu, Wd, _ = _rand_layer(rng, 9, 16, 5, 24)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, score="gate")
    ref = _dense_moe_einsum(x, Wr, Wg, Wu, Wd, 2, True)
    assert _rel(res.out, ref) <= 1e-12


def test_gate_mode_active_sets_nest_and_shared_threshold():
    rng = np.random.default_rng(20)
    x, Wr, Wg, Wu, Wd, sh = _rand_layer(rng, 6, 16, 4, 32, S=1, Fs=24)
    base = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, score="gate", **sh)
    pool = om.routed_abs_gate(base)
    prev = None
    for q in (0.2, 0.5, 0.8):
        tau = om.calibrate_tau(pool, q)
        res = om.layer_forward(x, Wr, Wg, Wu, Wd, tau, 2, True, score="gate", **sh)
        assert np.array_equal(res.active, res.gate_abs > tau)
        assert np.array_equal(res.active_shared, res.gate_abs_shared > 0.0)  # tau_shared = 0
        if prev is not None:
            assert not np.any(res.active & ~prev)  # a higher tau keeps a subset
        prev = res.active
    ts = om.calibrate_tau(om.shared_abs_gate(base), 0.5)
    res = om.layer_forward(x, Wr, Wg, Wu, Wd, 0.0, 2, True, score="gate", tau_shared=ts, **sh)
    assert np.array_equal(res.active_shared, res.gate_abs_shared > ts)


# ------------------------------------------------ planted mistakes are caught

def _run_pins():
    """The cheap pins as one callable; returns the number that fail."""
    fails = 0
    for fn in (test_swiglu_closed_form, test_router_closed_form,
               test_calibration_nearest_rank_hand_values, test_tau0_equals_dense_brute_force,
               test_micro_shape_scalar_brute_force, test_threshold_is_strict,
               test_unrenormalised_weights_are_top_probabilities,
               test_renormalised_weights_sum_to_one, test_gate_score_closed_form,
               test_gate_mode_micro_scalar_brute_force):
        try:
            fn()
        except AssertionError:
            fails += 1
    return fails


def test_planted_mistakes_are_caught(monkeypatch):
    assert _run_pins() == 0
    F64 = om._f64

    def silu_sign(xr, Wg_e, Wu_e):
        g = F64(xr) @ F64(Wg_e).T
        return g / (1.0 + np.exp(g)), F64(xr) @ F64(Wu_e).T

    def gate_up_swapped(xr, Wg_e, Wu_e):
        return om.__dict__["_orig_parts"](xr, Wu_e, Wg_e)

    def score_always_h(silu_g, h, score):
        return h

    def score_pre_activation(silu_g, h, score):
        # the gate's pre-activation instead of SiLU(g): g = SiLU(g) / sigmoid(g)
        if score != "gate":
            return h
        g = np.where(silu_g == 0.0, 0.0, silu_g)
        for _ in range(60):  # invert SiLU by fixed point g = s (1 + e^-g)
            g = silu_g * (1.0 + np.exp(-np.clip(g, -30, 30)))
        return g

    def down_transposed(h, act, Wd_e):
        W = F64(Wd_e)
        n = min(W.shape)
        W2 = W.copy()
        W2[:n, :n] = W[:n, :n].T
        return np.where(act, h, 0.0) @ W2

    def mask_ge(h, tau):
        return np.abs(h) >= tau

    orig_route = om.route

    def no_renorm(x, Wr, k, renorm, bias=None):
        return orig_route(x, Wr, k, False, bias)

    def tie_high(x, Wr, k, renorm, bias=None):
        r = orig_route(x, Wr, k, renorm, bias)
        p = r.probs
        order = np.argsort(-p[:, ::-1], axis=1, kind="stable")
        r.topk_idx = (p.shape[1] - 1 - order)[:, :k]
        return r

    orig_cal = om.calibrate_tau

    def cal_off_by_one(abs_h, q, round_f32=True):
        if q <= 0:
            return 0.0
        a = np.sort(np.asarray(abs_h).ravel())
        r = min(int(math.ceil(q * a.size)), a.size - 1)
        return float(np.float32(a[r])) if round_f32 else float(a[r])

    om.__dict__["_orig_parts"] = om.swiglu_parts
    mutants = [("swiglu_parts", silu_sign), ("swiglu_parts", gate_up_swapped),
               ("score_of", score_always_h), ("score_of", score_pre_activation),
               ("down_projection", down_transposed), ("active_mask", mask_ge),
               ("route", no_renorm), ("route", tie_high), ("calibrate_tau", cal_off_by_one)]
    for name, fn in mutants:
        with monkeypatch.context() as m:
            m.setattr(om, name, fn)
            assert _run_pins() > 0, f"planted mistake in {name} ({fn.__name__}) not caught"
    assert orig_cal is om.calibrate_tau
