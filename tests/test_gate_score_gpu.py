"""GPU parity of the gate-score variant (MOE_SCORE_GATE) against the oracle's
score="gate" mode: a neuron is active iff |SiLU(g)| > tau, the GEMV groups'
up projection reads only the active-row union of W_up, and an active neuron
contributes its full h = SiLU(g) u. Same criteria as the |h| score, with the
band taken on |SiLU(g)|."""

import os

import numpy as np
import pytest
import torch

from moe_inputs import LayerShape, make_tokens, make_weights
from oracle import moe_oracle as om
from _parity import (TAUS, DeviceWeights, compare, make_layer, oracle_forward, run_gpu, tau_of,
                     workload_tokens, workload_weights)

pytestmark = pytest.mark.gpu

SMALL = LayerShape(d_model=512, n_experts=4, top_k=2, d_ff=384, renormalize=True, dtype="bf16")
SMALL_SHARED = LayerShape(d_model=768, n_experts=5, top_k=2, d_ff=256, renormalize=False,
                          n_shared=1, d_ff_shared=384, dtype="bf16")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    torch.cuda.synchronize()


def _gate_taus(dw, x, q, shared_q=None):
    ref0 = oracle_forward(dw, x, 0.0, 0.0, score="gate")
    tau = om.calibrate_tau(om.routed_abs_gate(ref0), q)
    ts = om.calibrate_tau(om.shared_abs_gate(ref0), shared_q if shared_q is not None else q) \
        if ref0.h_shared is not None else 0.0
    return tau, ts


def _check(layer, dw, x, tau, ts, dtype, dense=False):
    gpu = run_gpu(layer, dw, x, tau, ts)
    ref = oracle_forward(dw, x, tau, ts, dense=dense, score="gate")
    info = compare(gpu, ref, tau, ts, dtype, dw=dw, dense=dense, score="gate")
    assert layer.status() == 0
    return gpu, ref, info


@pytest.fixture(scope="module")
def tiny():
    return workload_weights("tiny_f32")


@pytest.mark.parametrize("path", ["auto", "dense", "sparse_gemv"])
def test_tiny_f32_gate(tiny, path):
    wl, dw = tiny
    x = workload_tokens(wl, 16)
    tau, _ = tau_of("tiny_f32", 0.7, score="gate")
    layer = make_layer(wl.shape, 16, path=path, score="gate")
    _check(layer, dw, x, tau, 0.0, "f32", dense=(path == "dense"))


@pytest.fixture(scope="module")
def small():
    return DeviceWeights(make_weights(SMALL, 21))


@pytest.mark.parametrize("T", [1, 3, 8, 37, 100])
@pytest.mark.parametrize("path", ["auto", "dense", "sparse_gemv", "sparse_tc", "sparse_tc_allrows"])
def test_small_bf16_gate_paths(small, T, path):
    x = make_tokens(SMALL.d_model, T, 21, "bf16")
    tau, _ = _gate_taus(small, x, 0.7)
    layer = make_layer(SMALL, 128, path=path, score="gate")
    _check(layer, small, x, tau, 0.0, "bf16", dense=(path == "dense"))


@pytest.mark.parametrize("T", [2, 45])
@pytest.mark.parametrize("path", ["auto", "sparse_gemv"])
def test_small_bf16_gate_shared(T, path):
    dw = DeviceWeights(make_weights(SMALL_SHARED, 22))
    x = make_tokens(SMALL_SHARED.d_model, T, 22, "bf16")
    tau, ts = _gate_taus(dw, x, 0.7, 0.5)
    layer = make_layer(SMALL_SHARED, 64, path=path, score="gate")
    _check(layer, dw, x, tau, ts, "bf16")


def test_gate_tau0_equals_dense(small):
    x = make_tokens(SMALL.d_model, 9, 21, "bf16")
    a = run_gpu(make_layer(SMALL, 16, path="auto", score="gate"), small, x, 0.0)
    b = run_gpu(make_layer(SMALL, 16, path="dense"), small, x, 0.0)
    err = np.linalg.norm(a["out"] - b["out"]) / np.linalg.norm(b["out"])
    assert err <= 2e-2


@pytest.fixture(scope="module")
def mixtral():
    return workload_weights("mixtral_decode")


@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_mixtral_decode_gate(mixtral, T):
    wl, dw = mixtral
    tau, _ = tau_of("mixtral_decode", 0.7, score="gate")
    layer = make_layer(wl.shape, 64, score="gate")
    gpu, ref, _ = _check(layer, dw, workload_tokens(wl, T), tau, 0.0, "bf16")
    st = gpu["stats"]
    if T == 1:  # both groups on the GEMV path: the up and down kernels read the same rows
        assert st["up_rows_read"] == st["down_rows_read"] > 0
        assert st["up_rows_read"] < 2 * wl.shape.d_ff  # only the active-row unions

@pytest.mark.parametrize("name,T", [("mixtral_decode", 1), ("shared_routed_prefill", 1),
                                    ("many_small_experts", 1)])
def test_gate_fused_up_down_matches_separate_kernel(name, T):
    """One-token groups whose gate/up units fit one per CTA: the gate/up
    kernel does their sparse up and down projection itself (the rows with
    |SiLU(g)| > tau of W_up, then of W_down). Against the separate fused
    up + down kernel (path forced to the row stream): the same rows are read,
    the fp32 outputs agree to the rounding of h to bf16, and both match the
    oracle (routed and shared experts)."""
    if os.environ.get("MOE_FUSE_DOWN") == "0":
        pytest.skip("fused down projection turned off")
    wl, dw = workload_weights(name)
    e = TAUS[name]["taus_gate"][f"{wl.sparsities[0]:.2f}"]
    tau, ts = e["tau"], e.get("tau_shared", 0.0)
    x = workload_tokens(wl, T)
    fused = run_gpu(make_layer(wl.shape, 64, score="gate", out_f32=True), dw, x, tau, ts)
    sep = run_gpu(make_layer(wl.shape, 64, path="sparse_gemv", score="gate", out_f32=True), dw, x,
                  tau, ts)
    assert np.array_equal(fused["active_bits"], sep["active_bits"])
    sf, ss = fused["stats"], sep["stats"]
    assert sf["up_rows_fused"] == sf["up_rows_read"] == ss["up_rows_read"] > 0
    assert sf["down_rows_fused"] == sf["down_rows_read"] == ss["down_rows_read"]
    assert ss["up_rows_fused"] == 0 and ss["down_rows_fused"] == 0
    a, b = fused["out"], sep["out"]
    assert np.abs(a - b).max() <= 2e-3 * np.abs(b).max(), (np.abs(a - b).max(), np.abs(b).max())
    ref = oracle_forward(dw, x, tau, ts, score="gate")
    compare(fused, ref, tau, ts, "bf16", dw=dw, score="gate")
    compare(sep, ref, tau, ts, "bf16", dw=dw, score="gate")
