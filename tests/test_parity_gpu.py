"""GPU parity of the C-ABI layer against the CPU oracle, on every synthetic
workload at its full size, on small layers that span several tiles with
ragged tails, with each down-projection path forced, and on edge cases."""

import math
import os

import numpy as np
import pytest
import torch

from moe_inputs import LayerShape, make_tokens, make_weights
from oracle import moe_oracle as om
from _parity import (DeviceWeights, compare, make_layer, oracle_forward, run_gpu, tau_of,
                     unpack_bits, workload_tokens, workload_weights)

pytestmark = pytest.mark.gpu

PATHS = ["auto", "dense", "sparse_gemv", "sparse_tc", "sparse_tc_allrows"]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    yield
    torch.cuda.synchronize()


def _calibrated(dw, x, q, shared_q=None):
    ref0 = oracle_forward(dw, x, 0.0, 0.0)
    tau = om.calibrate_tau(om.routed_abs_h(ref0), q)
    ts = om.calibrate_tau(om.shared_abs_h(ref0), shared_q if shared_q is not None else q) \
        if ref0.h_shared is not None else 0.0
    return tau, ts


def _check(layer, dw, x, tau, ts, dtype, dense=False, top_k=None):
    gpu = run_gpu(layer, dw, x, tau, ts, top_k=top_k)
    ref = oracle_forward(dw, x, tau, ts, dense=dense, top_k=top_k)
    info = compare(gpu, ref, tau, ts, dtype, dw=dw, dense=dense)
    assert layer.status() == 0
    return gpu, ref, info


# ----------------------------------------------------------------- fp32 layer

@pytest.fixture(scope="module")
def tiny():
    return workload_weights("tiny_f32")


@pytest.mark.parametrize("path", ["auto", "dense", "sparse_gemv"])
def test_tiny_f32_full(tiny, path):
    wl, dw = tiny
    tau, _ = tau_of("tiny_f32", 0.7)
    x = workload_tokens(wl, 16)
    layer = make_layer(wl.shape, 16, path=path)
    gpu, ref, info = _check(layer, dw, x, tau, 0.0, "f32", dense=(path == "dense"))
    if path != "dense":
        st = gpu["stats"]
        assert st["n_routed_h"] == 16 * 2 * 512
        meas = 1.0 - st["n_routed_active"] / st["n_routed_h"]
        assert abs(meas - om.measured_sparsity(np.abs(ref.h), tau)) <= 2.0 / st["n_routed_h"] \
            + info["active_mismatch_in_band"] / st["n_routed_h"]


@pytest.mark.parametrize("T", [1, 5, 13, 16])
def test_tiny_f32_ragged_batches(tiny, T):
    wl, dw = tiny
    tau, _ = tau_of("tiny_f32", 0.7)
    layer = make_layer(wl.shape, 16)
    _check(layer, dw, workload_tokens(wl, T), tau, 0.0, "f32")


def test_tiny_f32_shared_and_smaller_k():
    sh = LayerShape(d_model=256, n_experts=6, top_k=3, d_ff=160, renormalize=False, n_shared=2,
                    d_ff_shared=96, dtype="f32")
    dw = DeviceWeights(make_weights(sh, 11))
    x = make_tokens(256, 21, 11, "f32")
    tau, ts = _calibrated(dw, x, 0.6, 0.4)
    layer = make_layer(sh, 32)
    _check(layer, dw, x, tau, ts, "f32")
    _check(layer, dw, x, tau, ts, "f32", top_k=2)


# ------------------------------------------------- small bf16 layers, all paths

SMALL = LayerShape(d_model=512, n_experts=4, top_k=2, d_ff=384, renormalize=True, dtype="bf16")
SMALL_SHARED = LayerShape(d_model=768, n_experts=5, top_k=2, d_ff=256, renormalize=False,
                          n_shared=1, d_ff_shared=384, dtype="bf16")


@pytest.fixture(scope="module")
def small():
    return DeviceWeights(make_weights(SMALL, 21))


@pytest.fixture(scope="module")
def small_shared():
    return DeviceWeights(make_weights(SMALL_SHARED, 22))


@pytest.mark.parametrize("T", [1, 3, 8, 37, 100, 300, 777])
@pytest.mark.parametrize("path", PATHS)
def test_small_bf16_paths(small, T, path):
    x = make_tokens(SMALL.d_model, T, 21, "bf16")
    tau, _ = _calibrated(small, x, 0.7)
    layer = make_layer(SMALL, 1024, path=path)
    _check(layer, small, x, tau, 0.0, "bf16", dense=(path == "dense"))


@pytest.mark.parametrize("T", [2, 45, 260])
@pytest.mark.parametrize("path", ["auto", "dense", "sparse_gemv", "sparse_tc"])
def test_small_bf16_shared(small_shared, T, path):
    x = make_tokens(SMALL_SHARED.d_model, T, 22, "bf16")
    tau, ts = _calibrated(small_shared, x, 0.7, 0.5)
    layer = make_layer(SMALL_SHARED, 512, path=path)
    _check(layer, small_shared, x, tau, ts, "bf16", dense=(path == "dense"))


@pytest.mark.parametrize("T", [2, 45])
def test_small_bf16_shared_dense(small_shared, T):
    """tau_shared < 0: the shared experts run dense (every shared neuron
    active) while the routed experts stay sparse."""
    x = make_tokens(SMALL_SHARED.d_model, T, 22, "bf16")
    tau, _ = _calibrated(small_shared, x, 0.7, 0.5)
    layer = make_layer(SMALL_SHARED, 512)
    gpu, ref, _ = _check(layer, small_shared, x, tau, -1.0, "bf16")
    st = gpu["stats"]
    assert st["n_shared_active"] == st["n_shared_h"] > 0
    assert st["n_routed_active"] < st["n_routed_h"]


def test_sparse_tau0_equals_dense(small):
    x = make_tokens(SMALL.d_model, 37, 21, "bf16")
    a = run_gpu(make_layer(SMALL, 64, path="auto"), small, x, 0.0)
    b = run_gpu(make_layer(SMALL, 64, path="dense"), small, x, 0.0)
    err = np.linalg.norm(a["out"] - b["out"]) / np.linalg.norm(b["out"])
    assert err <= 1e-6


def test_tau_infinity_gives_zero(small):
    x = make_tokens(SMALL.d_model, 9, 21, "bf16")
    gpu = run_gpu(make_layer(SMALL, 16, path="auto"), small, x, math.inf)
    assert np.all(gpu["out"] == 0.0)
    assert gpu["stats"]["n_routed_active"] == 0


def test_tau_infinity_leaves_shared_only(small_shared):
    x = make_tokens(SMALL_SHARED.d_model, 11, 22, "bf16")
    _, ts = _calibrated(small_shared, x, 0.7, 0.5)
    layer = make_layer(SMALL_SHARED, 16)
    _check(layer, small_shared, x, math.inf, ts, "bf16")


@pytest.mark.parametrize("T", [3, 37])
@pytest.mark.parametrize("path", ["auto", "dense"])
def test_nan_token_routes_to_valid_experts(small, T, path):
    """A token whose x row is NaN gets the experts 0..k-1 (NaN logits rank as
    -inf and an expert is chosen once), and every other token's routing,
    active set and output match the oracle run without that token."""
    bad = 1
    x = make_tokens(SMALL.d_model, T, 23, "bf16")
    tau, _ = _calibrated(small, x, 0.7)
    xn = x.clone()
    xn[bad] = float("nan")
    layer = make_layer(SMALL, 64, path=path)
    gpu = run_gpu(layer, small, xn, tau)
    assert gpu["topk_idx"][bad].tolist() == list(range(SMALL.top_k))
    keep = [t for t in range(T) if t != bad]
    k = SMALL.top_k
    pairs = [t * k + i for t in keep for i in range(k)]
    sub = {"out": gpu["out"][keep], "topk_idx": gpu["topk_idx"][keep],
           "topk_w": gpu["topk_w"][keep], "active_bits": gpu["active_bits"][pairs]}
    ref = oracle_forward(small, x[keep], tau, dense=(path == "dense"))
    compare(sub, ref, tau, 0.0, "bf16", dw=small, dense=(path == "dense"))
    assert layer.status() == 0


def test_empty_batch_is_a_noop(small):
    layer = make_layer(SMALL, 16)
    out = torch.full((0, SMALL.d_model), 7.0, dtype=torch.bfloat16, device="cuda")
    x = torch.empty((0, SMALL.d_model), dtype=torch.bfloat16, device="cuda")
    layer.forward(x, small.W_router, small.W_gate, small.W_up, small.W_down, 0.1, 2, out=out)
    torch.cuda.synchronize()
    assert layer.status() == 0


def test_max_tokens_and_rejections(small):
    layer = make_layer(SMALL, 40)
    x = make_tokens(SMALL.d_model, 40, 21, "bf16")
    tau, _ = _calibrated(small, x, 0.7)
    _check(layer, small, x, tau, 0.0, "bf16")
    big = make_tokens(SMALL.d_model, 41, 21, "bf16").cuda()
    with pytest.raises(Exception, match="T out of range"):
        layer.forward(big, small.W_router, small.W_gate, small.W_up, small.W_down, tau, 2)
    with pytest.raises(Exception, match="top_k"):
        layer.forward(big[:4], small.W_router, small.W_gate, small.W_up, small.W_down, tau, 3)


def test_deterministic(small):
    x = make_tokens(SMALL.d_model, 100, 21, "bf16")
    layer = make_layer(SMALL, 128)
    a = run_gpu(layer, small, x, 0.2)["out"]
    b = run_gpu(layer, small, x, 0.2)["out"]
    assert np.array_equal(a, b)


def test_deterministic_k_parts(small):
    """Few tensor-core groups (T = 20: four groups of ~10 tokens): each
    (group, column slice) unit is cut into K parts whose sums are added in
    part order by the last part to finish, so repeated runs agree bitwise."""
    x = make_tokens(SMALL.d_model, 20, 21, "bf16")
    layer = make_layer(SMALL, 64)
    tau = 0.2
    a = run_gpu(layer, small, x, tau)
    b = run_gpu(layer, small, x, tau)
    assert np.array_equal(a["out"], b["out"])
    assert a["stats"]["n_groups_tc_allrows"] >= 2
    compare(a, oracle_forward(small, x, tau), tau, 0.0, "bf16", dw=small)
    assert layer.status() == 0


def test_graph_replay_parity(small):
    """One forward captured into a CUDA graph, replayed on new inputs copied
    into its input buffer: every replay matches the oracle on that input."""
    T = 24
    layer = make_layer(SMALL, 64)
    xbuf = torch.empty((T, SMALL.d_model), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(xbuf)
    x0 = make_tokens(SMALL.d_model, T, 30, "bf16")
    tau, _ = _calibrated(small, x0, 0.7)

    def fwd():
        layer.forward(xbuf, small.W_router, small.W_gate, small.W_up, small.W_down, tau, 2,
                      router_bias=small.bias, out=out)

    xbuf.copy_(x0.cuda())
    fwd()  # first call outside capture (one-time kernel attributes)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        fwd()
    torch.cuda.synchronize()
    for seed in (31, 32, 33):
        x = make_tokens(SMALL.d_model, T, seed, "bf16")
        xbuf.copy_(x.cuda())
        g.replay()
        torch.cuda.synchronize()
        gpu = {"out": out.to(torch.float64).cpu().numpy()}
        gpu.update({k: v.cpu().numpy() for k, v in layer.debug().items()})
        compare(gpu, oracle_forward(small, x, tau), tau, 0.0, "bf16", dw=small)
    assert layer.status() == 0
    del g


def test_timing_and_stats(small):
    x = make_tokens(SMALL.d_model, 64, 21, "bf16").cuda()
    layer = make_layer(SMALL, 64)
    layer.set_timing(4)
    layer.forward(x, small.W_router, small.W_gate, small.W_up, small.W_down, 0.3, 2)
    t = layer.timing()
    assert set(t) >= {"route", "gate_up", "combine"}
    assert all(v >= 0 for v in t.values()) and t["gate_up"] > 0
    st = layer.stats()
    assert st["n_groups"] >= 1 and st["n_experts_touched"] >= 1


# ------------------------------------------------------------ full workloads

@pytest.fixture(scope="module")
def mixtral():
    return workload_weights("mixtral_decode")


@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_mixtral_decode(mixtral, T):
    wl, dw = mixtral
    tau, _ = tau_of("mixtral_decode", 0.7)
    layer = make_layer(wl.shape, 64)
    _check(layer, dw, workload_tokens(wl, T), tau, 0.0, "bf16")


@pytest.mark.parametrize("path", ["dense", "sparse_gemv", "sparse_tc", "sparse_tc_allrows"])
def test_mixtral_decode_paths(mixtral, path):
    wl, dw = mixtral
    tau, _ = tau_of("mixtral_decode", 0.7)
    layer = make_layer(wl.shape, 64, path=path)
    _check(layer, dw, workload_tokens(wl, 32), tau, 0.0, "bf16", dense=(path == "dense"))


# routed-only layer whose experts average <= 16 tokens at T <= 64, with a
# router bias that sends most tokens to one or two experts
SKEWED = LayerShape(d_model=512, n_experts=16, top_k=2, d_ff=384, renormalize=True,
                    dtype="bf16", router_bias_var=9.0)


@pytest.mark.parametrize("T", [40, 48, 64])
@pytest.mark.parametrize("path", PATHS)
def test_capped_groups_split_hot_experts(T, path):
    """Batches of 33-64 tokens whose experts average at most 16 tokens cap
    their groups at 32 tokens (32-column gate/up tiles); an expert holding
    more tokens is split into two groups, each read and summed on its own."""
    dw = DeviceWeights(make_weights(SKEWED, 31))
    x = make_tokens(SKEWED.d_model, T, 31, "bf16")
    tau, _ = _calibrated(dw, x, 0.7)
    layer = make_layer(SKEWED, 64, path=path)
    gpu, ref, info = _check(layer, dw, x, tau, 0.0, "bf16", dense=(path == "dense"))
    counts = np.bincount(ref.router.topk_idx.ravel(), minlength=SKEWED.n_experts)
    assert counts.max() > 32  # at least one expert is split


def test_many_small_experts():
    wl, dw = workload_weights("many_small_experts")
    tau, _ = tau_of("many_small_experts", 0.8)
    layer = make_layer(wl.shape, 256)
    gpu, ref, info = _check(layer, dw, workload_tokens(wl, 256), tau, 0.0, "bf16")
    counts = np.bincount(ref.router.topk_idx.ravel(), minlength=128)
    assert counts.max() >= 3 * max(counts.mean(), 1)  # the bias skews the load


def test_shared_routed_prefill():
    wl, dw = workload_weights("shared_routed_prefill")
    tau, ts = tau_of("shared_routed_prefill", 0.6)
    layer = make_layer(wl.shape, 4096)
    _check(layer, dw, workload_tokens(wl, 4096), tau, ts, "bf16")


@pytest.fixture(scope="module")
def sweep():
    return workload_weights("mixtral_sweep")


@pytest.mark.parametrize("T", [1, 16, 128, 512])
@pytest.mark.parametrize("q", [0.0, 0.5, 0.7, 0.9])
def test_mixtral_sweep(sweep, T, q):
    wl, dw = sweep
    tau, _ = tau_of("mixtral_sweep", q)
    layer = make_layer(wl.shape, 512)
    _check(layer, dw, workload_tokens(wl, T), tau, 0.0, "bf16")


def _expected_down_rows(gpu, F):
    """Rows the automatic per-group switch reads, from the GPU's own active
    sets: groups of <= 4 tokens stream their union (inside the gate/up kernel,
    tile by tile, unless MOE_FUSE_DOWN=0); groups of 5..8 tokens stream it
    iff 5 x union <= 4 x d_ff (one pass of 8 tokens), else all d_ff rows on
    the tensor cores, as do larger groups. Returns (rows, GEMV groups, TC
    groups, candidates on the row stream, candidates on the tensor cores,
    rows of the fused groups)."""
    act = unpack_bits(gpu["active_bits"], F)
    idx = gpu["topk_idx"].ravel()
    rows = n_gemv = n_tc = cand_gemv = cand_tc = fused = 0
    for e in np.unique(idx):
        m = int((idx == e).sum())
        u = int(act[idx == e].any(axis=0).sum())
        if m <= 4 or (m <= 8 and 5 * u <= 4 * F):
            rows += u
            n_gemv += 1
            cand_gemv += m > 4
            fused += u if m <= 4 else 0
        else:
            rows += F
            n_tc += 1
            cand_tc += m <= 8
    return rows, n_gemv, n_tc, cand_gemv, cand_tc, fused


def _fuses(shape, T):
    """Whether a forward of T tokens fuses the down projection of its groups
    of <= 4 tokens into the gate/up kernel: only when the gate/up launch has
    a CTA for every possible unit (group x 128-neuron tile), two CTAs per SM
    for groups of <= 32 tokens, and the fusion is not turned off."""
    if os.environ.get("MOE_FUSE_DOWN") == "0":
        return False
    P = T * shape.top_k
    units = (P // 128 + min(shape.n_experts, P)) * (shape.d_ff // 128)
    if shape.n_shared:
        units += shape.n_shared * ((T + 127) // 128) * (shape.d_ff_shared // 128)
    per_sm = 2 if min(T, 128) <= 32 else 1
    return units <= per_sm * torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("name,T", [("mixtral_decode", 1), ("many_small_experts", 1),
                                    ("many_small_experts", 4), ("shared_routed_prefill", 2),
                                    ("shared_routed_prefill", 4)])
def test_fused_down_matches_row_stream(name, T):
    """Small batches whose gate/up units fit one per CTA: the gate/up kernel's
    fused down projection (automatic path) and the row-stream kernel (path
    forced to the GEMV kernel) multiply the same bf16 h values by the same
    W_down rows with fp32 sums in different orders, so their fp32 outputs
    agree to fp32 rounding and read the same rows, and both match the oracle
    (routed groups of 1-4 tokens, d = 4096 and 2048, shared experts)."""
    if os.environ.get("MOE_FUSE_DOWN") == "0":
        pytest.skip("fused down projection turned off")
    wl, dw = workload_weights(name)
    assert _fuses(wl.shape, T)  # every case here has one gate/up unit per CTA at most
    q = wl.sparsities[0]
    tau, ts = tau_of(name, q)
    x = workload_tokens(wl, T)
    fused = run_gpu(make_layer(wl.shape, 64, out_f32=True), dw, x, tau, ts)
    gemv = run_gpu(make_layer(wl.shape, 64, path="sparse_gemv", out_f32=True), dw, x, tau, ts)
    a, b = fused["out"], gemv["out"]
    assert np.array_equal(fused["active_bits"], gemv["active_bits"])
    scale = np.abs(b).max()
    assert np.abs(a - b).max() <= 1e-5 * scale, (np.abs(a - b).max(), scale)
    sf, sg = fused["stats"], gemv["stats"]
    assert sf["down_rows_fused"] == sf["down_rows_read"] == sg["down_rows_gemv"] > 0
    assert sf["down_rows_gemv"] == 0 and sg["down_rows_fused"] == 0
    compare(fused, oracle_forward(dw, x, tau, ts), tau, ts, "bf16", dw=dw)


def test_one_token_layer_is_one_launch(mixtral):
    """T = 1 on the Mixtral-shaped layer: every CTA of the gate/up kernel
    routes the token itself, so the whole layer is one kernel launch (the
    first CTA writes the routing records the getters read); the routing, the
    active sets, the statistics and the output match the oracle, with the
    |h| score and with the gate score."""
    if os.environ.get("MOE_FUSE_DOWN") == "0" or os.environ.get("MOE_FUSE_ROUTE") == "0":
        pytest.skip("fused paths turned off")
    wl, dw = mixtral
    x = workload_tokens(wl, 1)
    for score in ("h", "gate"):
        tau, _ = tau_of("mixtral_decode", 0.7, score=score)
        layer = make_layer(wl.shape, 64, score=score)
        before = layer.launch_count()
        gpu = run_gpu(layer, dw, x, tau)
        assert layer.launch_count() - before == 1
        compare(gpu, oracle_forward(dw, x, tau, score=score), tau, 0.0, "bf16", dw=dw,
                score=score)
        st = gpu["stats"]
        assert st["n_groups"] == 2 and st["n_experts_touched"] == 2 and st["n_groups_gemv"] == 2
        assert st["down_rows_fused"] == st["down_rows_read"] > 0
        assert layer.status() == 0
        layer.close()


def test_small_groups_join_tensor_cores(mixtral):
    """When at least half of a batch's groups hold more than 8 tokens (all
    rows on the tensor cores by size), the batch's smaller groups join them
    on the tensor cores: Mixtral-shaped decode batch T = 32 has groups of
    4, 5, 8, 8, 9, 9, 10 and 11 tokens, so all eight read all d_ff rows there
    and the row-stream kernel gets none; the output matches the oracle."""
    wl, dw = mixtral
    tau, _ = tau_of("mixtral_decode", 0.7)
    x = workload_tokens(wl, 32)
    gpu, _, _ = _check(make_layer(wl.shape, 64), dw, x, tau, 0.0, "bf16")
    idx = gpu["topk_idx"].ravel()
    sizes = np.bincount(idx, minlength=wl.shape.n_experts)
    sizes = sizes[sizes > 0]
    assert 2 * int((sizes > 8).sum()) >= len(sizes) and (sizes <= 8).any()
    st = gpu["stats"]
    assert st["n_groups_tc_allrows"] == len(sizes) and st["n_groups_gemv"] == 0
    assert st["down_rows_read"] == len(sizes) * wl.shape.d_ff
    assert st["down_rows_gemv"] == 0 and st["down_rows_fused"] == 0


def test_candidate_groups_choose_by_union(sweep):
    """Groups of 5..8 tokens pick the row stream or all rows on the tensor
    cores after gate/up from their union size: both choices occur (high
    sparsity: row stream; tau = 0: tensor cores), the rows read and the group
    counts follow the rule, and the output matches the oracle."""
    wl, dw = sweep
    F = wl.shape.d_ff
    seen_gemv = seen_tc = 0
    for q in (0.0, 0.9):
        tau, _ = tau_of("mixtral_sweep", q)
        layer = make_layer(wl.shape, 512)
        gpu, _, _ = _check(layer, dw, workload_tokens(wl, 24), tau, 0.0, "bf16")
        rows, n_gemv, n_tc, cand_gemv, cand_tc, fused = _expected_down_rows(gpu, F)
        st = gpu["stats"]
        assert st["down_rows_read"] == rows
        assert st["down_rows_fused"] == (fused if _fuses(wl.shape, 24) else 0)
        assert st["n_groups_gemv"] == n_gemv and st["n_groups_tc_allrows"] == n_tc
        seen_gemv += cand_gemv
        seen_tc += cand_tc
    assert seen_gemv > 0 and seen_tc > 0


def _union_rows(gpu, F):
    """Active-row union size of every routed expert group, from the GPU's own
    active sets (one group per expert at these batch sizes)."""
    act = unpack_bits(gpu["active_bits"], F)
    idx = gpu["topk_idx"].ravel()
    return {int(e): (int((idx == e).sum()), int(act[idx == e].any(axis=0).sum()))
            for e in np.unique(idx)}


@pytest.mark.parametrize("T,q", [(16, 0.9), (24, 0.7)])
def test_auto_gathers_tensor_core_unions(sweep, T, q):
    """AUTO with gather_max_density = 1 and every group of >= 2 tokens on the
    tensor cores: each such group reads only its union rows, packed by the
    gather warps, so every group (row stream or tensor cores) reads exactly
    its union; with the density at 0 the same groups read all rows. Both
    outputs match the oracle."""
    wl, dw = sweep
    F = wl.shape.d_ff
    tau, _ = tau_of("mixtral_sweep", q)
    x = workload_tokens(wl, T)
    g1, _, _ = _check(make_layer(wl.shape, T, gemv_max_tokens=1, gather_max_density=1.0), dw, x,
                      tau, 0.0, "bf16")
    g0, _, _ = _check(make_layer(wl.shape, T, gemv_max_tokens=1, gather_max_density=0.0), dw, x,
                      tau, 0.0, "bf16")
    groups = _union_rows(g1, F)
    s1, s0 = g1["stats"], g0["stats"]
    assert s1["n_groups_tc_gather"] > 0 and s1["n_groups_tc_allrows"] == 0
    assert s1["down_rows_read"] == sum(u for _, u in groups.values())
    assert s0["n_groups_tc_gather"] == 0
    assert s0["n_groups_tc_allrows"] == s1["n_groups_tc_gather"]
    assert s0["down_rows_read"] == s1["down_rows_gemv"] + s0["n_groups_tc_allrows"] * F


@pytest.mark.parametrize("q", [0.998, None])
def test_gathered_k_parts_with_tiny_unions(sweep, q):
    """A few gathered tensor-core groups (6 tokens, groups of 2 and 3 tokens
    on the tensor cores) are cut into K parts to fill the grid; with unions
    of a few dozen rows (or none, tau = inf) most parts have no K-block and
    contribute zeros to the ticketed part sums. The output matches the
    oracle."""
    wl, dw = sweep
    x = workload_tokens(wl, 6)
    tau = _calibrated(dw, x, q)[0] if q is not None else math.inf
    layer = make_layer(wl.shape, 6, gemv_max_tokens=1, gather_max_density=1.0)
    gpu, _, _ = _check(layer, dw, x, tau, 0.0, "bf16")
    st = gpu["stats"]
    groups = _union_rows(gpu, wl.shape.d_ff)
    assert st["n_groups_tc_allrows"] == 0
    assert st["n_groups_tc_gather"] + st["n_groups_gemv"] == len(groups)
    assert st["n_groups_tc_gather"] >= sum(1 for m, _ in groups.values() if m >= 2) > 0
    assert st["down_rows_read"] == sum(u for _, u in groups.values())
    if q is None:
        assert not np.abs(gpu["out"]).any()
