"""The allocation-free routing entry point (moe_sparse_route_noalloc).

Some callers cannot call cudaMalloc: plug-ins that live inside another
framework's fixed memory plan, and serving loops that reserve all device
memory up front and treat any later allocation as a failure. For them the
library offers the router step with its scratch in a fixed device array.
The GPU tests call it through the C ABI twice in a row and check its routing
against the routing that moe_sparse_forward reports for the same inputs,
plus the validity of the grouping it returns; the CPU tests check that bad
arguments are refused before any CUDA call. The file is named so that pytest
collects it last.
"""

import numpy as np
import pytest
import torch

from moe_inputs import LayerShape, make_tokens, make_weights
from intra_expert_activation_b200 import MoESparseLayer, _lib

CASES = [
    (LayerShape(d_model=512, n_experts=8, top_k=2, d_ff=256, renormalize=True, dtype="bf16",
                router_bias_var=0.5), 37, 31),
    (LayerShape(d_model=512, n_experts=64, top_k=6, d_ff=256, renormalize=False, dtype="bf16"),
     300, 32),
    (LayerShape(d_model=256, n_experts=8, top_k=2, d_ff=128, renormalize=True, dtype="f32"), 3, 33),
]


def _route_noalloc(lib, x, Wr, bias, sh, T):
    dev = x.device
    k, E = sh.top_k, sh.n_experts
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    w = torch.full((T, k), -7.0, dtype=torch.float32, device=dev)
    off = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
    slot = torch.full((T * k,), -7, dtype=torch.int32, device=dev)
    perm = torch.full((T * k,), -7, dtype=torch.int32, device=dev)
    st = lib.moe_sparse_route_noalloc(
        x.data_ptr(), T, sh.d_model, Wr.data_ptr(), None if bias is None else bias.data_ptr(), E,
        k, int(sh.renormalize), _lib.MOE_BF16 if sh.dtype == "bf16" else _lib.MOE_F32,
        idx.data_ptr(), w.data_ptr(), off.data_ptr(), slot.data_ptr(), perm.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert st == _lib.MOE_OK, lib.moe_sparse_last_error(None)
    torch.cuda.synchronize()
    return [t.cpu().numpy() for t in (idx, w, off, slot, perm)]


@pytest.mark.gpu
@pytest.mark.parametrize("sh,T,seed", CASES)
def test_route_noalloc_matches_forward_routing(sh, T, seed):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    lib = _lib.load()
    w = make_weights(sh, seed)
    x = make_tokens(sh.d_model, T, seed, sh.dtype).cuda()
    d = lambda t: None if t is None else t.cuda().contiguous()
    layer = MoESparseLayer(sh.d_model, sh.d_ff, sh.n_experts, sh.top_k, T,
                           renormalize=sh.renormalize, dtype=sh.dtype, debug=True)
    layer.forward(x, d(w.W_router), d(w.W_gate), d(w.W_up), d(w.W_down), 0.1, sh.top_k,
                  router_bias=d(w.router_bias))
    ref = layer.debug()
    ref_idx = ref["topk_idx"].cpu().numpy()
    ref_w = ref["topk_w"].cpu().numpy()
    layer.close()

    k, E, P = sh.top_k, sh.n_experts, T * sh.top_k
    runs = [_route_noalloc(lib, x, d(w.W_router), d(w.router_bias), sh, T) for _ in range(2)]
    for idx, wt, off, slot, perm in runs:
        assert np.array_equal(idx, ref_idx)
        np.testing.assert_allclose(wt, ref_w, rtol=2e-5, atol=1e-7)
        counts = np.bincount(idx.ravel(), minlength=E)
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
        assert np.array_equal(np.sort(slot), np.arange(P))
        flat = idx.ravel()
        for p in range(P):
            e = flat[p]
            assert off[e] <= slot[p] < off[e + 1]
            assert perm[slot[p]] == p // k
        for e in range(E):  # within an expert, positions follow pair order
            ps = np.nonzero(flat == e)[0]
            assert np.array_equal(slot[ps], np.arange(off[e], off[e + 1]))
    for a, b in zip(runs[0], runs[1]):
        assert np.array_equal(a, b)


@pytest.mark.gpu
def test_route_noalloc_nan_rows_get_distinct_valid_experts():
    """A token whose x row holds NaN (every logit NaN) or +inf gets k distinct
    experts, the lowest ids, as NaN logits rank as -inf; the other tokens
    route exactly as without it."""
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    lib = _lib.load()
    sh, T = CASES[1][0], 40
    w = make_weights(sh, 34)
    x = make_tokens(sh.d_model, T, 34, sh.dtype).cuda()
    d = lambda t: None if t is None else t.cuda().contiguous()
    clean = _route_noalloc(lib, x, d(w.W_router), d(w.router_bias), sh, T)
    bad = x.clone()
    bad[3] = float("nan")
    bad[17, 5] = float("inf")
    for _ in range(2):
        idx, wt, off, slot, perm = _route_noalloc(lib, bad, d(w.W_router), d(w.router_bias),
                                                  sh, T)
        k, E = sh.top_k, sh.n_experts
        assert (idx >= 0).all() and (idx < E).all()
        for t in (3, 17):
            assert len(set(idx[t].tolist())) == k
        assert idx[3].tolist() == list(range(k))
        rest = [t for t in range(T) if t not in (3, 17)]
        assert np.array_equal(idx[rest], clean[0][rest])
        assert np.array_equal(np.sort(slot), np.arange(T * k))
        counts = np.bincount(idx.ravel(), minlength=E)
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))


def _call(lib, x, T, d, E, k, dtype, bufs):
    return lib.moe_sparse_route_noalloc(x, T, d, bufs, None, E, k, 1, dtype, bufs, bufs, bufs,
                                        bufs, bufs, None)


@pytest.mark.parametrize("args,code,msg", [
    # T, d_model, n_experts, top_k, dtype
    ((5000, 512, 8, 2, "bf16"), "MOE_ERR_UNSUPPORTED", b"4096"),
    ((4, 512, 300, 2, "bf16"), "MOE_ERR_UNSUPPORTED", b"n_experts"),
    ((4, 512, 8, 0, "bf16"), "MOE_ERR_INVALID", b"top_k"),
    ((4, 512, 8, 9, "bf16"), "MOE_ERR_INVALID", b"top_k"),
    ((4, 512, 32, 17, "bf16"), "MOE_ERR_INVALID", b"top_k"),
    ((4, 512, 8, 2, 7), "MOE_ERR_INVALID", b"dtype"),
    ((4, 384, 8, 2, "bf16"), "MOE_ERR_UNSUPPORTED", b"multiple of 256"),
    ((4, 192, 8, 2, "f32"), "MOE_ERR_UNSUPPORTED", b"multiple of 256"),
    ((-1, 512, 8, 2, "bf16"), "MOE_ERR_INVALID", b"T < 0"),
])
def test_route_noalloc_rejects_bad_arguments(args, code, msg):
    """Argument errors return before any CUDA call, with a message (CPU)."""
    lib = _lib.load()
    T, d, E, k, dt = args
    dtype = {"bf16": _lib.MOE_BF16, "f32": _lib.MOE_F32}.get(dt, dt)
    # non-NULL stand-ins: the checks return before anything is dereferenced
    st = _call(lib, 0x1000, T, d, E, k, dtype, 0x2000)
    assert st == getattr(_lib, code)
    assert msg in lib.moe_sparse_last_error(None)


def test_route_noalloc_rejects_null_and_misaligned_pointers():
    lib = _lib.load()
    st = lib.moe_sparse_route_noalloc(0x1000, 4, 512, 0x2000, None, 8, 2, 1, _lib.MOE_BF16,
                                      0x3000, 0x4000, None, 0x5000, 0x6000, None)
    assert st == _lib.MOE_ERR_INVALID
    assert b"expert_offsets" in lib.moe_sparse_last_error(None)
    st = lib.moe_sparse_route_noalloc(0x1000, 4, 512, 0x2000, None, 8, 2, 1, _lib.MOE_BF16,
                                      None, 0x4000, 0x7000, 0x5000, 0x6000, None)
    assert st == _lib.MOE_ERR_INVALID
    assert b"NULL" in lib.moe_sparse_last_error(None)
    st = lib.moe_sparse_route_noalloc(0x1008, 4, 512, 0x2000, None, 8, 2, 1, _lib.MOE_BF16,
                                      0x3000, 0x4000, 0x7000, 0x5000, 0x6000, None)
    assert st == _lib.MOE_ERR_INVALID
    assert b"16-byte aligned" in lib.moe_sparse_last_error(None)
    st = lib.moe_sparse_route_noalloc(0x1000, 4, 512, 0x2004, None, 8, 2, 1, _lib.MOE_F32,
                                      0x3000, 0x4000, 0x7000, 0x5000, 0x6000, None)
    assert st == _lib.MOE_ERR_INVALID
    assert b"16-byte aligned" in lib.moe_sparse_last_error(None)
