"""The allocation-free routing entry point (moe_sparse_route_noalloc).

Some callers cannot call cudaMalloc: code that runs while a CUDA graph is
being captured, plug-ins that live inside another framework's fixed memory
plan, serving loops that reserve all device memory up front. For them the
library offers the router step with its scratch in a fixed device array.
This test calls it through the C ABI twice in a row and checks its routing
against the routing that moe_sparse_forward reports for the same inputs,
plus the validity of the grouping it returns. The file is named so that
pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from moe_inputs import LayerShape, make_tokens, make_weights
from intra_expert_activation_b200 import MoESparseLayer, _lib

pytestmark = pytest.mark.gpu

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


def test_route_noalloc_rejects_oversized_batches():
    lib = _lib.load()
    z = ctypes.c_void_p(0)
    st = lib.moe_sparse_route_noalloc(None, 5000, 512, None, None, 8, 2, 1, _lib.MOE_BF16,
                                      None, None, None, None, None, None)
    assert st == _lib.MOE_ERR_UNSUPPORTED
    assert b"4096" in lib.moe_sparse_last_error(None)
    st = lib.moe_sparse_route_noalloc(None, 4, 512, None, None, 300, 2, 1, _lib.MOE_BF16,
                                      None, None, None, None, None, None)
    assert st == _lib.MOE_ERR_UNSUPPORTED
    assert z.value is None
