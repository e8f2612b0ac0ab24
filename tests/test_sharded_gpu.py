"""d_ff sharding with the CUDA layer: two gloo ranks on one GPU.

Each rank runs DffShardedLayer with the C-ABI library's layer over its half
of every expert's neurons (rows of W_gate, W_up, W_down and of the shared
experts' weights), the router replicated. Each rank's layer writes its
partial output in fp32 (out_f32), gloo sums the two partials in fp32, and the
sum is rounded to bf16 once. The ranks' kernels never wait on each other: the
only exchange is the host-side all-reduce, so one GPU serves both ranks. The
result is compared with the oracle on the full layer by the usual parity
criteria (routing bit-exact, active sets outside the band, relative Frobenius
error <= 2e-2), with the ranks' active bitmaps joined along the neurons.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from moe_inputs import WORKLOADS, LayerShape, make_tokens, make_weights
from _parity import DeviceWeights, compare, oracle_forward, tau_of, unpack_bits

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

SMALL_SHARED = LayerShape(d_model=768, n_experts=5, top_k=2, d_ff=512, renormalize=False,
                          n_shared=1, d_ff_shared=512, dtype="bf16")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(name):
    """(shape, weight seed, token seed, T, tau, tau_shared)"""
    if name == "mixtral_decode":
        wl = WORKLOADS[name]
        tau, _ = tau_of(name, 0.7)
        return wl.shape, wl.weight_seed, wl.token_seed, 8, tau, 0.0
    return SMALL_SHARED, 41, 41, 45, None, None


def _rank_main(rank, world, port, out_dir, name, tau, ts):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from intra_expert_activation_b200.sharded import DffShardedLayer
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=300))
    sh, wseed, xseed, T, _, _ = _case(name)
    w = make_weights(sh, wseed)
    dev = torch.device("cuda", 0)
    L = DffShardedLayer(sh.d_model, sh.d_ff, sh.n_experts, sh.top_k, T,
                        n_shared=sh.n_shared, d_ff_shared=sh.d_ff_shared,
                        renormalize=sh.renormalize, dtype=sh.dtype, debug=True, device=0)
    cu = lambda t: t.to(dev).contiguous()
    if sh.n_shared:
        L.set_shared(cu(L.shard(w.Ws_gate)), cu(L.shard(w.Ws_up)), cu(L.shard(w.Ws_down)), ts)
    x = make_tokens(sh.d_model, T, xseed, sh.dtype).to(dev)
    bias = None if w.router_bias is None else cu(w.router_bias)
    out = L.forward(x, cu(w.W_router), cu(L.shard(w.W_gate)), cu(L.shard(w.W_up)),
                    cu(L.shard(w.W_down)), tau, sh.top_k, router_bias=bias)
    dbg = L.layer.debug()
    torch.cuda.synchronize()
    res = {"out": out.to(torch.float64).cpu().numpy(), "dtype": str(out.dtype),
           "status": L.layer.status()}
    res.update({k: v.cpu().numpy() for k, v in dbg.items()})
    dist.barrier()
    dist.destroy_process_group()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **res)


def _join_bits(parts, F):
    """Active bitmaps of the ranks' neuron halves -> the full layer's words."""
    bits = np.concatenate([unpack_bits(p, F // len(parts)) for p in parts], axis=-1)
    pad = (-bits.shape[-1]) % 32
    bits = np.concatenate([bits, np.zeros(bits.shape[:-1] + (pad,), bool)], axis=-1)
    words = np.packbits(bits.reshape(*bits.shape[:-1], -1, 32), axis=-1, bitorder="little")
    return words.view(np.uint32).reshape(*bits.shape[:-1], -1)


@pytest.mark.timeout(900)
@pytest.mark.parametrize("name", ["small_shared", "mixtral_decode"])
def test_two_gloo_ranks_on_the_cuda_layer(tmp_path, name):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    sh, wseed, xseed, T, tau, ts = _case(name)
    w = make_weights(sh, wseed)
    x = make_tokens(sh.d_model, T, xseed, sh.dtype)
    dw = DeviceWeights(w, device="cpu")
    if tau is None:  # calibrate on this batch (70% routed, 50% shared)
        from oracle import moe_oracle as om
        ref0 = oracle_forward(dw, x, 0.0, 0.0)
        tau = om.calibrate_tau(om.routed_abs_h(ref0), 0.7)
        ts = om.calibrate_tau(om.shared_abs_h(ref0), 0.5)
    world = 2
    ctx = mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), name, tau, ts),
                   nprocs=world, join=False)
    ref = oracle_forward(dw, x, tau, ts)  # on the host while the ranks run
    while not ctx.join():
        pass
    res = [dict(np.load(tmp_path / f"rank{r}.npz")) for r in range(world)]
    for r in res:
        assert int(r["status"]) == 0
        assert str(r["dtype"]) == "torch.bfloat16"
    # the all-reduce gives every rank the same sum
    assert np.array_equal(res[0]["out"], res[1]["out"])
    for r in res[1:]:
        assert np.array_equal(r["topk_idx"], res[0]["topk_idx"])
    gpu = {"out": res[0]["out"], "topk_idx": res[0]["topk_idx"], "topk_w": res[0]["topk_w"],
           "active_bits": _join_bits([r["active_bits"] for r in res], sh.d_ff)}
    if sh.n_shared:
        gpu["active_bits_shared"] = _join_bits([r["active_bits_shared"] for r in res],
                                               sh.d_ff_shared)
    info = compare(gpu, ref, tau, ts, sh.dtype, dw=dw)
    print(f"{name}: {info}")
