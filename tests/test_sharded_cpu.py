"""d_ff sharding of the layer, on the CPU.

The decomposition it rests on is checked on the oracle: with every expert's
neurons split into n shards (router replicated), the per-shard layers' outputs
add up to the full layer's output, with the threshold applied per neuron (the
active sets are the full layer's, split). The sharded wrapper's own logic
(weight slicing, per-rank layer, fp32 sum all-reduce) runs as two gloo ranks
with an oracle-backed stand-in for the CUDA layer.
"""

import json
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import moe_oracle as om

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _layer(seed, T=6, d=16, E=4, F=24, S=1, Fs=12):
    rng = np.random.default_rng(seed)
    w = dict(x=rng.standard_normal((T, d)),
             Wr=rng.standard_normal((E, d)) / math.sqrt(d),
             Wg=rng.standard_normal((E, F, d)) / math.sqrt(d),
             Wu=rng.standard_normal((E, F, d)) / math.sqrt(d),
             Wd=rng.standard_normal((E, F, d)) / math.sqrt(F),
             Wsg=rng.standard_normal((S, Fs, d)) / math.sqrt(d),
             Wsu=rng.standard_normal((S, Fs, d)) / math.sqrt(d),
             Wsd=rng.standard_normal((S, Fs, d)) / math.sqrt(Fs))
    return w


def _full(w, tau, ts, k=2):
    return om.layer_forward(w["x"], w["Wr"], w["Wg"], w["Wu"], w["Wd"], tau, k, True,
                            Ws_gate=w["Wsg"], Ws_up=w["Wsu"], Ws_down=w["Wsd"], tau_shared=ts)


@pytest.mark.parametrize("n", [2, 3, 4])
def test_shards_add_up_to_the_layer(n):
    w = _layer(5, F=24, Fs=12)
    base = _full(w, 0.0, 0.0)
    tau = float(np.quantile(np.abs(base.h), 0.7))
    ts = float(np.quantile(np.abs(base.h_shared), 0.5))
    full = _full(w, tau, ts)
    F, Fs = w["Wg"].shape[1], w["Wsg"].shape[1]
    f, fs = F // n, Fs // n
    total = np.zeros_like(full.out)
    for r in range(n):
        sl, ss = slice(r * f, (r + 1) * f), slice(r * fs, (r + 1) * fs)
        part = om.layer_forward(w["x"], w["Wr"], w["Wg"][:, sl], w["Wu"][:, sl], w["Wd"][:, sl],
                                tau, 2, True, Ws_gate=w["Wsg"][:, ss], Ws_up=w["Wsu"][:, ss],
                                Ws_down=w["Wsd"][:, ss], tau_shared=ts)
        assert np.array_equal(part.active, full.active[:, :, sl])
        assert np.array_equal(part.active_shared, full.active_shared[:, :, ss])
        total += part.out
    np.testing.assert_allclose(total, full.out, rtol=1e-12, atol=1e-14)


def test_shard_rows_cover_every_neuron_once():
    from intra_expert_activation_b200.sharded import shard_rows
    W = torch.arange(3 * 12 * 5, dtype=torch.float32).reshape(3, 12, 5)
    parts = [shard_rows(W, r, 4) for r in range(4)]
    assert all(p.is_contiguous() and p.shape == (3, 3, 5) for p in parts)
    assert torch.equal(torch.cat(parts, dim=1), W)
    with pytest.raises(ValueError):
        shard_rows(W, 0, 5)


class _OracleLayer:
    """Stand-in for the CUDA layer in the host-logic test: the same calls,
    computed by the oracle on CPU tensors."""

    def __init__(self, d_model, d_ff, n_experts, top_k_max, max_tokens, n_shared=0,
                 d_ff_shared=0, **kw):
        self.d_ff, self.d_ff_shared = d_ff, d_ff_shared
        self.shared = None

    def set_shared(self, Wg_s, Wu_s, Wd_s, tau_shared):
        self.shared = (Wg_s, Wu_s, Wd_s, tau_shared)

    def forward(self, x, W_router, W_gate, W_up, W_down, tau, top_k, router_bias=None):
        assert W_gate.shape[1] == self.d_ff
        Wsg, Wsu, Wsd, ts = self.shared
        res = om.layer_forward(x.numpy(), W_router.numpy(), W_gate.numpy(), W_up.numpy(),
                               W_down.numpy(), tau, top_k, True, Ws_gate=Wsg.numpy(),
                               Ws_up=Wsu.numpy(), Ws_down=Wsd.numpy(), tau_shared=ts)
        return torch.from_numpy(res.out)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, tau, ts):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from intra_expert_activation_b200.sharded import DffShardedLayer
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w = {k: torch.from_numpy(v) for k, v in _layer(5, F=24, Fs=12).items()}
    L = DffShardedLayer(16, 24, 4, 2, 8, n_shared=1, d_ff_shared=12,
                        reduce_dtype=torch.float64, layer_factory=_OracleLayer)
    L.set_shared(L.shard(w["Wsg"]), L.shard(w["Wsu"]), L.shard(w["Wsd"]), ts)
    out = L.forward(w["x"], w["Wr"], L.shard(w["Wg"]), L.shard(w["Wu"]), L.shard(w["Wd"]),
                    tau, 2)
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(out.tolist(), f)


@pytest.mark.timeout(240)
def test_two_gloo_ranks_give_the_full_layer(tmp_path):
    w = _layer(5, F=24, Fs=12)
    base = _full(w, 0.0, 0.0)
    tau = float(np.quantile(np.abs(base.h), 0.7))
    ts = float(np.quantile(np.abs(base.h_shared), 0.5))
    full = _full(w, tau, ts).out
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), tau, ts), nprocs=world,
             join=True)
    for r in range(world):
        out = np.array(json.load(open(tmp_path / f"rank{r}.json")))
        np.testing.assert_allclose(out, full, rtol=1e-12, atol=1e-14)
