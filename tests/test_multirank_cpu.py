"""The benchmark's multi-process path on CPU: two gloo ranks.

The layer's multi-GPU mode is weak-scaling replicas (no data-path exchange):
each rank runs the whole workload on its own device, the job's time is the
slowest rank's time (an all-reduce with MAX after a barrier), and the
whole-job throughput counts every rank's tokens. These tests run that host
logic as two processes over gloo, plus the rule that only rank 0 runs and
prints the oracle arm.
"""

import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import io
    from contextlib import redirect_stdout

    import bench
    import torch.distributed as dist

    w, r, _ = bench.dist_init(backend="gloo")
    res = {"world": w, "rank": r}
    # each rank reports a different time; everyone must see the slowest
    res["max"] = bench.max_over_ranks(w, 10.0 + 5.0 * r, r)
    bench.barrier(w)
    res["value"] = bench.replica_value(105, 20, w, res["max"])
    # the oracle arm: rank 0 alone runs it and prints one line
    args = bench.argparse.Namespace(workload="tiny_f32", sparsity=0.7, steps=1, warmup=0,
                                    tokens="", gpus=w, score="h")
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(args, w, r)
    res["ref_rc"] = rc
    res["ref_out"] = buf.getvalue()
    bench.barrier(w)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.timeout(240)
def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, x in enumerate(res):
        assert x["world"] == world and x["rank"] == r
        assert x["max"] == 15.0  # the slowest rank's time, on every rank
        assert x["value"] == pytest.approx(105 * 20 * world / 15e-3)
        assert x["ref_rc"] == 0
    assert res[1]["ref_out"] == ""  # only rank 0 runs the oracle arm
    line = json.loads(res[0]["ref_out"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["config"]["parallelism"] == f"replicas x{world}"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
