"""The bounds-checked build (libmoe_sparse_check.so, MOE_SPARSE_LIB=check) on
the GPU: its bounded waits give up and report, and the parity suite passes on
it with the device status word left at zero.

Failure detection is exercised without a fault: a one-CTA test kernel waits,
with a small probe limit, on an mbarrier arrival or a global flag that never
comes; the wait gives up, records MOE_ERR_DEVICE_TIMEOUT in the context's
status word and the kernel returns, after which the same context still runs a
forward that matches the oracle. Each case runs in a child process, because
the library choice is made when the binding first loads.
"""

import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CHECK_LIB = os.path.join(ROOT, "intra_expert_activation_b200", "libmoe_sparse_check.so")

pytestmark = pytest.mark.gpu

_CHILD = r"""
import ctypes, sys
sys.path[:0] = [ROOT, ROOT + "/tests"]
import numpy as np, torch
from intra_expert_activation_b200 import _lib, MoESparseLayer
assert _lib.LIB_PATH.endswith("libmoe_sparse_check.so"), _lib.LIB_PATH
from moe_inputs import LayerShape, make_tokens, make_weights
from _parity import DeviceWeights, compare, oracle_forward, run_gpu, make_layer
from oracle import moe_oracle as om
sh = LayerShape(d_model=512, n_experts=4, top_k=2, d_ff=384, renormalize=True, dtype="bf16")
dw = DeviceWeights(make_weights(sh, 21))
layer = make_layer(sh, 64)
lib = _lib.load()
for which in (0, 1):
    st = lib.moe_sparse_check_wait_timeout(layer.ctx, 2000, which,
                                           torch.cuda.current_stream().cuda_stream)
    assert st == _lib.MOE_OK, lib.moe_sparse_last_error(layer.ctx)
    torch.cuda.synchronize()
    assert layer.status() == _lib.MOE_ERR_DEVICE_TIMEOUT, which
    assert layer.status() == 0  # reading the word clears it
assert lib.moe_sparse_check_wait_timeout(layer.ctx, 0, 0, None) == _lib.MOE_ERR_INVALID
assert lib.moe_sparse_check_wait_timeout(layer.ctx, 10, 2, None) == _lib.MOE_ERR_INVALID
x = make_tokens(sh.d_model, 37, 21, "bf16")
ref0 = oracle_forward(dw, x, 0.0)
tau = om.calibrate_tau(om.routed_abs_h(ref0), 0.7)
gpu = run_gpu(layer, dw, x, tau)
print(compare(gpu, oracle_forward(dw, x, tau), tau, 0.0, "bf16", dw=dw))
assert layer.status() == 0
print("CHILD_OK")
"""


def _run(code_or_args, timeout=900):
    env = {**os.environ, "MOE_SPARSE_LIB": "check"}
    args = [sys.executable, "-c", code_or_args] if isinstance(code_or_args, str) else \
        [sys.executable, *code_or_args]
    return subprocess.run(args, capture_output=True, text=True, cwd=ROOT, env=env,
                          timeout=timeout)


@pytest.fixture(scope="module", autouse=True)
def _checked_library():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    if not os.path.exists(CHECK_LIB):
        from intra_expert_activation_b200 import build
        build.build(check=True)


@pytest.mark.timeout(900)
def test_bounded_waits_time_out_into_the_status_word():
    r = _run(_CHILD.replace("ROOT", repr(ROOT)))
    assert r.returncode == 0 and "CHILD_OK" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]


@pytest.mark.timeout(1200)
def test_parity_suite_on_the_checked_build():
    """A cross-section of the GPU parity tests (every path on the small bf16
    layer, the fp32 layer, shared experts, the Mixtral-shaped decode batches,
    graph replay, NaN tokens) on the checked build; each asserts that the
    status word stays zero, i.e. no bounds check fired."""
    sel = ("small_bf16_paths or tiny_f32 or small_bf16_shared or mixtral_decode or "
           "graph_replay or nan_token or deterministic_k_parts")
    r = _run(["-m", "pytest", "tests/test_parity_gpu.py", "-m", "gpu", "-q", "-x",
              "-p", "no:cacheprovider", "-k", sel])
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    print(r.stdout.strip().splitlines()[-1])
