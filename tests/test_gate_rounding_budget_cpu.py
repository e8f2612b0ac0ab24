"""Error budget of one reading taken by the GPU gate-score path.

With the gate score, the gate-only GEMM keeps the masked SiLU(g) in bf16 until
the fused up + down kernel multiplies it by u, so the GPU computes
h = bf16(SiLU(g)) * u where the pages' definition (and the oracle) has
h = SiLU(g) * u. The active set is not affected (the threshold test runs on
the fp32 SiLU(g) before the rounding). This test measures, on the CPU with the
oracle's own steps, how much of the bf16 output tolerance (2e-2 relative
Frobenius) that rounding alone uses, and prints it.
"""

import numpy as np
import torch

from moe_inputs import LayerShape, make_tokens, make_weights
from moe_inputs.generate import widen_f64
from oracle import moe_oracle as om

SHAPE = LayerShape(d_model=512, n_experts=4, top_k=2, d_ff=384, renormalize=True, dtype="bf16")
BF16_TOL = 2e-2  # the bf16 parity bound on the output (relative Frobenius)


def _bf16(a: np.ndarray) -> np.ndarray:
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()


def _outputs(w, x, tau):
    """The oracle's gate-score output, and the same steps with SiLU(g)
    rounded to bf16 before it multiplies u."""
    args = [widen_f64(t) for t in (x, w.W_router, w.W_gate, w.W_up, w.W_down)]
    x64, Wr, Wg, Wu, Wd = args
    ref = om.layer_forward(x64, Wr, Wg, Wu, Wd, tau, SHAPE.top_k, SHAPE.renormalize, score="gate")
    r = ref.router
    T, d = x64.shape
    y = np.zeros((T, SHAPE.top_k, d))
    for e in range(SHAPE.n_experts):
        tt, ii = np.nonzero(r.topk_idx == e)
        if tt.size == 0:
            continue
        sg, u = om.swiglu_parts(x64[tt], Wg[e], Wu[e])
        act = om.active_mask(sg, tau)
        y[tt, ii] = om.down_projection(_bf16(sg) * u, act, Wd[e])
    rounded = np.einsum("tk,tkd->td", r.topk_w, y)
    return ref.out, rounded


def test_gate_score_silu_rounding_budget():
    w = make_weights(SHAPE, seed=1234)
    x = make_tokens(SHAPE.d_model, 64, seed=99, dtype="bf16")
    args = [widen_f64(t) for t in (x, w.W_router, w.W_gate, w.W_up, w.W_down)]
    ref0 = om.layer_forward(*args, 0.0, SHAPE.top_k, SHAPE.renormalize, score="gate")
    for q in (0.0, 0.7, 0.9):
        tau = om.calibrate_tau(om.routed_abs_gate(ref0), q) if q > 0 else 0.0
        exact, rounded = _outputs(w, x, tau)
        rel = np.linalg.norm(rounded - exact) / np.linalg.norm(exact)
        print(f"gate score, sparsity {q:.1f}: bf16(SiLU(g)) costs {rel:.2e} relative "
              f"Frobenius of the {BF16_TOL:.0e} output bound ({rel / BF16_TOL:.1%})")
        # bf16 keeps 8 significant bits: at most 2^-9 relative error per
        # SiLU(g); over a row's sum of neurons the measured share stays below
        # 2^-8, a fifth of the output bound
        assert 0.0 < rel < 2.0 ** -8
