"""Write tests/golden/tau_calibration.json: the thresholds of every workload.

tau is the nearest-rank quantile of |h| over the calibration batch's routed
(token, expert) pairs, computed by the CPU oracle in float64 and rounded to
float32 (shared experts get their own pool and tau). "taus_gate" holds the
same quantiles of the gate score |SiLU(g)| for the gate-score variant. Only
the oracle and the seeded input generator run here; nothing comes from the
CUDA path.

    python tests/golden/make_tau_calibration.py [workload ...]
"""

import json
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from moe_inputs import WORKLOADS, make_tokens, make_weights  # noqa: E402
from oracle import moe_oracle as om  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tau_calibration.json")


def calibrate(wl):
    sh = wl.shape
    w = make_weights(sh, wl.weight_seed)
    x = make_tokens(sh.d_model, wl.calib_tokens, wl.calib_seed, sh.dtype)
    res = om.layer_forward(x, w.W_router, w.W_gate, w.W_up, w.W_down, 0.0, sh.top_k,
                           sh.renormalize, router_bias=w.router_bias, Ws_gate=w.Ws_gate,
                           Ws_up=w.Ws_up, Ws_down=w.Ws_down, tau_shared=0.0)
    pool = om.routed_abs_h(res)
    entry = {"description": wl.description, "calib_seed": wl.calib_seed,
             "calib_tokens": wl.calib_tokens, "weight_seed": wl.weight_seed,
             "pool_size": int(pool.size), "min_router_gap": float(res.router.gap.min()),
             "taus": {}}
    entry["taus_gate"] = {}
    for key, rpool, spool_of in (("taus", pool, om.shared_abs_h),
                                 ("taus_gate", om.routed_abs_gate(res), om.shared_abs_gate)):
        for q in wl.sparsities:
            tau = om.calibrate_tau(rpool, q)
            e = {"tau": tau, "measured_sparsity": om.measured_sparsity(rpool, tau)}
            if res.h_shared is not None:
                spool = spool_of(res)
                ts = om.calibrate_tau(spool, q)
                e["tau_shared"] = ts
                e["measured_sparsity_shared"] = om.measured_sparsity(spool, ts)
            entry[key][f"{q:.2f}"] = e
    return entry


def main(names):
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    for name in names or list(WORKLOADS):
        t0 = time.time()
        data[name] = calibrate(WORKLOADS[name])
        print(f"{name}: {data[name]['taus']}  ({time.time() - t0:.1f} s)", flush=True)
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:])
