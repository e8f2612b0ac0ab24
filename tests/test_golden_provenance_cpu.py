"""The stored thresholds come from the committed calibration script: for the
small workloads the script's own routine, run now on the oracle and the
seeded generators, reproduces tests/golden/tau_calibration.json exactly."""

import importlib.util
import json
import os

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")


def _script():
    spec = importlib.util.spec_from_file_location(
        "make_tau_calibration", os.path.join(GOLDEN, "make_tau_calibration.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", ["tiny_f32"])
def test_stored_thresholds_reproduce(name):
    from moe_inputs import WORKLOADS
    stored = json.load(open(os.path.join(GOLDEN, "tau_calibration.json")))[name]
    fresh = _script().calibrate(WORKLOADS[name])
    for key in ("taus", "taus_gate"):
        assert stored[key].keys() == fresh[key].keys()
        for q, e in stored[key].items():
            assert e == fresh[key][q], (key, q)
    assert stored["pool_size"] == fresh["pool_size"]
