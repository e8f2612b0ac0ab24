"""Source rules the kernels keep, checked on the text of csrc/ (CPU):

* no TMA or bulk load with cluster multicast anywhere;
* no device trap or device assert: kernels report failures in the status
  word and return;
* every mbarrier wait goes through the bounded helpers in common.cuh (a wait
  that gives up after about a second and records MOE_ERR_DEVICE_TIMEOUT), and
  every other spin on global memory is a bounded loop over kSpinLimit.
"""

import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "intra_expert_activation_b200", "csrc")


def _sources():
    out = {}
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(CSRC, f)) as fh:
                out[f] = fh.read()
    return out


def _code(text):
    """The text without comments (so that prose may name what code must not)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_no_multicast_loads():
    for f, text in _sources().items():
        assert "multicast" not in _code(text), f


def test_no_device_trap_or_assert():
    for f, text in _sources().items():
        code = _code(text)
        assert "__trap" not in code and not re.search(r"\btrap;", code), f
        assert not re.search(r"(?<![_\w])assert\s*\(", code), f


def test_mbarrier_waits_are_bounded_helpers():
    src = _sources()
    for f, text in src.items():
        if f != "common.cuh":
            assert "mbarrier.try_wait" not in _code(text), f
    common = _code(src["common.cuh"])
    # the helpers loop at most kSpinLimit times and report the timeout
    assert "kSpinLimit" in common and "kErrDeviceTimeout" in common


def test_global_spins_are_bounded():
    for f, text in _sources().items():
        code = _code(text)
        for m in re.finditer(r"ld\.acquire\.gpu", code):
            window = code[max(0, m.start() - 400):m.start()]
            assert "kSpinLimit" in window, f"{f}: acquire spin without an iteration limit"
        assert not re.search(r"while\s*\(\s*(true|1)\s*\)", code), f
