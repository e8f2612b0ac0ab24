"""ctypes declarations of the C ABI in include/moe_sparse.h.

Loads ``libmoe_sparse.so`` from this package directory and fails loudly if
it is missing: there is no other implementation of the layer to fall back
to.
"""

from __future__ import annotations

import ctypes
import os

# MOE_SPARSE_LIB=check selects the bounds-checked build (build.py --check)
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libmoe_sparse_check.so" if os.environ.get("MOE_SPARSE_LIB") == "check"
                        else "libmoe_sparse.so")

MOE_OK = 0
MOE_ERR_INVALID = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_NOMEM = 4
MOE_ERR_DEVICE_TIMEOUT = 5
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_CUDA",
                4: "MOE_ERR_NOMEM", 5: "MOE_ERR_DEVICE_TIMEOUT"}

MOE_F32 = 0
MOE_BF16 = 1
MOE_SCORE_H = 0
MOE_SCORE_GATE = 1
SCORES = {"h": MOE_SCORE_H, "gate": MOE_SCORE_GATE}

PATHS = {"auto": 0, "dense": 1, "sparse_gemv": 2, "sparse_tc": 3, "sparse_tc_allrows": 4}

STAGES = ("route", "permute", "gate_up", "union_scan", "updown_gemv", "down_gemv", "down_tc",
          "combine")


class moe_sparse_desc(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32),
        ("d_ff", ctypes.c_int32),
        ("n_experts", ctypes.c_int32),
        ("top_k_max", ctypes.c_int32),
        ("max_tokens", ctypes.c_int32),
        ("renormalize", ctypes.c_int32),
        ("n_shared", ctypes.c_int32),
        ("d_ff_shared", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("path", ctypes.c_int32),
        ("debug", ctypes.c_int32),
        ("device", ctypes.c_int32),
        ("gemv_max_tokens", ctypes.c_int32),
        ("gather_max_density", ctypes.c_float),
        ("score", ctypes.c_int32),
        ("out_f32", ctypes.c_int32),
    ]


class moe_stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "n_routed_h", "n_routed_active", "n_shared_h", "n_shared_active", "down_rows_read",
        "n_groups", "n_groups_gemv", "n_groups_tc_gather", "n_groups_tc_allrows",
        "n_experts_touched", "up_rows_read", "gate_up_rows_read", "down_rows_gemv",
        "down_rows_fused", "up_rows_fused")]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32

SIGNATURES = {
    "moe_sparse_validate_desc": (ctypes.c_int, [ctypes.POINTER(moe_sparse_desc)]),
    "moe_sparse_workspace_bytes": (ctypes.c_int, [ctypes.POINTER(moe_sparse_desc),
                                                  ctypes.POINTER(ctypes.c_size_t)]),
    "moe_sparse_init": (ctypes.c_int, [ctypes.POINTER(moe_sparse_desc), ctypes.POINTER(_vp)]),
    "moe_sparse_set_shared": (ctypes.c_int, [_vp, _vp, _vp, _vp, ctypes.c_float]),
    "moe_sparse_forward": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                                          ctypes.c_float, _i32, _vp, _vp]),
    "moe_sparse_get_debug": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_sparse_get_stats": (ctypes.c_int, [_vp, ctypes.POINTER(moe_stats), _vp]),
    "moe_sparse_get_status": (ctypes.c_int, [_vp, ctypes.POINTER(_i32)]),
    "moe_sparse_set_timing": (ctypes.c_int, [_vp, _i32]),
    "moe_sparse_get_timing": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_float), _i32]),
    "moe_sparse_get_timing_all": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_float), _i32, _i32,
                                                 ctypes.POINTER(_i32)]),
    "moe_sparse_launch_count": (ctypes.c_int, [_vp, ctypes.POINTER(ctypes.c_int64)]),
    "moe_sparse_stage_name": (ctypes.c_char_p, [_i32]),
    "moe_sparse_last_error": (ctypes.c_char_p, [_vp]),
    "moe_sparse_route_noalloc": (ctypes.c_int, [_vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32,
                                                _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_sparse_destroy": (ctypes.c_int, [_vp]),
}

# include/moe_sparse_check.h: exported by the bounds-checked build only
CHECK_SIGNATURES = {
    "moe_sparse_check_wait_timeout": (ctypes.c_int, [_vp, ctypes.c_uint32, _i32, _vp]),
}

_LIB = None


def load() -> ctypes.CDLL:
    """The C-ABI library; raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m intra_expert_activation_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        for name, (res, args) in CHECK_SIGNATURES.items():  # checked build only
            if hasattr(lib, name):
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
        _LIB = lib
    return _LIB


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str, message: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def check(status: int, where: str, ctx=None) -> None:
    if status != MOE_OK:
        msg = load().moe_sparse_last_error(ctx)
        raise MoEError(status, where, msg.decode() if msg else "")
