"""Python binding of the C ABI: argument marshalling only.

Every step of the layer runs in the CUDA kernels of libmoe_sparse.so; this
module checks tensor dtypes, devices and contiguity, passes raw device
pointers and the current CUDA stream, and turns status codes into
exceptions. PyTorch is used only for device memory and streams.
"""

from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib

_DT = {"f32": (torch.float32, _lib.MOE_F32), "bf16": (torch.bfloat16, _lib.MOE_BF16)}


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


class MoESparseLayer:
    """One context of the layer (``moe_sparse_init`` ... ``moe_sparse_destroy``).

    Shapes and layouts are those of include/moe_sparse.h:
    x [T][d_model], W_router [E][d_model], W_gate / W_up / W_down
    [E][d_ff][d_model], out [T][d_model], all in ``dtype`` on the device.
    """

    def __init__(self, d_model: int, d_ff: int, n_experts: int, top_k_max: int,
                 max_tokens: int, renormalize: bool = True, n_shared: int = 0,
                 d_ff_shared: int = 0, dtype: str = "bf16", path: str = "auto",
                 debug: bool = False, device: int = 0, gemv_max_tokens: int = 0,
                 gather_max_density: float = 0.5, score: str = "h", out_f32: bool = False):
        self.lib = _lib.load()
        self.torch_dtype, code = _DT[dtype]
        self.dtype = dtype
        self.device = torch.device("cuda", device)
        self.d_model, self.d_ff, self.n_experts = d_model, d_ff, n_experts
        self.n_shared, self.d_ff_shared = n_shared, d_ff_shared
        self.desc = _lib.moe_sparse_desc(
            d_model, d_ff, n_experts, top_k_max, max_tokens, int(renormalize), n_shared,
            d_ff_shared, code, _lib.PATHS[path], int(debug), device, gemv_max_tokens,
            gather_max_density, _lib.SCORES[score], int(out_f32))
        self.score = score
        # out: float32 (the combine's sums, unrounded) or the layer's dtype
        self.out_dtype = torch.float32 if out_f32 else self.torch_dtype
        self.ctx = ctypes.c_void_p()
        _lib.check(self.lib.moe_sparse_init(ctypes.byref(self.desc), ctypes.byref(self.ctx)),
                   "moe_sparse_init")
        self._last = None
        self._keep = ()

    # -------------------------------------------------------------- helpers
    def _check(self, t: torch.Tensor, name: str, dtype=None) -> None:
        dtype = dtype or self.torch_dtype
        if t.device != self.device:
            raise ValueError(f"{name} must be on {self.device}, got {t.device}")
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    @staticmethod
    def _stream(stream) -> int:
        if stream is None:
            stream = torch.cuda.current_stream()
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)

    # -------------------------------------------------------------- API
    def set_shared(self, Wg_s: torch.Tensor, Wu_s: torch.Tensor, Wd_s: torch.Tensor,
                   tau_shared: float) -> None:
        for t, n in ((Wg_s, "Wg_s"), (Wu_s, "Wu_s"), (Wd_s, "Wd_s")):
            self._check(t, n)
        self._keep = (Wg_s, Wu_s, Wd_s)
        _lib.check(self.lib.moe_sparse_set_shared(self.ctx, _ptr(Wg_s), _ptr(Wu_s), _ptr(Wd_s),
                                                  float(tau_shared)),
                   "moe_sparse_set_shared", self.ctx)

    def forward(self, x: torch.Tensor, W_router: torch.Tensor, W_gate: torch.Tensor,
                W_up: torch.Tensor, W_down: torch.Tensor, tau: float, top_k: int,
                router_bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        for t, n in ((x, "x"), (W_router, "W_router"), (W_gate, "W_gate"), (W_up, "W_up"),
                     (W_down, "W_down")):
            self._check(t, n)
        if router_bias is not None:
            self._check(router_bias, "router_bias", torch.float32)
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.d_model), dtype=self.out_dtype, device=self.device)
        else:
            self._check(out, "out", self.out_dtype)
        _lib.check(self.lib.moe_sparse_forward(
            self.ctx, _ptr(x), T, _ptr(W_router), _ptr(router_bias), _ptr(W_gate), _ptr(W_up),
            _ptr(W_down), float(tau), int(top_k), _ptr(out), self._stream(stream)),
            "moe_sparse_forward", self.ctx)
        self._last = (T, int(top_k))
        return out

    def debug(self, stream=None) -> dict:
        """Routing and active bitmaps of the last forward, pair order t*top_k+i."""
        T, k = self._last
        dev = self.device
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        res = {"topk_idx": idx, "topk_w": w}
        bits = bits_s = None
        if self.desc.debug:
            bits = torch.empty((T * k, (self.d_ff + 31) // 32), dtype=torch.int32, device=dev)
            res["active_bits"] = bits
            if self.n_shared:
                bits_s = torch.empty((self.n_shared, T, (self.d_ff_shared + 31) // 32),
                                     dtype=torch.int32, device=dev)
                res["active_bits_shared"] = bits_s
        _lib.check(self.lib.moe_sparse_get_debug(self.ctx, _ptr(idx), _ptr(w), _ptr(bits),
                                                 _ptr(bits_s), self._stream(stream)),
                   "moe_sparse_get_debug", self.ctx)
        return res

    def stats(self, stream=None) -> dict:
        s = _lib.moe_stats()
        _lib.check(self.lib.moe_sparse_get_stats(self.ctx, ctypes.byref(s), self._stream(stream)),
                   "moe_sparse_get_stats", self.ctx)
        return {n: getattr(s, n) for n, _ in _lib.moe_stats._fields_}

    def status(self) -> int:
        v = ctypes.c_int32()
        _lib.check(self.lib.moe_sparse_get_status(self.ctx, ctypes.byref(v)),
                   "moe_sparse_get_status", self.ctx)
        return v.value

    def set_timing(self, ring: int) -> None:
        """Record per-stage CUDA events for the last ``ring`` forwards (0: off)."""
        _lib.check(self.lib.moe_sparse_set_timing(self.ctx, int(ring)),
                   "moe_sparse_set_timing", self.ctx)

    def timing(self) -> dict:
        """Stage milliseconds of the last timed forward."""
        arr = (ctypes.c_float * len(_lib.STAGES))()
        _lib.check(self.lib.moe_sparse_get_timing(self.ctx, arr, len(_lib.STAGES)),
                   "moe_sparse_get_timing", self.ctx)
        return dict(zip(_lib.STAGES, list(arr)))

    def timing_all(self, max_forwards: int = 4096) -> list:
        """Stage milliseconds of every timed forward since the last call."""
        ns = len(_lib.STAGES)
        arr = (ctypes.c_float * (ns * max_forwards))()
        n = ctypes.c_int32()
        _lib.check(self.lib.moe_sparse_get_timing_all(self.ctx, arr, ns, max_forwards,
                                                      ctypes.byref(n)),
                   "moe_sparse_get_timing_all", self.ctx)
        return [dict(zip(_lib.STAGES, arr[f * ns:(f + 1) * ns])) for f in range(n.value)]

    def launch_count(self) -> int:
        n = ctypes.c_int64()
        _lib.check(self.lib.moe_sparse_launch_count(self.ctx, ctypes.byref(n)),
                   "moe_sparse_launch_count", self.ctx)
        return n.value

    def close(self) -> None:
        if self.ctx:
            self.lib.moe_sparse_destroy(self.ctx)
            self.ctx = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
