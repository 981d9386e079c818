"""ctypes binding of libmoe_ffn.so, one Python function per C entry point.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. There is no fallback: if the library is missing or fails to load,
``load_library`` raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional

from .build import lib_path

__all__ = ["MoEError", "load_library", "EXPORTED_SYMBOLS", "Plan", "STATUS_NAMES"]

# Every function include/moe_ffn.h declares.
EXPORTED_SYMBOLS = [
    "moe_plan_create", "moe_last_status", "moe_plan_set_logit_bias", "moe_workspace_bytes",
    "moe_plan_set_workspace", "moe_forward", "moe_get_routing", "moe_get_permutation",
    "moe_plan_device_status", "moe_plan_enable_timing", "moe_plan_kernel_times",
    "moe_plan_kernel_name", "moe_plan_last_launch_count", "moe_plan_destroy", "moe_strerror",
    "moe_last_error", "moe_forward_noalloc", "moe_plan_set_option", "moe_plan_capacity_seats",
]
MOE_OPTION_PAIR_MIN_ROWS = 1
MOE_OPTION_WIDE_TILES = 2
MOE_OPTION_MERGE_SHARED = 3
MOE_OPTION_EXPERT_CAPACITY = 4
MOE_OPTION_BIAS_SELECTION_ONLY = 5
MOE_OPTION_CAPACITY_FACTOR_PERMILLE = 6
MOE_OPTION_FUSED_ROUTER = 7
MOE_OPTION_SWIGLU_TILE_COLS = 8
MOE_OPTION_SHARED_CONCURRENT = 9
MOE_OPTION_TILE_ROWS = 10
MOE_OPTION_INTERLEAVE = 11
MOE_OPTION_CTAS_PER_SM = 12
MOE_OPTION_DOWN_TILE_COLS = 13
MOE_OPTION_GATHER_ROWS = 14
MOE_OPTION_TEST_WAIT_TIMEOUT = 100

STATUS_NAMES = {0: "MOE_OK", 1: "MOE_INVALID_CONFIG", 2: "MOE_INVALID_ARG",
                3: "MOE_WORKSPACE_TOO_SMALL", 4: "MOE_CUDA_ERROR", 5: "MOE_UNSUPPORTED",
                6: "MOE_DEVICE_TIMEOUT", 7: "MOE_DEVICE_INCONSISTENT"}


class MoEError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_LIB: Optional[ctypes.CDLL] = None

_vp, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or lib_path()
    if not os.path.exists(p):
        raise MoEError(4, f"CUDA library not found at {p}; build it with "
                          "`python -m mixture_experts_ffn_expert_b200.build`")
    lib = ctypes.CDLL(p)
    sig = {
        "moe_plan_create": (_vp, [_i, _i, _i, _i, _i, _i]),
        "moe_last_status": (_i, []),
        "moe_plan_set_option": (_i, [_vp, _i, _i64]),
        "moe_plan_set_logit_bias": (_i, [_vp, _vp]),
        "moe_workspace_bytes": (_sz, [_vp, _i64]),
        "moe_plan_set_workspace": (_i, [_vp, _vp, _sz]),
        "moe_forward": (_i, [_vp, _i64] + [_vp] * 10),
        "moe_forward_noalloc": (_i, [_vp, _i64] + [_vp] * 10),
        "moe_get_routing": (_i, [_vp, _i64, _vp, _vp, _vp, _vp, _vp]),
        "moe_get_permutation": (_i, [_vp, _i64, _vp, _vp, _vp]),
        "moe_plan_device_status": (_i, [_vp]),
        "moe_plan_enable_timing": (_i, [_vp, _i]),
        "moe_plan_kernel_times": (_i, [_vp, _i, ctypes.POINTER(ctypes.c_float), _i]),
        "moe_plan_kernel_name": (ctypes.c_char_p, [_vp, _i]),
        "moe_plan_last_launch_count": (_i, [_vp]),
        "moe_plan_capacity_seats": (_i64, [_vp, _i64]),
        "moe_plan_destroy": (None, [_vp]),
        "moe_strerror": (ctypes.c_char_p, [_i]),
        "moe_last_error": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _LIB = lib
    return lib


def _check(lib, status: int):
    if status != 0:
        raise MoEError(status, (lib.moe_last_error() or b"").decode())


class Plan:
    """Owns one ``moe_plan_t``. Pointers and streams are plain integers."""

    def __init__(self, d: int, f: int, n_routed: int, top_k: int, n_shared: int,
                 renorm: bool):
        self.lib = load_library()
        self.d, self.f, self.n_routed, self.top_k = d, f, n_routed, top_k
        self.n_shared, self.renorm = n_shared, bool(renorm)
        h = self.lib.moe_plan_create(d, f, n_routed, top_k, n_shared, int(bool(renorm)))
        if not h:
            raise MoEError(self.lib.moe_last_status(), (self.lib.moe_last_error() or b"").decode())
        self.handle = h

    def set_option(self, option: int, value: int) -> None:
        _check(self.lib, self.lib.moe_plan_set_option(self.handle, option, value))

    def workspace_bytes(self, T: int) -> int:
        return int(self.lib.moe_workspace_bytes(self.handle, T))

    def set_workspace(self, ptr: int, nbytes: int) -> None:
        _check(self.lib, self.lib.moe_plan_set_workspace(self.handle, ptr or None, nbytes))

    def set_logit_bias(self, ptr: Optional[int]) -> None:
        _check(self.lib, self.lib.moe_plan_set_logit_bias(self.handle, ptr or None))

    def forward(self, T: int, x: int, W_g: int, W1: int, W3: int, W2: int,
                W1s: Optional[int], W3s: Optional[int], W2s: Optional[int], out: int,
                stream: int = 0) -> None:
        _check(self.lib, self.lib.moe_forward(self.handle, T, x, W_g, W1, W3, W2,
                                              W1s or None, W3s or None, W2s or None, out,
                                              stream or None))

    def get_routing(self, T: int, idx: Optional[int], w: Optional[int], counts: Optional[int],
                    offsets: Optional[int], stream: int = 0) -> None:
        _check(self.lib, self.lib.moe_get_routing(self.handle, T, idx or None, w or None,
                                                  counts or None, offsets or None,
                                                  stream or None))

    def get_permutation(self, T: int, perm_src: Optional[int], inv_pos: Optional[int],
                        stream: int = 0) -> None:
        _check(self.lib, self.lib.moe_get_permutation(self.handle, T, perm_src or None,
                                                      inv_pos or None, stream or None))

    def device_status(self) -> int:
        return int(self.lib.moe_plan_device_status(self.handle))

    def enable_timing(self, on: bool = True) -> None:
        _check(self.lib, self.lib.moe_plan_enable_timing(self.handle, int(on)))

    def kernel_times(self, back: int = 0) -> List[float]:
        """Per-kernel milliseconds of the timed forward `back` steps before the latest."""
        buf = (ctypes.c_float * 16)()
        n = self.lib.moe_plan_kernel_times(self.handle, back, buf, 16)
        if n < 0:
            _check(self.lib, -n)
        return [float(buf[i]) for i in range(min(n, 16))]

    def kernel_names(self) -> List[str]:
        n = self.lib.moe_plan_last_launch_count(self.handle)
        return [(self.lib.moe_plan_kernel_name(self.handle, i) or b"?").decode()
                for i in range(min(n, 16))]

    def last_launch_count(self) -> int:
        return int(self.lib.moe_plan_last_launch_count(self.handle))

    def capacity_seats(self, T: int) -> int:
        """Seats per expert a forward over T tokens uses (0: dropless)."""
        n = int(self.lib.moe_plan_capacity_seats(self.handle, T))
        if n < 0:
            _check(self.lib, -n)
        return n

    def close(self) -> None:
        if getattr(self, "handle", None):
            self.lib.moe_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
