"""ctypes binding of ``libmoe_b200.so`` (the C ABI declared in include/moe.h).

Argument marshalling only: every step of the forward pass runs in the
library's CUDA kernels. There is no fallback: if the library is missing or a
call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_uint32, c_void_p

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
# The library to load: the normal build, or another build of the same sources
# (e.g. libmoe_b200_debug.so, the MOE_DEBUG_BOUNDS build) named by
# MOE_B200_LIBRARY (a file name inside the package, or a path).
LIB_NAME = os.environ.get("MOE_B200_LIBRARY", "libmoe_b200.so")
LIB_PATH = LIB_NAME if os.path.isabs(LIB_NAME) else os.path.join(PKG_DIR, LIB_NAME)
MOE_BUILD_DEBUG_BOUNDS = 1

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_MISALIGNED = 0, 1, 2, 3
MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_DEVICE_CHECK = 4, 5, 6
MOE_F32, MOE_BF16, MOE_BF16_INT8W = 0, 1, 2
MOE_ACT_GELU_TANH, MOE_ACT_GELU_ERF, MOE_ACT_SILU = 0, 1, 2
MOE_PATH_AUTO, MOE_PATH_TOKEN_TILE, MOE_PATH_WEIGHT_STREAM, MOE_PATH_TOKEN_TILE_SINGLE = 0, 1, 2, 3

# Every function include/moe.h exports, with (restype, argtypes).
EXPORTS = {}


class MoeScales(ctypes.Structure):
    _fields_ = [("s_gate", c_void_p), ("s_up", c_void_p), ("s_down", c_void_p)]


class MoeArgs(ctypes.Structure):
    _fields_ = [("x", c_void_p), ("w_router", c_void_p), ("w_gate", c_void_p), ("w_up", c_void_p),
                ("w_down", c_void_p), ("w_scales", POINTER(MoeScales)), ("out", c_void_p),
                ("T", c_int64), ("d", c_int64), ("f", c_int64), ("E", c_int32), ("k", c_int32),
                ("dtype", c_int)]


class MoeOptions(ctypes.Structure):
    _fields_ = [("activation", c_int), ("router_bias", c_void_p), ("path", c_int), ("down_splits", c_int32),
                ("stage_events", POINTER(c_void_p)), ("renormalize", c_int32), ("residual", c_void_p),
                ("post_norm_weight", c_void_p), ("norm_eps", c_float), ("row_gather", c_int32),
                ("separate_combine", c_int32)]


class MoeDebug(ctypes.Structure):
    _fields_ = [("idx", c_void_p), ("gates", c_void_p), ("counts", c_void_p), ("offsets", c_void_p),
                ("perm_token", c_void_p), ("perm_slot", c_void_p), ("h", c_void_p)]


class MoeRouted(ctypes.Structure):
    _fields_ = [("idx", c_void_p), ("gates", c_void_p), ("counts", c_void_p), ("offsets", c_void_p),
                ("perm_token", c_void_p), ("perm_slot", c_void_p), ("slot_pos", c_void_p),
                ("gate_perm", c_void_p), ("xp", c_void_p)]


class MoeExpertRows(ctypes.Structure):
    _fields_ = [("xp", c_void_p), ("counts", c_void_p), ("gate", c_void_p), ("w_gate", c_void_p),
                ("w_up", c_void_p), ("w_down", c_void_p), ("w_scales", POINTER(MoeScales)), ("y", c_void_p),
                ("R", c_int64), ("d", c_int64), ("f", c_int64), ("n_experts", c_int32), ("dtype", c_int)]


EXPORTS.update({
    "moe_forward": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, POINTER(MoeScales), c_void_p,
                            c_int64, c_int64, c_int64, c_int32, c_int32, c_int, c_void_p]),
    "moe_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int32, c_int32, c_int]),
    "moe_workspace_size_ex": (c_size_t, [c_int64, c_int64, c_int64, c_int32, c_int32, c_int, c_int, c_int32]),
    "moe_forward_ex": (c_int, [POINTER(MoeArgs), POINTER(MoeOptions), POINTER(MoeDebug), c_void_p, c_size_t,
                               c_void_p]),
    "moe_forward_noalloc": (c_int, [POINTER(MoeArgs), POINTER(MoeOptions), c_void_p]),
    "moe_device_status": (c_int, [c_void_p, c_void_p, POINTER(c_uint32)]),
    "moe_selftest_bounded_wait": (c_int, [c_void_p, c_uint32, c_void_p]),
    "moe_status_string": (c_char_p, [c_int]),
    "moe_abi_version": (c_int32, []),
    "moe_build_flags": (c_int32, []),
    "moe_route_workspace_size": (c_size_t, [c_int64, c_int64, c_int]),
    "moe_route_dispatch": (c_int, [c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int, c_int32,
                                   POINTER(MoeRouted), c_void_p, c_size_t, c_void_p]),
    "moe_experts_workspace_size": (c_size_t, [c_int64, c_int64, c_int64, c_int32, c_int, c_int, c_int32]),
    "moe_experts_forward": (c_int, [POINTER(MoeExpertRows), POINTER(MoeOptions), c_void_p, c_size_t, c_void_p]),
    "moe_combine": (c_int, [c_void_p, c_void_p, c_int64, c_int64, c_int, c_void_p, c_void_p, c_float, c_void_p,
                            c_void_p, c_size_t, c_void_p]),
    "moe_gather_rows": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int64, c_void_p, c_void_p, c_size_t,
                                c_void_p]),
})

_LIB = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library once; raise if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mixture_experts_ffn_14_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB
