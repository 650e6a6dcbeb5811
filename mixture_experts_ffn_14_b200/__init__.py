"""B200 (sm_100a) Grok-1 MoE feed-forward sublayer: Python binding of the C ABI.

Functions carry the C names (include/moe.h) and take torch CUDA tensors; they
only marshal arguments into ``libmoe_b200.so``. Errors raise ``MoeError``.

    import torch, mixture_experts_ffn_14_b200 as moe
    out = torch.empty_like(x)
    moe.moe_forward(x, w_router, w_gate, w_up, w_down, out)
"""

from __future__ import annotations

import ctypes

from . import _native as N
from ._native import (  # noqa: F401
    MOE_ACT_GELU_ERF, MOE_ACT_GELU_TANH, MOE_ACT_SILU, MOE_BF16, MOE_BF16_INT8W, MOE_F32, MOE_PATH_AUTO,
    MOE_PATH_TOKEN_TILE, MOE_PATH_TOKEN_TILE_SINGLE, MOE_PATH_WEIGHT_STREAM,
)

__all__ = ["MoeError", "moe_forward", "moe_forward_ex", "moe_forward_noalloc", "moe_workspace_size",
           "moe_workspace_size_ex", "moe_build_flags",
           "moe_device_status", "moe_selftest_bounded_wait", "moe_status_string", "moe_abi_version",
           "dtype_code"]


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {moe_status_string(status)} (status {status})")


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("moe: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("moe: tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch

    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def dtype_code(x, w_gate) -> int:
    import torch

    if w_gate.dtype == torch.int8:
        return MOE_BF16_INT8W
    if x.dtype == torch.float32:
        return MOE_F32
    return MOE_BF16


def _scales(scales):
    if scales is None:
        return None
    sg, su, sd = scales
    return N.MoeScales(_ptr(sg), _ptr(su), _ptr(sd))


def moe_status_string(status: int) -> str:
    return N.lib().moe_status_string(status).decode()


def moe_abi_version() -> int:
    return N.lib().moe_abi_version()


def moe_build_flags() -> int:
    """Build options of the loaded library (bit MOE_BUILD_DEBUG_BOUNDS)."""
    return N.lib().moe_build_flags()


def moe_workspace_size(T, d, f, E=8, k=2, dtype=MOE_BF16, path=MOE_PATH_AUTO, down_splits=0) -> int:
    """Workspace bytes of a moe_forward_ex call; the C call with the automatic
    kernel choices, or its _ex form when ``path`` / ``down_splits`` are set."""
    if path == MOE_PATH_AUTO and down_splits == 0:
        return N.lib().moe_workspace_size(T, d, f, E, k, dtype)
    return N.lib().moe_workspace_size_ex(T, d, f, E, k, dtype, path, down_splits)


def moe_workspace_size_ex(T, d, f, E=8, k=2, dtype=MOE_BF16, path=MOE_PATH_AUTO, down_splits=0) -> int:
    return N.lib().moe_workspace_size_ex(T, d, f, E, k, dtype, path, down_splits)


def moe_forward(x, w_router, w_gate, w_up, w_down, out, scales=None, stream=None):
    """out[T, d] = MoE FFN of x[T, d] (library-owned workspace)."""
    T, d = x.shape
    E, _, f = w_gate.shape
    sc = _scales(scales)
    st = N.lib().moe_forward(_ptr(x), _ptr(w_router), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                             ctypes.byref(sc) if sc is not None else None, _ptr(out),
                             T, d, f, E, 2, dtype_code(x, w_gate), _stream(stream))
    if st != N.MOE_OK:
        raise MoeError(st, "moe_forward")
    return out


def _options(activation, router_bias, path, down_splits, stage_events, renormalize, residual, post_norm_weight,
             norm_eps, row_gather=False, separate_combine=False):
    ev = None
    if stage_events is not None:
        handles = [e.cuda_event for e in stage_events]
        if len(handles) != 6 or not all(handles):
            raise ValueError("moe: stage_events needs 6 created CUDA events")
        ev = (ctypes.c_void_p * 6)(*handles)
    opts = N.MoeOptions(activation, _ptr(router_bias), path, down_splits,
                        ctypes.cast(ev, ctypes.POINTER(ctypes.c_void_p)) if ev is not None else None,
                        int(bool(renormalize)), _ptr(residual), _ptr(post_norm_weight), float(norm_eps),
                        int(bool(row_gather)), int(bool(separate_combine)))
    return opts, ev


def moe_forward_ex(x, w_router, w_gate, w_up, w_down, out, workspace, scales=None, router_bias=None,
                   activation=MOE_ACT_GELU_TANH, path=MOE_PATH_AUTO, down_splits=0, debug=None, stream=None,
                   stage_events=None, renormalize=False, residual=None, post_norm_weight=None, norm_eps=1e-5,
                   row_gather=False, separate_combine=False, raise_on_error=True):
    """Forward pass on a caller workspace (a uint8 CUDA tensor). ``debug`` is a
    dict with any of idx, gates, counts, offsets, perm_token, perm_slot, h.
    ``stage_events``: 6 torch.cuda.Event (already created, e.g. recorded once)
    that the library records around its five stages. ``renormalize``,
    ``activation``, ``residual``, ``post_norm_weight`` / ``norm_eps``: the
    moe_options_t variants (Mixtral routing, SiLU, post-RMSNorm + residual).
    ``row_gather``: token tiles gather their gate/up rows from x with TMA row
    gathers instead of reading the dispatch stage's permuted copy.
    ``separate_combine``: sum each token's two expert rows in a combine kernel
    instead of the down projection's epilogue (same result bit for bit)."""
    T, d = x.shape
    E, _, f = w_gate.shape
    sc = _scales(scales)
    args = N.MoeArgs(_ptr(x), _ptr(w_router), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                     ctypes.pointer(sc) if sc is not None else None, _ptr(out), T, d, f, E, 2,
                     dtype_code(x, w_gate))
    opts, _keep = _options(activation, router_bias, path, down_splits, stage_events, renormalize, residual,
                           post_norm_weight, norm_eps, row_gather, separate_combine)
    dbg = None
    if debug:
        dbg = N.MoeDebug(*[_ptr(debug.get(n)) for n in
                           ("idx", "gates", "counts", "offsets", "perm_token", "perm_slot", "h")])
    ws_bytes = workspace.numel() * workspace.element_size()
    st = N.lib().moe_forward_ex(ctypes.byref(args), ctypes.byref(opts),
                                ctypes.byref(dbg) if dbg is not None else None,
                                _ptr(workspace), ws_bytes, _stream(stream))
    if st != N.MOE_OK and raise_on_error:
        raise MoeError(st, "moe_forward_ex")
    return st


def moe_forward_noalloc(x, w_router, w_gate, w_up, w_down, out, scales=None, router_bias=None,
                        activation=MOE_ACT_GELU_TANH, path=MOE_PATH_AUTO, down_splits=0, stream=None,
                        renormalize=False, residual=None, post_norm_weight=None, norm_eps=1e-5,
                        raise_on_error=True):
    """Forward pass that allocates no device memory: the library runs it in a
    fixed 32 MiB scratch array of its own, for callers that must not call
    cudaMalloc while they run (e.g. a framework that owns all device memory in
    a pre-reserved pool). Problems that need more scratch are rejected with
    MOE_ERR_WORKSPACE. Calls on one device share the scratch, so calls that
    may overlap on the GPU must be ordered by the caller."""
    T, d = x.shape
    E, _, f = w_gate.shape
    sc = _scales(scales)
    args = N.MoeArgs(_ptr(x), _ptr(w_router), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                     ctypes.pointer(sc) if sc is not None else None, _ptr(out), T, d, f, E, 2,
                     dtype_code(x, w_gate))
    opts, _ = _options(activation, router_bias, path, down_splits, None, renormalize, residual, post_norm_weight,
                       norm_eps)
    st = N.lib().moe_forward_noalloc(ctypes.byref(args), ctypes.byref(opts), _stream(stream))
    if st != N.MOE_OK and raise_on_error:
        raise MoeError(st, "moe_forward_noalloc")
    return st


def moe_selftest_bounded_wait(workspace, limit_us=1000, stream=None):
    """Launch the failure-path check: a bounded wait that nothing satisfies,
    recording status bit 0x10 in ``workspace`` (read it with moe_device_status)."""
    st = N.lib().moe_selftest_bounded_wait(_ptr(workspace), limit_us, _stream(stream))
    if st != N.MOE_OK:
        raise MoeError(st, "moe_selftest_bounded_wait")


def moe_device_status(workspace=None, stream=None):
    """(status, code) recorded by the kernels of the last call on ``workspace``."""
    code = ctypes.c_uint32(0)
    st = N.lib().moe_device_status(_ptr(workspace), _stream(stream), ctypes.byref(code))
    return st, code.value
