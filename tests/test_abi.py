"""C ABI checks that need no GPU: the library loads, exports every function
include/moe.h declares, and rejects bad arguments on the host with the
documented status before touching the device."""

import ctypes
import os
import re

import pytest

import mixture_experts_ffn_14_b200 as moe
from mixture_experts_ffn_14_b200 import _native as N
from mixture_experts_ffn_14_b200 import build as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(N.LIB_PATH):
        B.build()
    return N.lib()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"MOE_EXPORT\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)


def test_every_declared_function_is_exported():
    names = declared_functions()
    assert set(names) == set(N.EXPORTS), (names, sorted(N.EXPORTS))
    raw = ctypes.CDLL(N.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_status_strings_and_version():
    assert moe.moe_abi_version() == 2
    texts = {moe.moe_status_string(s) for s in range(7)}
    assert len(texts) == 7
    assert moe.moe_status_string(99) == "unknown status"


def test_workspace_size_rules():
    ws = moe.moe_workspace_size
    assert ws(4096, 6144, 32768) > 0
    assert ws(64, 128, 256, dtype=moe.MOE_F32) > 0
    assert ws(0, 6144, 32768) == 0                      # nothing to do
    assert ws(-1, 6144, 32768) == 0
    assert ws(64, 6144, 32768, E=7) == 0                # E != 8
    assert ws(64, 6144, 32768, k=1) == 0                # k != 2
    assert ws(64, 6000, 32768) == 0                     # d % 256
    assert ws(64, 6144, 32700) == 0                     # f % 128
    assert ws(64, 96, 256, dtype=moe.MOE_F32) == 0      # fp32 d % 64
    assert ws(64, 6144, 32768, dtype=7) == 0
    assert ws(64, 6144, 32768, down_splits=7) == 0      # 512 K blocks not divisible by 7
    assert ws(64, 6144, 32768, path=9) == 0
    assert ws(1000, 6144, 32768) < ws(2000, 6144, 32768)
    # the weight-stream path keeps split-K partial sums: more bytes than one split
    one = ws(64, 6144, 32768, path=moe.MOE_PATH_WEIGHT_STREAM, down_splits=1)
    eight = ws(64, 6144, 32768, path=moe.MOE_PATH_WEIGHT_STREAM, down_splits=8)
    assert eight - one >= 7 * 128 * 6144 * 4
    assert ws(64, 6144, 32768) % 256 == 0
    # the six-argument C call is the _ex call with the automatic choices
    for T, d, f, dt in ((4096, 6144, 32768, 1), (64, 6144, 32768, 1), (1024, 6144, 32768, 2), (64, 128, 256, 0)):
        assert N.lib().moe_workspace_size(T, d, f, 8, 2, dt) == N.lib().moe_workspace_size_ex(T, d, f, 8, 2, dt, 0, 0)


def test_form_and_split_choices_at_the_grok_shape():
    # Seen through the workspace size (weight-stream layouts keep four combine
    # counters per token and column tile, and every split its own fp32 partial
    # sums). Weight-stream form up to 128 tokens with bf16 weights, up to 256
    # with int8 weights; token tiles above.
    d, f = 6144, 32768

    def ws(T, dt, path=moe.MOE_PATH_AUTO, splits=0):
        return moe.moe_workspace_size(T, d, f, dtype=dt, path=path, down_splits=splits)

    for dt, last in ((moe.MOE_BF16, 128), (moe.MOE_BF16_INT8W, 256)):
        assert ws(last, dt) == ws(last, dt, moe.MOE_PATH_WEIGHT_STREAM)
        assert ws(last + 1, dt) != ws(last + 1, dt, moe.MOE_PATH_WEIGHT_STREAM)
    # the token-tile down projection's split factor (a measured model): two
    # splits for a few rows per expert, none once the tiles fill the SMs
    for dt, T, want in ((moe.MOE_BF16, 384, 2), (moe.MOE_BF16, 768, 1), (moe.MOE_BF16, 4096, 1),
                        (moe.MOE_BF16_INT8W, 768, 2), (moe.MOE_BF16_INT8W, 1024, 1)):
        got = [s for s in (1, 2, 4, 8) if ws(T, dt, splits=s) == ws(T, dt)]
        assert got == [want], (dt, T, got)


def _args(T=64, d=512, f=384, E=8, k=2, dtype=moe.MOE_BF16, base=0x10000000):
    # Fake, never dereferenced device addresses: every call below must return
    # from the host-side checks before any CUDA call.
    a = N.MoeArgs(base, base + 0x1000, base + 0x2000, base + 0x3000, base + 0x4000, None, base + 0x5000,
                  T, d, f, E, k, dtype)
    return a


def _call(a, ws=0x20000000, ws_bytes=1 << 40, opts=None):
    return N.lib().moe_forward_ex(ctypes.byref(a), ctypes.byref(opts) if opts else None, None, ws, ws_bytes, None)


def test_forward_ex_host_checks():
    assert _call(_args(T=0)) == N.MOE_OK                       # T = 0: no-op
    assert N.lib().moe_forward_ex(None, None, None, None, 0, None) == N.MOE_ERR_INVALID_ARG
    a = _args()
    a.x = None
    assert _call(a) == N.MOE_ERR_INVALID_ARG
    assert _call(_args(E=4)) == N.MOE_ERR_UNSUPPORTED
    assert _call(_args(k=1)) == N.MOE_ERR_UNSUPPORTED
    assert _call(_args(d=500)) == N.MOE_ERR_UNSUPPORTED
    assert _call(_args(T=-3)) == N.MOE_ERR_INVALID_ARG
    assert _call(_args(T=(1 << 24) + 1)) == N.MOE_ERR_UNSUPPORTED
    assert _call(_args(dtype=5)) == N.MOE_ERR_INVALID_ARG
    a = _args()
    a.w_up = a.w_up + 4
    assert _call(a) == N.MOE_ERR_MISALIGNED
    a = _args(dtype=moe.MOE_BF16_INT8W)
    assert _call(a) == N.MOE_ERR_INVALID_ARG                   # int8 without scales
    sc = N.MoeScales(0x30000000, 0x30001000, 0x30002008)
    a.w_scales = ctypes.pointer(sc)
    assert _call(a) == N.MOE_ERR_MISALIGNED
    assert _call(_args(), ws=0) == N.MOE_ERR_WORKSPACE
    assert _call(_args(), ws=0x20000010) == N.MOE_ERR_WORKSPACE  # not 256-aligned
    assert _call(_args(), ws_bytes=1024) == N.MOE_ERR_WORKSPACE
    bad = N.MoeOptions(7, None, 0, 0)
    assert _call(_args(), opts=bad) == N.MOE_ERR_INVALID_ARG
    bad = N.MoeOptions(0, None, 0, -2)
    assert _call(_args(), opts=bad) == N.MOE_ERR_INVALID_ARG
    bad = N.MoeOptions(0, 0x40000004, 0, 0)
    assert _call(_args(), opts=bad) == N.MOE_ERR_MISALIGNED
    bad = N.MoeOptions(0, None, 1, 5)   # 6 K blocks of f=384 are not divisible by 5
    assert _call(_args(), opts=bad) == N.MOE_ERR_UNSUPPORTED


def test_forward_host_checks():
    f = N.lib().moe_forward
    assert f(None, None, None, None, None, None, None, 0, 512, 384, 8, 2, 1, None) == N.MOE_OK
    assert f(None, None, None, None, None, None, None, 5, 512, 384, 8, 2, 1, None) == N.MOE_ERR_INVALID_ARG
    assert f(None, None, None, None, None, None, None, 5, 512, 384, 6, 2, 1, None) == N.MOE_ERR_UNSUPPORTED


def test_binding_refuses_host_tensors():
    import torch

    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    w = torch.zeros(8, 256, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        moe.moe_forward(x, torch.zeros(256, 8), w, w, torch.zeros(8, 128, 256, dtype=torch.bfloat16),
                        torch.empty_like(x), stream=0)


def test_option_checks():
    a = _args()
    bad = N.MoeOptions(3, None, 0, 0, None, 0, None, None, 0.0)      # no such activation
    assert _call(a, opts=bad) == N.MOE_ERR_INVALID_ARG
    bad = N.MoeOptions(0, None, 0, 0, None, 2, None, None, 0.0)      # renormalize must be 0 or 1
    assert _call(a, opts=bad) == N.MOE_ERR_INVALID_ARG
    bad = N.MoeOptions(0, None, 0, 0, None, 0, None, 0x50000000, 0.0)  # post-norm needs eps > 0
    assert _call(a, opts=bad) == N.MOE_ERR_INVALID_ARG
    bad = N.MoeOptions(0, None, 0, 0, None, 0, None, 0x50000004, 1e-5)
    assert _call(a, opts=bad) == N.MOE_ERR_MISALIGNED
    bad = N.MoeOptions(0, None, 0, 0, None, 0, 0x50000008, None, 0.0)
    assert _call(a, opts=bad) == N.MOE_ERR_MISALIGNED
    bad = N.MoeOptions(0, None, 0, 0, None, 0, None, None, 0.0, 2)   # row_gather must be 0 or 1
    assert _call(a, opts=bad) == N.MOE_ERR_INVALID_ARG


def test_selftest_argument_checks():
    f = N.lib().moe_selftest_bounded_wait
    assert f(None, 1000, None) == N.MOE_ERR_WORKSPACE
    assert f(0x20000010, 1000, None) == N.MOE_ERR_WORKSPACE      # not 256-byte aligned
    assert f(0x20000000, 0, None) == N.MOE_ERR_INVALID_ARG
    assert f(0x20000000, 20_000_000, None) == N.MOE_ERR_INVALID_ARG
