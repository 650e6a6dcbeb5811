"""The allocation-free forward entry point (moe_forward_noalloc), called through
the C ABI, against the workspace entry point (moe_forward_ex) on the same
inputs, on two calls in a row with different batches (so the second call
cannot pass on what the first left in the shared scratch).

This file is collected last on purpose: it runs after every other test, and
also passes alone in a fresh process (the first call sets up the scratch)."""

import numpy as np
import pytest
import torch

import mixture_experts_ffn_14_b200 as moe
from mixture_experts_ffn_14_b200 import workloads as W

from _harness import ATOL, RTOL, full_check, np64, run_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _ex(inp, x, **kw):
    T, d = x.shape
    f = inp["w_gate"].shape[2]
    dt = moe.dtype_code(x, inp["w_gate"])
    ws = torch.empty(moe.moe_workspace_size(T, d, f, dtype=dt, path=kw.get("path", 0)), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty_like(x)
    scales = (inp["s_gate"], inp["s_up"], inp["s_down"]) if "s_gate" in inp else None
    moe.moe_forward_ex(x, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out, ws, scales=scales,
                       router_bias=inp.get("router_bias"), **kw)
    return out


def _noalloc(inp, x, **kw):
    out = torch.empty_like(x)
    scales = (inp["s_gate"], inp["s_up"], inp["s_down"]) if "s_gate" in inp else None
    moe.moe_forward_noalloc(x, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out, scales=scales,
                            router_bias=inp.get("router_bias"), **kw)
    return out


def _close(a, b):
    a, b = np64(a), np64(b)
    assert (np.abs(a - b) <= ATOL + RTOL * np.abs(b)).all()


SCRATCH = 32 << 20   # the fixed scratch of moe_forward_noalloc


def _against_oracle(inp, x, got):
    """The noalloc output for batch x against the oracle: the routing comes
    from a workspace call on the same batch (checked bit for bit against the
    oracle's), the output element by element at the stated tolerance."""
    case = dict(inp)
    case["x"] = x
    gpu = run_gpu(case, want_h=False)
    gpu["out"] = np64(got)
    return full_check(case, gpu, check_h=False)


@pytest.mark.parametrize("dtype", ["bf16", "bf16_int8w"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    w = W.Workload("noalloc", 64, 1024, 2048, dtype=dtype, seed=41)
    inp = W.make_torch(w, DEV)
    xs = [inp["x"], W.make_x(w, DEV, 64, seed_name="x_second")]
    for x in xs:
        got = _noalloc(inp, x)
        ref = _ex(inp, x)
        torch.cuda.synchronize()
        _close(got, ref)


def test_noalloc_f32_and_token_tile_path():
    p = W.make_numpy(64, 128, 256, seed=3)
    inp = {k: torch.from_numpy(v).to(DEV) for k, v in p.items()}
    x2 = torch.from_numpy(W.make_numpy(64, 128, 256, seed=4)["x"]).to(DEV)
    for x in (inp["x"], x2):
        _close(_noalloc(inp, x), _ex(inp, x))
    w = W.Workload("noalloc_tt", 200, 512, 512, dtype="bf16", seed=42)
    inp = W.make_torch(w, DEV)
    for x in (inp["x"], W.make_x(w, DEV, 200, seed_name="x_second")):
        _close(_noalloc(inp, x, path=moe.MOE_PATH_TOKEN_TILE), _ex(inp, x, path=moe.MOE_PATH_TOKEN_TILE))
    torch.cuda.synchronize()


def test_noalloc_rejects_problems_beyond_the_scratch():
    w = W.Workload("noalloc_big", 4096, 512, 2048, dtype="bf16", seed=43)
    inp = W.make_torch(w, DEV)
    out = torch.empty_like(inp["x"])
    st = moe.moe_forward_noalloc(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out,
                                 raise_on_error=False)
    assert st == 4  # MOE_ERR_WORKSPACE: needs more than the 32 MiB fixed scratch


def test_noalloc_status_word_is_readable():
    # A noalloc caller has no workspace pointer: moe_device_status(NULL) reads
    # the fixed scratch's status word too.
    w = W.Workload("noalloc_status", 64, 256, 256, dtype="bf16", seed=44)
    inp = W.make_torch(w, DEV)
    _noalloc(inp, inp["x"])
    st, code = moe.moe_device_status()
    assert st == 0 and code == 0


def test_noalloc_zero_tokens_returns_ok():
    w = W.Workload("noalloc_empty", 64, 256, 256, dtype="bf16", seed=45)
    inp = W.make_torch(w, DEV)
    x0 = inp["x"][:0]
    out = torch.empty_like(x0)
    assert moe.moe_forward_noalloc(x0, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out,
                                   raise_on_error=False) == 0


def test_noalloc_tiny_f32_matches_oracle_twice():
    p = W.make_numpy(64, 128, 256, seed=0)
    inp = {k: torch.from_numpy(v).to(DEV) for k, v in p.items()}
    x2 = torch.from_numpy(W.make_numpy(64, 128, 256, seed=5)["x"]).to(DEV)
    for x in (inp["x"], x2):
        got = _noalloc(inp, x)
        torch.cuda.synchronize()
        _against_oracle(inp, x, got)


def test_noalloc_lowers_split_k_to_fit_the_scratch():
    # bf16, T = 64, d = 2048, f = 16384: the automatic split-K factor (32)
    # needs more than the fixed scratch, 16 fits: the entry point must lower it.
    T, d, f = 64, 2048, 16384
    assert moe.moe_workspace_size(T, d, f, dtype=moe.MOE_BF16) > SCRATCH
    assert moe.moe_workspace_size(T, d, f, dtype=moe.MOE_BF16, down_splits=16) <= SCRATCH
    w = W.Workload("noalloc_lower", T, d, f, dtype="bf16", seed=46)
    inp = W.make_torch(w, DEV)
    for x in (inp["x"], W.make_x(w, DEV, T, seed_name="x_second")):
        got = _noalloc(inp, x)
        ref = _ex(inp, x, down_splits=16)
        torch.cuda.synchronize()
        assert torch.equal(got, ref)   # same kernels, same split factor: bitwise
        _against_oracle(inp, x, got)


@pytest.mark.slow
def test_noalloc_grok_decode_shape_matches_oracle():
    # The decode shape the header names (T = 64, d = 6144, f = 32768, bf16):
    # its automatic split-K factor does not fit and is lowered.
    wl = W.WORKLOADS["decode"]
    assert moe.moe_workspace_size(wl.T, wl.d, wl.f, dtype=moe.MOE_BF16) > SCRATCH
    inp = W.make_torch(wl, DEV)
    got = _noalloc(inp, inp["x"])
    torch.cuda.synchronize()
    st, code = moe.moe_device_status()
    assert st == 0 and code == 0
    _against_oracle(inp, inp["x"], got)
    del inp
    torch.cuda.empty_cache()
