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

from _harness import ATOL, RTOL, np64

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
