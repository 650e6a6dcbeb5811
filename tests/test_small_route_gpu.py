"""Router and dispatch for small batches (T <= 128) through the C ABI
(moe_route_dispatch), which runs them as one cluster launch. Each variant of
that kernel is covered:

- the permuted copy written from registers (T <= 64 with a short slice of x
  per CTA);
- the copy read again from x (T > 64, or a long slice: d = 12288 bf16,
  d = 8192 fp32);
- fp32, bf16 and int8-weight activations (the last converted to fp16);
- a router bias and renormalised gates.

Routing is checked against the oracle: experts bit-exact under the near-tie
rule, gates within tolerance. counts, offsets and the permutation are checked
bit-exact against the oracle's dispatch. slot_pos and gate_perm must agree with
the permutation, and every permuted row must equal its token's row of x
bit for bit (its fp16 rounding for int8 weights)."""

import numpy as np
import pytest
import torch

from mixture_experts_ffn_14_b200 import expert_parallel as EP
from mixture_experts_ffn_14_b200 import workloads as W

from _harness import check_routing_and_dispatch, expected_routing, np64

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = [
    ("bf16", 1, 256), ("bf16", 7, 6144), ("bf16", 64, 6144), ("bf16", 65, 6144), ("bf16", 128, 6144),
    ("bf16", 33, 12288), ("bf16", 128, 1024),
    ("f32", 1, 64), ("f32", 64, 4096), ("f32", 40, 8192), ("f32", 100, 512),
    ("bf16_int8w", 64, 6144), ("bf16_int8w", 97, 2048),
]


def _route(dtype, T, d, seed, bias=False, renormalize=False):
    wl = W.Workload("small", T, d, 128, dtype="f32" if dtype == "f32" else "bf16", seed=seed)
    x = W.make_x(wl, DEV, T)
    g = torch.Generator(device=DEV)
    g.manual_seed(1000 + seed)
    w_router = torch.randn((d, 8), generator=g, device=DEV) / float(np.sqrt(d))
    router_bias = torch.randn(8, generator=g, device=DEV) * 0.5 if bias else None
    # only the weights' element type matters to the routing entry point
    w_gate = torch.zeros((1, 1, 1), dtype=torch.int8 if dtype == "bf16_int8w" else x.dtype, device=DEV)
    comp = EP.LibraryCompute(w_router, w_gate, None, None, router_bias=router_bias, renormalize=renormalize)
    r = comp.route_dispatch(x)
    torch.cuda.synchronize()
    return x, w_router, router_bias, r


@pytest.mark.parametrize("dtype,T,d", CASES)
def test_small_route_dispatch_matches_the_oracle(dtype, T, d):
    _check(dtype, T, d, seed=T * 7 + d % 97)


@pytest.mark.parametrize("bias,renormalize", [(True, False), (False, True), (True, True)])
def test_small_route_dispatch_bias_and_renormalised_gates(bias, renormalize):
    _check("bf16", 48, 2048, seed=11, bias=bias, renormalize=renormalize)


def _check(dtype, T, d, seed, bias=False, renormalize=False):
    x, w_router, router_bias, r = _route(dtype, T, d, seed, bias, renormalize)
    gpu = {k: r[k].cpu().numpy() for k in ("idx", "gates", "offsets", "perm_token", "perm_slot")}
    gpu["counts"] = np.asarray(r["counts"], dtype=np.int64)
    routing, _ = expected_routing(np64(x), np64(w_router), np64(router_bias) if bias else None, gpu["idx"],
                                  renormalize)
    check_routing_and_dispatch(gpu, routing)

    perm_token = r["perm_token"].long()
    perm_slot = r["perm_slot"].long()
    slot_pos = r["slot_pos"].long()
    # slot_pos inverts the permutation
    tok = torch.arange(T, device=DEV)
    for s in (0, 1):
        assert torch.equal(perm_token[slot_pos[:, s]], tok)
        assert torch.equal(perm_slot[slot_pos[:, s]], torch.full_like(tok, s))
    # gate_perm carries each row's gate, bit for bit
    assert torch.equal(r["gate_perm"], r["gates"][perm_token, perm_slot])
    # the permuted rows of x
    want = x[perm_token]
    if dtype == "bf16_int8w":
        want = want.to(torch.float16)
    assert torch.equal(r["xp"], want)
    # offsets are the exclusive prefix of the counts
    assert np.array_equal(gpu["offsets"], np.concatenate([[0], np.cumsum(gpu["counts"])]))
