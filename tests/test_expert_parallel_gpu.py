"""The expert-parallel form's GPU data plane (moe_route_dispatch,
moe_gather_rows, moe_experts_forward, moe_combine through the C ABI) with
W = 2, 4, 8 ranks on one GPU. Each rank is a host thread with its own batch of
tokens and only its own experts' weights; the all-to-alls are copies through
host-side barriers (``ThreadExchange``), so no kernel ever waits for another
rank's kernel. Every rank's output must equal, bit for bit, the single-GPU
moe_forward_ex of its tokens with all weights (same kernel form and split-K),
and match the oracle at the stated tolerance."""

import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import mixture_experts_ffn_14_b200 as moe
from mixture_experts_ffn_14_b200 import expert_parallel as EP
from mixture_experts_ffn_14_b200 import workloads as W

from _harness import full_check, np64, run_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


class Board:
    def __init__(self, world):
        self.world = world
        self.slots = [None] * world
        self.barrier = threading.Barrier(world, timeout=120)


class ThreadExchange:
    """all_to_all among the threads sharing `board` (one per virtual rank).
    All threads launch on the same CUDA stream, so a copy issued after the
    barrier runs after the peer's kernels that produced its input."""

    def __init__(self, board, rank):
        self.board, self.rank, self.world = board, rank, board.world

    def all_to_all(self, out, inp, out_splits, in_splits):
        b = self.board
        b.slots[self.rank] = (inp, list(in_splits))
        b.barrier.wait()
        at = 0
        for s in range(self.world):
            pin, ps = b.slots[s]
            start, n = sum(ps[:self.rank]), ps[self.rank]
            assert n == out_splits[s]
            if n:
                out[at:at + n].copy_(pin[start:start + n])
            at += n
        b.barrier.wait()
        return out


def _inputs(world, dtype, seed):
    w = W.Workload("ep", 64, 512, 384, dtype=dtype, seed=seed)
    full = W.make_torch(w, DEV)
    xs = [W.make_x(w, DEV, T, seed_name=f"x_rank{r}") for r, T in enumerate([150, 61, 300, 1, 97, 0, 220, 33][:world])]
    return full, xs


def _local_compute(full, rank, world):
    n = EP.experts_per_rank(world)
    sl = slice(rank * n, rank * n + n)
    scales = None
    if "s_gate" in full:
        scales = tuple(full[k][sl].contiguous() for k in ("s_gate", "s_up", "s_down"))
    return EP.LibraryCompute(full["w_router"], full["w_gate"][sl].contiguous(), full["w_up"][sl].contiguous(),
                             full["w_down"][sl].contiguous(), scales=scales, path=moe.MOE_PATH_TOKEN_TILE_SINGLE,
                             down_splits=1)


def _single_gpu(full, x):
    T, d = x.shape
    out = torch.empty_like(x)
    if T == 0:
        return out
    f = full["w_gate"].shape[2]
    dt = moe.dtype_code(x, full["w_gate"])
    ws = torch.empty(moe.moe_workspace_size(T, d, f, dtype=dt, path=moe.MOE_PATH_TOKEN_TILE_SINGLE, down_splits=1),
                     dtype=torch.uint8, device=DEV)
    scales = (full["s_gate"], full["s_up"], full["s_down"]) if "s_gate" in full else None
    moe.moe_forward_ex(x, full["w_router"], full["w_gate"], full["w_up"], full["w_down"], out, ws, scales=scales,
                       path=moe.MOE_PATH_TOKEN_TILE_SINGLE, down_splits=1)
    return out


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("dtype", ["bf16", "bf16_int8w"])
def test_expert_parallel_data_plane_matches_single_gpu_bitwise(world, dtype):
    full, xs = _inputs(world, dtype, seed=200 + world)
    board = Board(world)

    def rank_fn(r):
        comp = _local_compute(full, r, world)
        return EP.ep_forward(xs[r], comp, ThreadExchange(board, r))

    with ThreadPoolExecutor(max_workers=world) as pool:
        outs = list(pool.map(rank_fn, range(world)))
    torch.cuda.synchronize()
    for r in range(world):
        ref = _single_gpu(full, xs[r])
        torch.cuda.synchronize()
        assert torch.equal(outs[r], ref), f"rank {r}: differs from the single-GPU forward"
        if xs[r].shape[0]:
            case = dict(full)
            case["x"] = xs[r]
            gpu = run_gpu(case, want_h=False)
            gpu["out"] = np64(outs[r])
            full_check(case, gpu, check_h=False)


def test_gather_rows_and_combine_entry_points():
    g = torch.Generator(device=DEV)
    g.manual_seed(5)
    src = torch.randn((50, 96), generator=g, device=DEV)
    idx = torch.randint(0, 50, (77,), generator=g, device=DEV, dtype=torch.int32)
    comp = EP.LibraryCompute(None, torch.empty((1, 1, 1), device=DEV), None, None)
    assert torch.equal(comp.gather_rows(src, idx), src[idx.long()])
    col = src[:, :1].contiguous()                      # 4-byte rows
    assert torch.equal(comp.gather_rows(col, idx), col[idx.long()])
    # combine: out[t] = y[slot_pos[t,0]] + y[slot_pos[t,1]] (fp32 sum, bf16 out)
    T, d = 25, 96
    y = torch.randn((2 * T, d), generator=g, device=DEV)
    perm = torch.randperm(2 * T, generator=g, device=DEV).to(torch.int32).reshape(T, 2).contiguous()
    routed = {"T": T, "dtype": moe.MOE_BF16, "slot_pos": perm}
    out = comp.combine(routed, y)
    ref = (y[perm[:, 0].long()] + y[perm[:, 1].long()]).to(torch.bfloat16)
    assert torch.equal(out, ref)


def test_expert_parallel_over_nccl_single_rank():
    # The multi-GPU code path itself (DistExchange over a torch.distributed NCCL
    # group, LibraryCompute through the C ABI) with one rank: every exchange is
    # a copy to itself, and the result must equal the single-GPU forward bit for
    # bit with the same kernel form and split-K.
    import os
    import socket

    import torch.distributed as dist

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device(DEV))
    try:
        full, xs = _inputs(1, "bf16", seed=300)
        comp = _local_compute(full, 0, 1)
        out = EP.ep_forward(xs[0], comp, EP.DistExchange())
        torch.cuda.synchronize()
        assert torch.equal(out, _single_gpu(full, xs[0]))
    finally:
        dist.destroy_process_group()
