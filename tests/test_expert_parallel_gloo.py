"""The expert-parallel exchange (the pages' expert-axis sharding, Grok-1 book
ch. 1, section 1.6.3) on the CPU: 2 and 4 gloo ranks, each with its own
batch of tokens and the weights of its own experts, run ``ep_forward`` with
real all-to-alls. The compute steps are the oracle's (this file's
``OracleCompute``), so the test checks the host logic of the exchange: split
sizes, the receive layout, the expert-major reordering and the way back. Every
rank's output must equal the oracle's single-process forward of its tokens,
and the plans must account for every row."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mixture_experts_ffn_14_b200 import expert_parallel as EP
from mixture_experts_ffn_14_b200 import workloads as W

D, F = 16, 32


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _weights():
    p = W.make_numpy(1, D, F, seed=7)
    return p["w_router"].astype(np.float64), p["w_gate"].astype(np.float64), p["w_up"].astype(np.float64), \
        p["w_down"].astype(np.float64)


def _tokens(rank):
    # ragged batches, a different number of tokens per rank (rank 3: none)
    T = [23, 40, 7, 0][rank % 4]
    return np.random.default_rng(100 + rank).standard_normal((T, D))


class OracleCompute(EP.LocalCompute):
    """The oracle as the compute steps, on CPU float64 tensors."""

    def __init__(self, rank, world):
        self.wr, self.wg, self.wu, self.wd = _weights()
        self.mine = list(EP.local_experts(rank, world))

    def empty(self, shape, like):
        return torch.empty(shape, dtype=like.dtype)

    def route_dispatch(self, x):
        x = x.numpy()
        T = x.shape[0]
        if T == 0:
            return {"counts": [0] * 8, "xp": torch.zeros((0, D), dtype=torch.float64),
                    "gate_perm": torch.zeros(0, dtype=torch.float64), "slot_pos": np.zeros((0, 2), np.int64)}
        r = oracle.route(x, self.wr)
        dsp = oracle.dispatch(r["idx"], 8)
        xp = x[dsp["perm_token"]]
        gp = r["gates"][dsp["perm_token"], dsp["perm_slot"]]
        return {"counts": [int(c) for c in dsp["counts"]], "xp": torch.from_numpy(xp.copy()),
                "gate_perm": torch.from_numpy(gp.copy()), "slot_pos": dsp["slot_pos"]}

    def gather_rows(self, src, index):
        return src[index.long()]

    def experts(self, rows, expert_rows, gates):
        y = torch.zeros(rows.shape, dtype=torch.float64)
        at = 0
        for j, n in enumerate(expert_rows):
            if n:
                e = self.mine[j]
                blk, _ = oracle.expert_ffn(rows[at:at + n].numpy(), self.wg[e], self.wu[e], self.wd[e])
                y[at:at + n] = torch.from_numpy(blk) * gates[at:at + n, None]
            at += n
        assert at == rows.shape[0]
        return y

    def combine(self, routed, y):
        sp = routed["slot_pos"]
        return y[sp[:, 0]] + y[sp[:, 1]]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _tokens(rank)
        comp = OracleCompute(rank, world)
        out = EP.ep_forward(torch.from_numpy(x), comp).numpy()
        wr, wg, wu, wd = _weights()
        ref = oracle.forward_sparse(x, wr, (wg, wu, wd))["out"] if x.shape[0] else np.zeros((0, D))
        err = float(np.abs(out - ref).max()) if out.size else 0.0
        # the plan's accounting, gathered on every rank
        routed = comp.route_dispatch(torch.from_numpy(x))
        rc = EP.exchange_counts(routed["counts"], EP.DistExchange())
        plan = EP.make_plan(rank, world, routed["counts"], rc)
        q.put((rank, x.shape[0], err, routed["counts"], plan.send_rows, plan.recv_rows, plan.expert_rows))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_exchange_matches_the_oracle(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, T, err, counts, snd, rcv, erows in res:
        assert err < 1e-12, (rank, err)
        assert sum(snd) == 2 * T                     # every token slot leaves once
    total = np.sum([r[3] for r in res], axis=0)      # global rows per expert
    n = 8 // world
    for rank, _, _, _, _, rcv, erows in res:
        assert erows == [int(v) for v in total[rank * n:(rank + 1) * n]]
        assert sum(rcv) == sum(erows)
    # what GPU s sends to GPU r is what GPU r expects from GPU s
    for s in range(world):
        for r in range(world):
            assert res[s][4][r] == res[r][5][s]


def test_plan_layout_by_hand():
    # 2 GPUs, 4 experts each. GPU 1's view: GPU 0 sends 3 rows of expert 4 and
    # 1 of expert 6; GPU 1 itself keeps 2 rows of expert 5 and 2 of expert 6.
    counts_gpu1 = [1, 0, 0, 0, 0, 2, 2, 0]
    recv = [[3, 0, 1, 0], [0, 2, 2, 0]]
    p = EP.make_plan(1, 2, counts_gpu1, recv)
    assert p.send_rows == [1, 4]
    assert p.recv_rows == [4, 4]
    assert p.expert_rows == [3, 2, 3, 0]
    # receive buffer: [g0e4 g0e4 g0e4 g0e6 | g1e5 g1e5 g1e6 g1e6]
    # expert-major:   [g0e4 x3 | g1e5 x2 | g0e6, g1e6 x2]
    assert p.to_expert_major.tolist() == [0, 1, 2, 4, 5, 3, 6, 7]
    assert (p.to_expert_major[p.to_source_major] == np.arange(8)).all()
    assert list(EP.local_experts(1, 2)) == [4, 5, 6, 7]
    with pytest.raises(ValueError):
        EP.experts_per_rank(3)
