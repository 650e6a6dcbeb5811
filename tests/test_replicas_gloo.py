"""The N > 1 benchmark path on the CPU: two gloo ranks run as replicas, the
timing is the max over ranks and the job's throughput counts both ranks' work
(the path does not shard, so there is no data-path collective to test)."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [12.5, 20.0][rank]          # rank 1 is the slow replica
        t_max = bench.max_over_ranks(my_ms, dist, "cpu")
        dist.barrier()
        q.put((rank, t_max, bench.job_throughput(world, 10, 3.0, t_max)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_time_and_summed_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [20.0, 20.0]
    # 2 ranks x 10 steps x 3 units in 20 ms of wall time on the slowest rank
    assert res[0][2] == pytest.approx(2 * 10 * 3.0 / 0.020)


def test_launch_count_rule():
    from mixture_experts_ffn_14_b200 import workloads as W

    # The down projection's epilogue sums each token's rows: no combine kernel.
    # bf16 gate/up from 512 tokens: 256-row tiles alone; down: both 128-row forms
    assert bench.launches_per_step(W.WORKLOADS["prefill"], "auto") == 5
    import dataclasses
    assert bench.launches_per_step(W.WORKLOADS["decode"], "auto") == 3   # router + dispatch in one launch
    assert bench.launches_per_step(W.WORKLOADS["int8"], "auto") == 4
    assert bench.launches_per_step(W.WORKLOADS["prefill"], "token_tile") == 4
    assert bench.launches_per_step(W.WORKLOADS["skewed"], "auto") == 5
    assert bench.launches_per_step(dataclasses.replace(W.WORKLOADS["prefill"], T=384), "auto") == 6
    assert bench.launches_per_step(dataclasses.replace(W.WORKLOADS["prefill"], T=512), "auto") == 5
    # bf16 weights take token tiles above 128 tokens, int8 weights above 256
    assert bench.launches_per_step(dataclasses.replace(W.WORKLOADS["prefill"], T=128), "auto") == 3
    assert bench.launches_per_step(dataclasses.replace(W.WORKLOADS["prefill"], T=200), "auto") == 6
    assert bench.launches_per_step(dataclasses.replace(W.WORKLOADS["int8"], T=200), "auto") == 4
    assert bench.launches_per_step(dataclasses.replace(W.WORKLOADS["int8"], T=300), "auto") == 4
    big = dataclasses.replace(W.WORKLOADS["prefill"], T=40000)   # > 1024 router blocks: + scan
    assert bench.launches_per_step(big, "auto") == 6
