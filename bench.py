#!/usr/bin/env python
"""Benchmark of the Grok-1-shape MoE feed-forward sublayer on B200.

One step = one forward of the whole sublayer (router, dispatch, gate/up GEMM,
down GEMM, combine) over T = 4096 tokens, d = 6144, f = 32768, E = 8, top-2,
bf16 activations and weights, fp32 router and accumulation. Inputs are seeded
synthetic tensors already resident in HBM. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica on its own GPU (the layer does not shard on this path): no data-path
collective; the timing is the max over ranks and `value` sums the work of all
ranks. `--impl reference` times the CPU oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FLUSH_BYTES = 256 << 20           # > 126 MB L2


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode (T=64) side measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--cpu-sample", type=int, default=64, help="tokens in the timed oracle sample")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, torch_dev):
        import torch

        self.proc = None
        self.lines = []
        try:
            pr = torch.cuda.get_device_properties(torch_dev)
            self.bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.bus:
            cmd += ["-i", self.bus]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ CPU oracle --

def oracle_sample(inp, tokens):
    """Time the oracle (as it stands) on `tokens` of the workload; expert
    matrices are copied from the device one expert at a time (float32, exact
    for bf16) and the oracle converts them to float64 itself."""
    import numpy as np

    import oracle

    x = inp["x"].float().cpu().numpy()
    wr = inp["w_router"].float().cpu().numpy()

    def get(e):
        return tuple(inp[w][e].float().cpu().numpy() for w in ("w_gate", "w_up", "w_down"))

    t0 = time.perf_counter()
    res = oracle.forward_sparse(x, wr, get, tokens=np.asarray(tokens))
    dt = time.perf_counter() - t0
    return dt, res


def blas_threads():
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------- main --

def main():
    a = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    import numpy as np
    import torch

    from mixture_experts_ffn_14_b200 import workloads as W

    wl = W.WORKLOADS["prefill"]
    flops = wl.flops
    workload_name = f"grok1-prefill T={wl.T} d={wl.d} f={wl.f} E={wl.E} k={wl.k} bf16"

    if a.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(a, wl, workload_name, world)

    import mixture_experts_ffn_14_b200 as moe

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()

    inp = W.make_torch(wl, dev)
    T, d, f = wl.T, wl.d, wl.f
    ws = torch.empty(moe.moe_workspace_size(T, d, f), dtype=torch.uint8, device=dev)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step(events=None):
        moe.moe_forward_ex(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out, ws,
                           stage_events=events)

    for _ in range(a.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    st, code = moe.moe_device_status(ws)
    if st != 0:
        raise SystemExit(f"device status {st} code {code:#x}")

    K = a.steps
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for evs in stage_ev:          # materialise the event handles
        for e in evs:
            e.record()
    torch.cuda.synchronize()

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    with ClockSampler(dev) as clk:
        for i in range(K):
            flush.zero_()                       # L2 flush, outside the step's events
            starts[i].record()
            step(stage_ev[i])
            ends[i].record()
        torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()

    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    stage_names = ["router", "dispatch", "gate_up_gemm", "down_gemm", "combine"]
    stage_ms = {n: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in stage_ev)
                for j, n in enumerate(stage_names)}
    t_max = total_ms
    if dist is not None:
        tt = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_max = float(tt.item())

    value = world * K * flops / (t_max / 1e3) / 1e12
    tok_s = world * K * T / (t_max / 1e3)

    # dominant kernel: the gate/up GEMM (2/3 of the FLOPs)
    gu_flops = 8 * T * d * f
    gu_tflops = gu_flops / (stage_ms["gate_up_gemm"] / 1e3) / 1e12
    down_tflops = (4 * T * d * f) / (stage_ms["down_gemm"] / 1e3) / 1e12
    peak_t = pk["bf16_tflops_sustained"]
    roofline = {"bound": "tensor", "kernel": "moe_expert_gemm_kernel<GATEUP> (gate+up GEMM, GELU*up epilogue)",
                "achieved": round(gu_tflops, 1), "peak": peak_t, "unit": "TFLOP/s",
                "frac": round(gu_tflops / peak_t, 4), "traffic": None,
                "peak_source": f"{pk['source']} bf16 sustained",
                "down_gemm": {"achieved": round(down_tflops, 1), "frac": round(down_tflops / peak_t, 4)}}

    # ---- end-to-end through moe_forward with pinned host buffers -------------
    e2e = run_e2e(a, moe, inp, out, flush, dist, dev, world, flops) if not a.no_e2e else None

    # ---- decode side measurement: same weights, T = 64 ------------------------
    decode = None
    if not a.no_decode:
        decode = run_decode(a, moe, W, wl, inp, dev, pk)

    # ---- CPU oracle baseline (rank 0, N = 1 only) -------------------------------
    cpu = None
    if not a.no_cpu_baseline and world == 1 and rank == 0:
        rng = np.random.default_rng(0)
        sample = np.sort(rng.choice(T, size=min(a.cpu_sample, T), replace=False))
        dt, _ = oracle_sample(inp, sample)
        cpu = {"value": round(12 * d * f * len(sample) / dt / 1e12, 6), "unit": "TFLOP/s",
               "cores": blas_threads(), "kind": "oracle",
               "sample": f"{len(sample)} of {T} tokens (routing of all {T}), fp64 numpy, {dt:.1f} s"}
    return finish(a, rank, world, dist, K, T, t_max, value, tok_s, stage_ms, roofline, e2e, decode, cpu, clk,
                  wall, workload_name)


def run_e2e(a, moe, inp, out, flush, dist, dev, world, flops):
    import torch

    T, d = inp["x"].shape
    K = a.steps
    x_host = inp["x"].cpu().pin_memory()
    out_host = torch.empty((T, d), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(inp["x"])
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        moe.moe_forward(x_dev, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out)
        out_host.copy_(out, non_blocking=True)

    for _ in range(a.warmup):
        flush.zero_()
        e2e_step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    for i in range(K):
        flush.zero_()
        e_s[i].record()
        e2e_step()
        e_e[i].record()
    torch.cuda.synchronize()
    e2e_ms = sum(s.elapsed_time(e) for s, e in zip(e_s, e_e))
    if dist is not None:
        tt = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        e2e_ms = float(tt.item())
    return {"value": round(world * K * flops / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2,
            "api": "moe_forward (library workspace), pinned host x -> device -> pinned host out"}


def run_decode(a, moe, W, wl, inp, dev, pk):
    import torch

    K = a.steps
    d, f = wl.d, wl.f
    Td = W.WORKLOADS["decode"].T
    xd = W.make_x(wl, dev, Td, seed_name="x_decode")
    wsd = torch.empty(moe.moe_workspace_size(Td, d, f), dtype=torch.uint8, device=dev)
    outd = torch.empty((Td, d), dtype=torch.bfloat16, device=dev)
    cnt = torch.empty(8, dtype=torch.int32, device=dev)
    evd = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for evs in evd:
        for e in evs:
            e.record()

    def dstep(events=None, dbg=None):
        moe.moe_forward_ex(xd, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], outd, wsd,
                           stage_events=events, debug=dbg)

    for _ in range(a.warmup):
        dstep(dbg={"counts": cnt})
    torch.cuda.synchronize()
    touched = int((cnt > 0).sum().item())
    for i in range(K):
        dstep(evd[i])
    torch.cuda.synchronize()
    d_ms = statistics.mean(ev[0].elapsed_time(ev[5]) for ev in evd)
    d_gu = statistics.mean(ev[2].elapsed_time(ev[3]) for ev in evd)
    d_dn = statistics.mean(ev[3].elapsed_time(ev[4]) for ev in evd)
    wbytes = touched * 3 * d * f * 2
    return {"workload": f"grok1-decode T={Td} d={d} f={f} bf16 (same weights)",
            "ms_per_step": round(d_ms, 4), "experts_touched": touched,
            "hbm_gbs": round(wbytes / (d_ms / 1e3) / 1e9, 1),
            "frac": round(wbytes / (d_ms / 1e3) / 1e9 / pk["hbm_gbs"], 4),
            "gate_up_gbs": round(touched * 2 * d * f * 2 / (d_gu / 1e3) / 1e9, 1),
            "down_gbs": round(touched * d * f * 2 / (d_dn / 1e3) / 1e9, 1),
            "stage_ms": {"gate_up_gemm": round(d_gu, 4), "down_gemm": round(d_dn, 4)},
            "peak_gbs": pk["hbm_gbs"], "bytes_per_step": wbytes}


def finish(a, rank, world, dist, K, T, t_max, value, tok_s, stage_ms, roofline, e2e, decode, cpu, clk, wall,
           workload_name):
    clocks = clk.summary()
    d, f = 6144, 32768
    line = {
        "metric": "MoE-layer TFLOP/s, Grok-1 prefill (tokens/s and decode HBM GB/s alongside)",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K, "warmup": a.warmup,
        "ms_per_step": round(t_max / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) activations, N(0, 1/sqrt(fan_in)) random-init weights",
        "config": {"workload": workload_name, "T": T, "d": d, "f": f, "E": 8, "k": 2,
                   "l2": "flushed (256 MB write) between steps, outside the step events; weights 9.66 GB > L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "tokens_per_s": round(tok_s, 1),
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": roofline,
        "gpu_launches": 5 * K,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"]},
        "wall_s_timed_region": round(wall, 3),
    }
    if e2e:
        line["e2e"] = e2e
    if decode:
        line["decode"] = decode
    if cpu:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_reference(a, wl, workload_name, world):
    """The oracle on the host cores, same metric: each step is the oracle's
    forward for 8 tokens that all route to one expert pair (so a step converts
    two experts' weights), cycling through the pairs present in the batch."""
    import numpy as np
    import torch

    import oracle
    from mixture_experts_ffn_14_b200 import workloads as W

    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    inp = W.make_torch(wl, dev)
    x = inp["x"].float().cpu().numpy()
    wr = inp["w_router"].float().cpu().numpy()
    r = oracle.route(x, wr)
    pairs = {}
    for t, (e0, e1) in enumerate(r["idx"]):
        pairs.setdefault((min(e0, e1), max(e0, e1)), []).append(t)
    groups = [v[:8] for _, v in sorted(pairs.items()) if len(v) >= 8]

    def get(e):
        return tuple(inp[w][e].float().cpu().numpy() for w in ("w_gate", "w_up", "w_down"))

    def one(i):
        toks = np.asarray(groups[i % len(groups)])
        t0 = time.perf_counter()
        oracle.forward_sparse(x, wr, get, tokens=toks, routing=r)
        return time.perf_counter() - t0, len(toks)

    for i in range(a.warmup):
        one(i)
    total, ntok = 0.0, 0
    for i in range(a.steps):
        dt, n = one(a.warmup + i)
        total += dt
        ntok += n
    v = 12 * wl.d * wl.f * ntok / total / 1e12
    line = {
        "impl": "reference", "metric": "MoE-layer TFLOP/s, Grok-1 prefill (tokens/s and decode HBM GB/s alongside)",
        "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(total / a.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the b200 arm)",
        "config": {"workload": workload_name, "T": wl.T, "d": wl.d, "f": wl.f, "E": 8, "k": 2},
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": "per step 8 tokens routed to one expert pair (routing of all 4096 tokens done once)"},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
