#!/usr/bin/env python
"""Benchmark of the Grok-1-shape MoE feed-forward sublayer on B200.

One step = one forward of the whole sublayer (router, dispatch, gate/up GEMM,
down GEMM, combine) over one batch, inputs already resident in HBM. The
default workload is the Grok-1 prefill shape: T = 4096 tokens, d = 6144,
f = 32768, E = 8, top-2, bf16 activations and weights, fp32 router and
accumulation. Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                  [--workload prefill|decode|int8|skewed] [--T ..] [--d ..] [--f ..]
                  [--path auto|token_tile|weight_stream|token_tile_single] [--row-gather]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica on its own GPU (the layer does not shard on this path): no data-path
collective; the timing is the max over ranks and `value` sums the work of all
ranks. `--impl reference` times the CPU oracle on the host cores instead.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FLUSH_BYTES = 256 << 20           # > 126 MB L2
METRIC = "MoE-layer TFLOP/s, Grok-1 prefill (tokens/s and decode HBM GB/s alongside)"
STAGES = ["router", "dispatch", "gate_up_gemm", "down_gemm", "combine"]


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", choices=["prefill", "decode", "int8", "skewed"], default="prefill")
    ap.add_argument("--T", type=int, default=None, help="override the token count")
    ap.add_argument("--d", type=int, default=None, help="override the hidden size")
    ap.add_argument("--f", type=int, default=None, help="override the expert width")
    ap.add_argument("--path", choices=["auto", "token_tile", "weight_stream", "token_tile_single"], default="auto",
                    help="kernel family (default: the library's automatic choice)")
    ap.add_argument("--row-gather", action="store_true",
                    help="token tiles gather their gate/up rows from x (TMA row gather) instead of the copy")
    ap.add_argument("--separate-combine", action="store_true",
                    help="sum each token's rows in the combine kernel instead of the down projection's epilogue")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode (T=64) side measurement")
    ap.add_argument("--no-int8", action="store_true", help="skip the int8-weight (T=1024) side measurement")
    ap.add_argument("--no-skewed", action="store_true", help="skip the skewed-load (T=16384) side measurement")
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
    """SM clock, power and clock-event reasons sampled DURING the `with` block.

    NVML (read-only queries) every 20 ms from a background thread; if NVML is
    unavailable, nvidia-smi every 100 ms, keeping the samples whose own
    timestamp falls inside the block."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))
    SMI_FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, torch_dev):
        import torch

        self.samples = []        # (sm_mhz, sm_max_mhz, power_w, {reason names})
        self.source = None
        self._stop = None
        self._thread = None
        self._proc = None
        self._t0 = self._t1 = None
        try:
            pr = torch.cuda.get_device_properties(torch_dev)
            self.bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        except Exception:
            self.bus = None

    # ---- NVML
    def _nvml_loop(self, nv, h):
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(smax), pw, {n for n, m in self.REASONS if bits & m}))
            except Exception:
                pass
            self._stop.wait(0.02)

    def _start_nvml(self):
        import threading

        import pynvml as nv

        nv.nvmlInit()
        h = nv.nvmlDeviceGetHandleByPciBusId(self.bus.encode()) if self.bus else nv.nvmlDeviceGetHandleByIndex(0)
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
        self._thread.start()
        self.source = "nvml"

    # ---- nvidia-smi fallback
    def _start_smi(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.bus:
            cmd += ["-i", self.bus]
        self._proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        time.sleep(0.5)  # let it start sampling before the region opens
        self.source = "nvidia-smi"

    def _finish_smi(self):
        time.sleep(0.15)
        self._proc.terminate()
        try:
            out, _ = self._proc.communicate(timeout=5)
        except Exception:
            self._proc.kill()
            out = ""
        stamped = []
        for ln in out.splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                t = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                smp = (float(parts[2]), float(parts[3]), float(parts[4]),
                       {n for n, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                           "sw_power_cap"), parts[6:10]) if v.lower() == "active"})
            except ValueError:
                continue
            stamped.append((t, smp))
        inside = [smp for t, smp in stamped if self._t0 <= t <= self._t1]
        if not inside and stamped:  # region shorter than a sample period: the nearest sample
            mid = 0.5 * (self._t0 + self._t1)
            inside = [min(stamped, key=lambda ts: abs(ts[0] - mid))[1]]
        self.samples = inside

    def __enter__(self):
        try:
            self._start_nvml()
        except Exception:
            try:
                self._start_smi()
            except Exception:
                self.source = None
        self._t0 = time.time()
        return self

    def __exit__(self, *exc):
        self._t1 = time.time()
        if self.source == "nvml":
            self._stop.set()
            self._thread.join(timeout=5)
        elif self.source == "nvidia-smi":
            self._finish_smi()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [x[0] for x in self.samples]
        reasons = set().union(*(x[3] for x in self.samples))
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.samples[-1][1], "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(x[2] for x in self.samples),
                "power_w_median": statistics.median(x[2] for x in self.samples), "source": self.source}


# ------------------------------------------------------------ CPU oracle --

def expert_getter(inp):
    """One expert's matrices as float32 host arrays (exact for bf16; int8
    weights dequantised by the oracle's own routine)."""
    import oracle

    def get(e):
        if "s_gate" in inp:
            return tuple(oracle.dequant_int8(inp[w][e].cpu().numpy(), inp[s][e].float().cpu().numpy())
                         for w, s in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")))
        return tuple(inp[w][e].float().cpu().numpy() for w in ("w_gate", "w_up", "w_down"))
    return get


def oracle_sample(inp, tokens):
    """Time the oracle, as it stands, on `tokens` of the batch (routing of all
    tokens included); the oracle converts each expert to float64 itself."""
    import numpy as np

    import oracle

    x = inp["x"].float().cpu().numpy()
    wr = inp["w_router"].float().cpu().numpy()
    bias = inp["router_bias"].cpu().numpy() if "router_bias" in inp else None
    t0 = time.perf_counter()
    oracle.forward_sparse(x, wr, expert_getter(inp), tokens=np.asarray(tokens), router_bias=bias)
    return time.perf_counter() - t0


def oracle_pair_sample(inp, ntok=8):
    """Time the oracle, as it stands, on up to `ntok` tokens that all route to
    the most frequent expert pair of the batch (so the sample converts two
    experts' weights, not eight). Returns (seconds, tokens, pair)."""
    import numpy as np

    import oracle

    x = inp["x"].float().cpu().numpy()
    wr = inp["w_router"].float().cpu().numpy()
    bias = inp["router_bias"].cpu().numpy() if "router_bias" in inp else None
    r = oracle.route(x, wr, bias)
    pairs = {}
    for t, (e0, e1) in enumerate(r["idx"]):
        pairs.setdefault((int(min(e0, e1)), int(max(e0, e1))), []).append(t)
    pair, toks = max(pairs.items(), key=lambda kv: (len(kv[1]), kv[0]))
    toks = np.asarray(toks[:ntok])
    t0 = time.perf_counter()
    oracle.forward_sparse(x, wr, expert_getter(inp), tokens=toks, routing=r)
    return time.perf_counter() - t0, len(toks), pair


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


# --------------------------------------------------------------- helpers --

def workload(a):
    from mixture_experts_ffn_14_b200 import workloads as W

    wl = W.WORKLOADS[a.workload]
    over = {k: getattr(a, k) for k in ("T", "d", "f") if getattr(a, k) is not None}
    if over:
        wl = dataclasses.replace(wl, **over)
    dt = {"bf16": "bf16", "bf16_int8w": "int8 weights + bf16 scales, bf16 activations"}[wl.dtype]
    name = f"grok1-{wl.name} T={wl.T} d={wl.d} f={wl.f} E={wl.E} k={wl.k} {dt}"
    if wl.skew:
        name += ", router bias -> ~50/15/15/4x5 % of slots"
    return wl, name


class Runner:
    """One forward through the C ABI (moe_forward_ex on a preallocated workspace)."""

    PATHS = {"auto": 0, "token_tile": 1, "weight_stream": 2, "token_tile_single": 3}

    def __init__(self, moe, inp, T, d, f, dev, path="auto", row_gather=False, separate_combine=False):
        import torch

        self.moe, self.inp = moe, inp
        self.row_gather = row_gather
        self.separate_combine = separate_combine
        self.path = self.PATHS[path]
        dt = moe.dtype_code(inp["x"], inp["w_gate"])
        self.ws = torch.empty(moe.moe_workspace_size(T, d, f, dtype=dt, path=self.path), dtype=torch.uint8,
                              device=dev)
        self.scales = (inp["s_gate"], inp["s_up"], inp["s_down"]) if "s_gate" in inp else None

    def __call__(self, x, out, events=None, debug=None):
        i = self.inp
        self.moe.moe_forward_ex(x, i["w_router"], i["w_gate"], i["w_up"], i["w_down"], out, self.ws,
                                scales=self.scales, router_bias=i.get("router_bias"), stage_events=events,
                                debug=debug, path=self.path, row_gather=self.row_gather,
                                separate_combine=self.separate_combine)


def timed_steps(run, x, out, K, flush, clk=None):
    """K steps, each bracketed by CUDA events (and the library's stage events),
    with an L2 flush before each step outside its events."""
    import torch

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K)]
    for evs in stage_ev:          # materialise the event handles
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    for i in range(K):
        if flush is not None:
            flush.zero_()
        starts[i].record()
        run(x, out, stage_ev[i])
        ends[i].record()
    torch.cuda.synchronize()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    stage_ms = {n: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in stage_ev)
                for j, n in enumerate(STAGES)}
    return step_ms, stage_ms


def max_over_ranks(v, dist, dev):
    """Largest value over the ranks (the slowest replica's time). `dev` is the
    device the reduction runs on: a CUDA device under NCCL, the CPU under gloo."""
    if dist is None:
        return v
    import torch

    t = torch.tensor([v], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, steps, work_per_step, t_max_ms):
    """Whole-job rate: every rank did `steps` steps of `work_per_step` units,
    the job took as long as its slowest rank."""
    return world * steps * work_per_step / (t_max_ms / 1e3)


def weight_stream_form(wl, path):
    """Whether the step streams its weights (weight-stream down projection, a
    bound set by HBM): forced, or on the automatic path for small batches
    (T <= 256 with int8 weights, T <= 128 with bf16 weights, whose gate/up GEMM
    then runs 128-row token tiles; the library's choice)."""
    if path == "weight_stream":
        return True
    if path != "auto":
        return False
    return wl.T <= (256 if wl.dtype == "bf16_int8w" else 128)


def launches_per_step(wl, path):
    """Kernels of ours per step: router, dispatch (one cluster launch for both
    at T <= 128) and two GEMMs (the down projection's epilogue sums each
    token's rows, so no combine kernel runs). With the automatic token-tile
    choice on bf16 weights a GEMM launches both 128-row forms (the one not
    chosen returns at once), except the gate/up GEMM from 512 tokens, which
    runs 256-row tiles alone. Above 1024 router blocks (T > 32768) a histogram
    scan runs before the dispatch."""
    both = path == "auto" and wl.dtype == "bf16" and not weight_stream_form(wl, path)
    tall_gateup = both and wl.T >= 512
    scan = (wl.T + 31) // 32 > 1024          # block-histogram scan before the dispatch
    route = 1 if wl.T <= 128 else 2
    gemms = (1 if tall_gateup else (2 if both else 1)) + (2 if both else 1)
    return route + gemms + (1 if scan else 0)


# ---------------------------------------------------------------- main --

def main():
    a = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl, workload_name = workload(a)

    if a.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(a, wl, workload_name, world)

    import numpy as np
    import torch

    import mixture_experts_ffn_14_b200 as moe
    from mixture_experts_ffn_14_b200 import workloads as W

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    pk = peaks()

    T, d, f = wl.T, wl.d, wl.f
    inp = W.make_torch(wl, dev)
    run = Runner(moe, inp, T, d, f, dev, a.path, a.row_gather, a.separate_combine)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    counts = torch.empty(8, dtype=torch.int32, device=dev)

    # Decode on the same weights first: measured right after the 1 kW prefill
    # steps, the GPU's clocks are still lowered (decode 6 % slower).
    decode = None
    if not a.no_decode and wl.name == "prefill" and a.T is None:
        decode = run_decode(a, moe, W, wl, inp, dev, pk)

    for _ in range(a.warmup):
        flush.zero_()
        run(inp["x"], out, debug={"counts": counts})
    torch.cuda.synchronize()
    st, code = moe.moe_device_status(run.ws)
    if st != 0:
        raise SystemExit(f"device status {st} code {code:#x}")
    touched = int((counts > 0).sum().item())
    expert_counts = [int(v) for v in counts.cpu().tolist()]
    K = a.steps

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        wall0 = time.perf_counter()
        step_ms, stage_ms = timed_steps(run, inp["x"], out, K, flush)
        wall = time.perf_counter() - wall0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = clk.summary()

    t_max = max_over_ranks(sum(step_ms), dist, dev)
    flops = wl.flops
    value = job_throughput(world, K, flops, t_max) / 1e12
    tok_s = job_throughput(world, K, T, t_max)
    wbytes = touched * 3 * d * f * (1 if wl.dtype == "bf16_int8w" else 2)
    roofline = roofline_entry(wl, pk, stage_ms, touched, clocks, a.path)

    e2e = None if a.no_e2e else run_e2e(a, moe, inp, run, out, flush, dist, dev, world, flops)
    int8 = skewed = None
    if wl.name == "prefill" and a.T is None and a.d is None and a.f is None:
        if not a.no_skewed:
            # The skewed-load workload on the prefill weights: a fresh
            # T = 16384 batch and the per-expert router bias.
            ws = W.WORKLOADS["skewed"]
            inp_s = {k: inp[k] for k in ("w_router", "w_gate", "w_up", "w_down")}
            inp_s["x"] = W.make_x(ws, dev, ws.T, seed_name="x_skewed")
            inp_s["router_bias"] = torch.tensor(W.SKEW_BIAS, dtype=torch.float32, device=dev)
            skewed = run_side(a, moe, ws, f"grok1-skewed T={ws.T} d={d} f={f} E=8 k=2 bf16, router bias "
                              "-> ~50/15/15/4x5 % of slots (prefill weights)", inp_s, dev, pk, dist, world)
            del inp_s
        if not a.no_int8:
            wi = W.WORKLOADS["int8"]
            inp_i = W.make_torch(wi, dev)
            int8 = run_side(a, moe, wi, f"grok1-int8 T={wi.T} d={wi.d} f={wi.f} E=8 k=2 int8 weights + bf16 "
                            "per-channel scales, bf16 activations", inp_i, dev, pk, dist, world)
            del inp_i
        torch.cuda.empty_cache()
    cpu = None
    if not a.no_cpu_baseline and world == 1 and rank == 0:
        rng = np.random.default_rng(0)
        sample = np.sort(rng.choice(T, size=min(a.cpu_sample, T), replace=False))
        dt = oracle_sample(inp, sample)
        cpu = {"value": round(12 * d * f * len(sample) / dt / 1e12, 6), "unit": "TFLOP/s",
               "cores": blas_threads(), "kind": "oracle",
               "sample": f"{len(sample)} of {T} tokens (routing of all {T}), fp64 numpy, {dt:.1f} s"}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": a.warmup, "ms_per_step": round(t_max / K, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) activations, N(0, 1/sqrt(fan_in)) random-init weights",
        "config": {"workload": workload_name, "T": T, "d": d, "f": f, "E": 8, "k": 2,
                   "l2": "flushed (256 MB write) between steps, outside the step events; "
                         f"weights {wbytes / 1e9:.2f} GB > L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "tokens_per_s": round(tok_s, 1),
        "expert_slots": expert_counts,
        "path": a.path,
        "row_gather": bool(a.row_gather),
        "combine": "combine kernel" if a.separate_combine else "in the down projection's epilogue",
        "hbm_gbs_weights": round(world * K * wbytes / (t_max / 1e3) / 1e9, 1),
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": roofline,
        "gpu_launches": (launches_per_step(wl, a.path) + (1 if a.separate_combine else 0)) * K,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                   "power_w_max": clocks.get("power_w_max"), "power_w_median": clocks.get("power_w_median"),
                   "samples": clocks.get("samples"), "source": clocks.get("source")},
        "wall_s_timed_region": round(wall, 3),
    }
    if e2e:
        line["e2e"] = e2e
    if decode:
        line["decode"] = decode
    if int8:
        line["int8"] = int8
    if skewed:
        line["skewed"] = skewed
    if cpu:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def gemm_code_hash(sources):
    """SHA-256 of the GEMM sources with comments and trailing blanks removed: a
    traffic record stays valid while the code is the one it was captured on."""
    import hashlib
    import re

    h = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, src)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()


def recorded_traffic(wl):
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu record of
    this workload, or None when there is none or the GEMM code changed since."""
    import re

    records = {("prefill", 4096, 6144, 32768): "gemm_traffic_prefill_T4096.md",
               ("decode", 64, 6144, 32768): "gemm_traffic_decode_T64.md",
               ("int8", 1024, 6144, 32768): "gemm_traffic_int8_T1024.md",
               ("skewed", 16384, 6144, 32768): "gemm_traffic_skewed_T16384.md"}
    name = records.get((wl.name, wl.T, wl.d, wl.f))
    path = os.path.join(ROOT, "profiles", name) if name else None
    if not path or not os.path.exists(path):
        return None
    m = re.search(r"```json\n(.*?)\n```", open(path).read(), re.S)
    if not m:
        return None
    rec = json.loads(m.group(1))
    if gemm_code_hash(rec["gemm_sources"]) != rec["gemm_code_sha256"]:
        return None
    k = rec["kernels"]["gate_up"]
    return k["dram_read_bytes"] + k["dram_write_bytes"]


def roofline_entry(wl, pk, stage_ms, touched, clocks, path="auto"):
    """The gate/up GEMM is the dominant kernel (2/3 of the FLOPs; in the
    weight-stream form 2/3 of the weight bytes). A step here is milliseconds
    long and the timed region well under a second, so a tensor-bound fraction
    is taken against the burst bf16 peak (the MMAs of the int8-weight path run
    on fp16 operands, whose dense rate equals bf16's); the fraction of the
    sustained (power-capped) peak is reported beside it."""
    T, d, f = wl.T, wl.d, wl.f
    gu_ms, dn_ms = stage_ms["gate_up_gemm"], stage_ms["down_gemm"]
    esz = 1 if wl.dtype == "bf16_int8w" else 2
    if weight_stream_form(wl, path):   # weight-stream form: HBM bound
        gu_bytes = touched * 2 * d * f * esz
        gu = gu_bytes / (gu_ms / 1e3) / 1e9
        dn = touched * d * f * esz / (dn_ms / 1e3) / 1e9
        # bf16 weights on the automatic path: the gate/up GEMM in 128-row token
        # tiles, the down projection in weight-stream tiles
        kern = ("moe_expert_gemm_kernel<GATEUP, TOKEN_TILE> (128-row tiles)"
                if path == "auto" and wl.dtype == "bf16" else "moe_expert_gemm_kernel<GATEUP, WEIGHT_STREAM>")
        return {"bound": "hbm", "kernel": kern,
                "achieved": round(gu, 1), "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(gu / pk["hbm_gbs"], 4),
                "traffic": recorded_traffic(wl), "peak_source": f"{pk['source']} HBM copy",
                "algorithmic_per_launch": gu_bytes,
                "down_gemm": {"achieved": round(dn, 1), "frac": round(dn / pk["hbm_gbs"], 4)}}
    peak_t, peak_s = pk["bf16_tflops"], pk["bf16_tflops_sustained"]
    gu = 8 * T * d * f / (gu_ms / 1e3) / 1e12
    dn = 4 * T * d * f / (dn_ms / 1e3) / 1e12
    wbytes = wl.E * 2 * d * f * esz
    act = 2 * T * d * 2 + 2 * T * f * 2
    if esz == 1:
        kern = "gate/up expert GEMM, int8 weights, 256-row token tiles"
    elif T >= 512 and path == "auto" and wl.dtype == "bf16":
        kern = "gate/up expert GEMM, bf16, 256-row token tiles on single CTAs"
    else:
        kern = "gate/up expert GEMM, token tiles (single-CTA or CTA-pair form, chosen on the device)"
    out = {"bound": "tensor", "kernel": kern,
           "achieved": round(gu, 1), "peak": peak_t, "unit": "TFLOP/s", "frac": round(gu / peak_t, 4),
           "frac_sustained": round(gu / peak_s, 4), "peak_sustained": peak_s,
           "traffic": recorded_traffic(wl),
           "peak_source": f"{pk['source']} bf16 burst (dense; fp16 operands run at the same rate)",
           "algorithmic_per_launch": 8 * T * d * f,
           "algorithmic_bytes_per_launch": wbytes + act,
           "down_gemm": {"achieved": round(dn, 1), "frac": round(dn / peak_t, 4),
                         "frac_sustained": round(dn / peak_s, 4)}}
    if esz == 1:
        out["weight_gbs"] = round(wbytes / (gu_ms / 1e3) / 1e9, 1)
    return out


def run_e2e(a, moe, inp, run, out, flush, dist, dev, world, flops):
    """Same metric through the public API with every batch in pinned host memory.

    Each timed step copies its x in (host -> device), runs the layer and copies
    its result out (device -> host). Two device buffers per side let the copy of
    step i+1's input and of step i-1's output run on their own streams while
    step i computes, as a serving loop would; the region spans all K steps and
    ends when the last output has reached the host. The serial form (copy in,
    compute, copy out, one after the other) is reported beside it."""
    import torch

    T, d = inp["x"].shape
    K = a.steps
    x_host = inp["x"].cpu().pin_memory()
    out_host = [torch.empty((T, d), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xs = [torch.empty_like(inp["x"]) for _ in range(2)]
    outs = [torch.empty((T, d), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    plain = "s_gate" not in inp and "router_bias" not in inp
    main = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    used = [torch.cuda.Event() for _ in range(2)]      # step done with xs[b] / outs[b]
    fetched = [torch.cuda.Event() for _ in range(2)]   # outs[b] has reached the host

    def forward(x_dev, o):
        if plain:
            moe.moe_forward(x_dev, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], o, stream=main)
        else:
            run(x_dev, o)

    def step(i):
        b = i % 2
        ready = torch.cuda.Event()
        with torch.cuda.stream(h2d):
            h2d.wait_event(used[b])
            xs[b].copy_(x_host, non_blocking=True)
            ready.record(h2d)
        main.wait_event(ready)
        main.wait_event(fetched[b])
        forward(xs[b], outs[b])
        used[b].record(main)
        with torch.cuda.stream(d2h):
            d2h.wait_event(used[b])
            out_host[b].copy_(outs[b], non_blocking=True)
            fetched[b].record(d2h)

    for i in range(a.warmup):
        step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(main)
    h2d.wait_event(t0)
    d2h.wait_event(t0)
    for i in range(K):
        step(i)
    main.wait_stream(h2d)
    main.wait_stream(d2h)
    t1.record(main)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)

    # Serial form: each step's copies and compute back to back on one stream.
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for i in range(K):
        flush.zero_()
        e_s[i].record(main)
        xs[0].copy_(x_host, non_blocking=True)
        forward(xs[0], outs[0])
        out_host[0].copy_(outs[0], non_blocking=True)
        e_e[i].record(main)
    torch.cuda.synchronize()
    serial_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)), dist, dev)
    return {"value": round(world * K * flops / (e2e_ms / 1e3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 2,
            "ms_per_step": round(e2e_ms / K, 4),
            "api": ("moe_forward (library workspace)" if plain else "moe_forward_ex")
                   + ", pinned host x -> device -> pinned host out",
            "overlap": "double-buffered: copies of step i+1's input and step i-1's output on their own streams "
                       "during step i; region from the first copy-in to the last copy-out",
            "l2": "not flushed: every step streams the full weight set (> 70x L2)",
            "serial_value": round(world * K * flops / (serial_ms / 1e3) / 1e12, 2),
            "serial_ms_per_step": round(serial_ms / K, 4)}


def run_decode(a, moe, W, wl, inp, dev, pk):
    """Decode batch (T = 64) on the same weights: the weight-stream form."""
    import torch

    K = a.steps
    d, f = wl.d, wl.f
    Td = W.WORKLOADS["decode"].T
    xd = W.make_x(wl, dev, Td, seed_name="x_decode")
    run = Runner(moe, inp, Td, d, f, dev)
    outd = torch.empty((Td, d), dtype=torch.bfloat16, device=dev)
    cnt = torch.empty(8, dtype=torch.int32, device=dev)
    for _ in range(a.warmup):
        run(xd, outd, debug={"counts": cnt})
    torch.cuda.synchronize()
    touched = int((cnt > 0).sum().item())
    # The step time without the stage events (each event record between two
    # kernels costs the stream a few microseconds), then the same K steps with
    # them for the breakdown.
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        for i in range(K):
            starts[i].record()
            run(xd, outd)
            ends[i].record()
        torch.cuda.synchronize()
    d_ms = statistics.mean(s.elapsed_time(e) for s, e in zip(starts, ends))
    step_ev_ms, stage_ms = timed_steps(run, xd, outd, K, None)
    # Host time of one call (argument checks, plan, tensor maps, launches),
    # measured while the device works through the queue: when it approaches
    # the step time, eager steps wait on the host.
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    for _ in range(K):
        run(xd, outd)
    host_us = (time.perf_counter() - h0) / K * 1e6
    torch.cuda.synchronize()
    wbytes = touched * 3 * d * f * 2
    # The same step captured once in a CUDA graph and replayed (no per-launch
    # host work, no stage events): what a serving loop that replays graphs sees.
    graph = torch.cuda.CUDAGraph()
    # thread_local: CUDA calls of other threads (NCCL's, under torchrun) do not
    # disturb the capture.
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        run(xd, outd)
    torch.cuda.synchronize()
    for _ in range(a.warmup):
        graph.replay()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    g0.record()
    for _ in range(K):
        graph.replay()
    g1.record()
    torch.cuda.synchronize()
    g_ms = g0.elapsed_time(g1) / K
    del graph
    return {"workload": f"grok1-decode T={Td} d={d} f={f} bf16 (same weights)",
            "ms_per_step": round(d_ms, 4), "experts_touched": touched,
            "ms_per_step_with_stage_events": round(statistics.mean(step_ev_ms), 4),
            "clocks": clk.summary(),
            "order": "measured before the prefill steps; no L2 flush (each step streams the touched experts' "
                     "weights, > 70x L2)",
            "hbm_gbs": round(wbytes / (d_ms / 1e3) / 1e9, 1),
            "frac": round(wbytes / (d_ms / 1e3) / 1e9 / pk["hbm_gbs"], 4),
            "gate_up_gbs": round(touched * 2 * d * f * 2 / (stage_ms["gate_up_gemm"] / 1e3) / 1e9, 1),
            "down_gbs": round(touched * d * f * 2 / (stage_ms["down_gemm"] / 1e3) / 1e9, 1),
            "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "graph_ms_per_step": round(g_ms, 4), "graph_hbm_gbs": round(wbytes / (g_ms / 1e3) / 1e9, 1),
            "host_us_per_call": round(host_us, 1),
            "peak_gbs": pk["hbm_gbs"], "bytes_per_step": wbytes}


def run_side(a, moe, wl2, name, inp2, dev, pk, dist, world):
    """One more Grok-1-shape workload measured like the main line: K timed
    steps with an L2 flush between them, CUDA events on the launching stream,
    the library's stage events, clocks sampled during the steps, its own
    roofline entry and a bounded oracle sample on the host cores."""
    import torch

    K = a.steps
    T, d, f = wl2.T, wl2.d, wl2.f
    run = Runner(moe, inp2, T, d, f, dev)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    cnt = torch.empty(8, dtype=torch.int32, device=dev)
    for _ in range(a.warmup):
        flush.zero_()
        run(inp2["x"], out, debug={"counts": cnt})
    torch.cuda.synchronize()
    st, code = moe.moe_device_status(run.ws)
    if st != 0:
        raise SystemExit(f"{wl2.name}: device status {st} code {code:#x}")
    slots = [int(v) for v in cnt.cpu().tolist()]
    touched = sum(1 for v in slots if v > 0)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        step_ms, stage_ms = timed_steps(run, inp2["x"], out, K, flush)
    torch.cuda.synchronize()
    clocks = clk.summary()
    t_max = max_over_ranks(sum(step_ms), dist, dev)
    esz = 1 if wl2.dtype == "bf16_int8w" else 2
    wbytes = touched * 3 * d * f * esz
    entry = {
        "workload": name, "T": T, "d": d, "f": f,
        "ms_per_step": round(t_max / K, 4),
        "value": round(job_throughput(world, K, wl2.flops, t_max) / 1e12, 2), "unit": "TFLOP/s",
        "tokens_per_s": round(job_throughput(world, K, T, t_max), 1),
        "hbm_gbs_weights": round(world * K * wbytes / (t_max / 1e3) / 1e9, 1),
        "weight_bytes": wbytes,
        "expert_slots": slots,
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": roofline_entry(wl2, pk, stage_ms, touched, clocks),
        "gpu_launches": launches_per_step(wl2, "auto") * K,
        "clocks": {k: clocks.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "power_w_max", "samples")},
    }
    if not a.no_cpu_baseline and world == 1:
        dt, n, pair = oracle_pair_sample(inp2, 8)
        entry["cpu_baseline"] = {
            "value": round(12 * d * f * n / dt / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{n} of {T} tokens routed to experts {pair} (routing of all {T}), fp64 numpy, {dt:.1f} s"}
    del run
    return entry


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
    bias = inp["router_bias"].cpu().numpy() if "router_bias" in inp else None
    r = oracle.route(x, wr, bias)
    pairs = {}
    for t, (e0, e1) in enumerate(r["idx"]):
        pairs.setdefault((min(e0, e1), max(e0, e1)), []).append(t)
    groups = [v[:8] for _, v in sorted(pairs.items()) if len(v) >= 1]
    get = expert_getter(inp)

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
        "impl": "reference", "metric": METRIC,
        "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": round(total / a.steps * 1e3, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeded inputs as the b200 arm)",
        "config": {"workload": workload_name, "T": wl.T, "d": wl.d, "f": wl.f, "E": 8, "k": 2},
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"per step up to 8 tokens routed to one expert pair (routing of all {wl.T} "
                                   "tokens done once)"},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
