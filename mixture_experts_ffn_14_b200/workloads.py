"""Seeded synthetic inputs for the MoE feed-forward sublayer.

This module only draws random numbers and casts them; it holds none of the
method's arithmetic, so both the CUDA path and the oracle may take their
inputs from it. Nothing here touches the CUDA library.

Distributions (one recipe for every workload):
  x          ~ N(0, 1)
  w_router   ~ N(0, std = 1/sqrt(d)), float32, layout [d, E]
  w_gate/up  ~ N(0, std = 1/sqrt(d)), layout [E, d, f]
  w_down     ~ N(0, std = 1/sqrt(f)), layout [E, f, d]
  int8 form: q ~ U{-127..127}; per-output-channel scale s ~ U(0.5, 1.5)/(127 sqrt(fan_in))
             stored as bf16; gate/up scales [E, f], down scales [E, d].
  skewed form: a per-expert router-logit bias [5, c, c, 0, 0, 0, 0, 0] with
             c = 0.8644; for i.i.d. N(0,1) logits this sends ~50% of the token
             slots to expert 0, ~15% each to experts 1 and 2 and ~4% to each of
             the other five (c solves P(expert 1 is the larger of the biased
             logits 1..7) = 0.30, a Gaussian order-statistics integral).
"""

from __future__ import annotations

import zlib
from dataclasses import dataclass, field

import numpy as np

SKEW_BIAS = (5.0, 0.8644201890485588, 0.8644201890485588, 0.0, 0.0, 0.0, 0.0, 0.0)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    f: int
    E: int = 8
    k: int = 2
    dtype: str = "bf16"          # "f32", "bf16" or "bf16_int8w"
    seed: int = 0
    skew: bool = False
    note: str = field(default="", compare=False)

    @property
    def flops(self) -> int:
        """Algorithmic FLOPs of one forward: 2*k*(2*d*f + f*d) per token."""
        return self.T * self.k * 2 * 3 * self.d * self.f

    def weight_bytes(self) -> int:
        per = 1 if self.dtype == "bf16_int8w" else (4 if self.dtype == "f32" else 2)
        return self.E * 3 * self.d * self.f * per


WORKLOADS = {
    "tiny": Workload("tiny", 64, 128, 256, dtype="f32", seed=0,
                     note="Tiny MoE layer T=64 d=128 f=256 E=8 top-2, fp32"),
    "prefill": Workload("prefill", 4096, 6144, 32768, dtype="bf16", seed=1,
                        note="Grok-1-shape prefill T=4096 d=6144 f=32768 E=8 top-2, bf16"),
    "decode": Workload("decode", 64, 6144, 32768, dtype="bf16", seed=2,
                       note="Grok-1-shape decode T=64 d=6144 f=32768 E=8 top-2, bf16"),
    "int8": Workload("int8", 1024, 6144, 32768, dtype="bf16_int8w", seed=3,
                     note="int8-weight Grok-1 shape T=1024, per-channel bf16 scales"),
    "skewed": Workload("skewed", 16384, 6144, 32768, dtype="bf16", seed=4, skew=True,
                       note="skewed-load prefill T=16384, router bias -> ~50/15/15/4x5 %"),
}


def tensor_seed(seed: int, name: str) -> int:
    """Per-tensor seed derived from the workload seed and the tensor's name."""
    return (zlib.crc32(name.encode()) ^ (seed * 0x9E3779B1)) & 0x7FFFFFFF


# --------------------------------------------------------------------------
# numpy generator (small shapes; float32 values)
# --------------------------------------------------------------------------

def make_numpy(T: int, d: int, f: int, E: int = 8, seed: int = 0) -> dict:
    """float32 inputs from numpy's PCG64 (default_rng(seed))."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_router = (rng.standard_normal((d, E)) / np.sqrt(d)).astype(np.float32)
    w_gate = (rng.standard_normal((E, d, f)) / np.sqrt(d)).astype(np.float32)
    w_up = (rng.standard_normal((E, d, f)) / np.sqrt(d)).astype(np.float32)
    w_down = (rng.standard_normal((E, f, d)) / np.sqrt(f)).astype(np.float32)
    return {"x": x, "w_router": w_router, "w_gate": w_gate, "w_up": w_up, "w_down": w_down}


def make_numpy_int8(T: int, d: int, f: int, E: int = 8, seed: int = 0) -> dict:
    """int8 weights + per-output-channel scales (values already representable in bf16)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_router = (rng.standard_normal((d, E)) / np.sqrt(d)).astype(np.float32)
    qg = rng.integers(-127, 128, size=(E, d, f), dtype=np.int64).astype(np.int8)
    qu = rng.integers(-127, 128, size=(E, d, f), dtype=np.int64).astype(np.int8)
    qd = rng.integers(-127, 128, size=(E, f, d), dtype=np.int64).astype(np.int8)
    sg = rng.uniform(0.5, 1.5, size=(E, f)) / (127 * np.sqrt(d))
    su = rng.uniform(0.5, 1.5, size=(E, f)) / (127 * np.sqrt(d))
    sd = rng.uniform(0.5, 1.5, size=(E, d)) / (127 * np.sqrt(f))
    return {"x": x, "w_router": w_router, "w_gate": qg, "w_up": qu, "w_down": qd,
            "s_gate": round_bf16_np(sg), "s_up": round_bf16_np(su), "s_down": round_bf16_np(sd)}


def round_bf16_np(a) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even); returns float32."""
    a32 = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = a32.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


# --------------------------------------------------------------------------
# torch generator (any shape; runs where the tensors will live)
# --------------------------------------------------------------------------

def make_torch(w: Workload, device, T: int | None = None) -> dict:
    """Inputs for workload ``w`` as torch tensors on ``device``.

    Weights are drawn one expert at a time in float32 and cast to the storage
    dtype (round-to-nearest-even), so peak extra memory is one expert matrix.
    ``T`` overrides the workload's token count (same weights)."""
    import torch

    T = w.T if T is None else T
    dev = torch.device(device)

    def gen(name):
        g = torch.Generator(device=dev)
        g.manual_seed(tensor_seed(w.seed, name))
        return g

    act = torch.float32 if w.dtype == "f32" else torch.bfloat16
    out = {}
    out["x"] = torch.randn((T, w.d), generator=gen("x"), device=dev, dtype=torch.float32).to(act)
    out["w_router"] = torch.randn((w.d, w.E), generator=gen("w_router"), device=dev,
                                  dtype=torch.float32) / float(np.sqrt(w.d))

    def dense(name, K, N, fan_in):
        t = torch.empty((w.E, K, N), device=dev, dtype=act)
        g = gen(name)
        for e in range(w.E):
            t[e].copy_(torch.randn((K, N), generator=g, device=dev, dtype=torch.float32)
                       / float(np.sqrt(fan_in)))
        return t

    def quant(name, K, N):
        t = torch.empty((w.E, K, N), device=dev, dtype=torch.int8)
        g = gen(name)
        for e in range(w.E):
            t[e].copy_(torch.randint(-127, 128, (K, N), generator=g, device=dev,
                                     dtype=torch.int32).to(torch.int8))
        return t

    def scale(name, N, fan_in):
        u = torch.rand((w.E, N), generator=gen(name), device=dev, dtype=torch.float32)
        return ((0.5 + u) / (127.0 * float(np.sqrt(fan_in)))).to(torch.bfloat16)

    if w.dtype == "bf16_int8w":
        out["w_gate"] = quant("w_gate", w.d, w.f)
        out["w_up"] = quant("w_up", w.d, w.f)
        out["w_down"] = quant("w_down", w.f, w.d)
        out["s_gate"] = scale("s_gate", w.f, w.d)
        out["s_up"] = scale("s_up", w.f, w.d)
        out["s_down"] = scale("s_down", w.d, w.f)
    else:
        out["w_gate"] = dense("w_gate", w.d, w.f, w.d)
        out["w_up"] = dense("w_up", w.d, w.f, w.d)
        out["w_down"] = dense("w_down", w.f, w.d, w.f)
    if w.skew:
        out["router_bias"] = torch.tensor(SKEW_BIAS[: w.E], device=dev, dtype=torch.float32)
    return out


def make_x(w: Workload, device, T: int, seed_name: str = "x"):
    """A fresh activation batch [T, d] for workload ``w`` (same recipe as ``x``)."""
    import torch

    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(tensor_seed(w.seed, seed_name))
    act = torch.float32 if w.dtype == "f32" else torch.bfloat16
    return torch.randn((T, w.d), generator=g, device=dev, dtype=torch.float32).to(act)
