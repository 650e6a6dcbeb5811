"""Oracle: a plain, slow, obviously correct CPU evaluation of the Grok-1 MoE
feed-forward sublayer (router -> top-2 -> GeGLU experts -> gate-weighted sum).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py``, never by the product
path. It shares no code, constant or helper with the CUDA library.

Precision: every floating-point step is float64 with no intermediate rounding,
except that the router logits are rounded once to float32. The routing
decision (which two experts) is an integer decided by comparing logits; the
CUDA router compares float32 logits, so both sides take that decision in
float32 (the kernel's precision: the pages only say "fp32 routing").

Sources (page title, section):
  [blueprint] grok-field-guide, "Grok-1 blueprint", section "MoE 子层" (MoE sublayer):
              router projects each 6144-d token to 8 logits, softmax, top-2; each
              expert is a gated FFN (two input projections, GELU on one, elementwise
              product, projection back to hidden size); selected outputs are
              multiplied by their gates and summed.
  [ch10]      Grok-1 book, ch. 10 "与其他 MoE 对比" (comparison with other MoE):
              §10.3 routing table (softmax before top-k, gates not renormalised,
              capacity field defined but unused, no token drop);
              §10.3.1 Grok-1 vs Mixtral (Grok keeps top-k softmax probabilities as
              gates, their sum is below 1);
              §10.3.2 capacity-factor box (no drop logic in the inference code);
              §10.4 expert-structure table and "GeGLU vs SwiGLU" box
              (down(act(up_1 x) * up_2 x), act = GELU for Grok-1, f = 32768).
  [ch1]       Grok-1 book, ch. 1 "引言" (introduction), §1.2 "314B = 8 x ? + 共享":
              SwiGLU box (f = ffn_size(6144, 8) = 8*6144*2//3 = 32768; the three
              expert matrices are bias-free), INT8 box (int8 values plus one scale
              per row/channel, dequantised at compute time).
  [ch11]      Grok-1 book, ch. 11 "工程教训与遗产" (engineering lessons), §11.3.1
              item 3: the published code evaluates all 8 experts densely and keeps
              2 with a one-hot mask.

Readings where the pages are silent, ambiguous or disagree:
  R1  GELU is the tanh approximation 0.5 z (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3)))
      by default; [ch10] §10.4 writes GELU as z * Phi(z) (erf form), kept as mode "erf".
  R2  GELU is applied to the w_gate projection; w_up is linear; w_down projects back.
  R3  Gates are the softmax probabilities of the two selected experts, not
      renormalised, so 0 < g0 + g1 <= 1 ([ch10] §10.3.1; the ssnai page's "gates sum
      to 1" check contradicts it and is not followed).
  R4  Top-2 is by descending float32 logit; an exact tie goes to the lower expert
      index; slot 0 holds the larger one.
  R5  Dispatch order is stable by (expert ascending, token ascending); there is no
      capacity limit and no drop ([ch10] §10.3.2).
  R6  w_router is [d, E]; an optional per-expert router bias is added to the logits
      before the float32 rounding (used only to build the skewed-load workload).
  R7  int8 weights: W[e, i, j] = q[e, i, j] * s[e, j], one scale per output channel j
      ([ch1] INT8 box), dequantised here in float64.
  R8  Mixtral-style routing ([ch10] §10.3.1 listing): the top-k probabilities divided
      by their sum; this equals a softmax over the k selected logits, so the table's
      "top-k -> softmax" and the listing's "softmax -> top-k -> renormalise" agree.
      Its experts use SiLU (z * sigmoid(z)) on the gate branch ([ch10] §10.4 box).
  R9  Sandwich post-norm ([ch10] §10.3.1: the post-RMSNorm compensates the gate sum
      below 1; [blueprint] "MoE sublayer": the combined output is added back to the
      trunk). The pages give no RMSNorm formula: the standard
      w * y / sqrt(mean(y^2) + eps) over the hidden axis is used, eps a parameter.
"""

from __future__ import annotations

import math
from typing import Callable, Sequence

import numpy as np

ACTIVATIONS = ("tanh", "erf", "silu")
GELU_MODES = ACTIVATIONS  # name kept for the GELU forms

_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)


def ffn_size(emb_size: int, widening_factor: float) -> int:
    """Expert hidden width: int(widening * emb) * 2 // 3 ([ch1] §1.2 SwiGLU box)."""
    return int(widening_factor * emb_size) * 2 // 3


def gelu_tanh(z: np.ndarray) -> np.ndarray:
    """GELU, tanh approximation (reading R1), float64."""
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + np.tanh(_SQRT_2_OVER_PI * (z + 0.044715 * z * z * z)))


def gelu_erf(z: np.ndarray) -> np.ndarray:
    """GELU as z * Phi(z), Phi the standard normal CDF ([ch10] §10.4 box), float64."""
    z = np.asarray(z, dtype=np.float64)
    erf = np.vectorize(math.erf, otypes=[np.float64])
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def silu(z: np.ndarray) -> np.ndarray:
    """SiLU z * sigmoid(z), float64 (Mixtral experts, reading R8)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def _gelu(z: np.ndarray, mode: str) -> np.ndarray:
    if mode == "tanh":
        return gelu_tanh(z)
    if mode == "erf":
        return gelu_erf(z)
    if mode == "silu":
        return silu(z)
    raise ValueError(f"unknown activation {mode!r}")


def post_norm_residual(y, residual=None, weight=None, eps: float = 1e-5) -> np.ndarray:
    """Sandwich post-norm and residual add of the sublayer output (reading R9):
    out = residual + weight * y / sqrt(mean(y^2) + eps) over the last axis;
    either part may be absent (weight None: no norm; residual None: no add)."""
    y64 = np.asarray(y, dtype=np.float64)
    out = y64
    if weight is not None:
        ms = np.mean(y64 * y64, axis=-1, keepdims=True)
        out = np.asarray(weight, dtype=np.float64) * y64 / np.sqrt(ms + eps)
    if residual is not None:
        out = np.asarray(residual, dtype=np.float64) + out
    return out


def softmax_fp64(logits: np.ndarray) -> np.ndarray:
    """Softmax over the expert axis, evaluated in float64 ([ch10] §10.3.1)."""
    l64 = np.asarray(logits, dtype=np.float64)
    m = np.max(l64, axis=-1, keepdims=True)
    e = np.exp(l64 - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def route(x, w_router, router_bias=None, k: int = 2, renormalize: bool = False) -> dict:
    """Router: logits = x . w_router (+ bias), rounded once to float32;
    probs = softmax(logits) in float64; top-k experts by descending logit
    (ties -> lower index); gates = probs of the chosen experts, NOT renormalised
    (Grok-1), or divided by their sum with ``renormalize`` (Mixtral, reading R8).

    [blueprint] "MoE sublayer"; [ch10] §10.3 table and §10.3.1; readings R3, R4, R6, R8.

    x: [T, d]; w_router: [d, E]; router_bias: [E] or None.
    Returns dict with logits32 [T,E] float32, probs [T,E] float64,
    idx [T,k] int32, gates [T,k] float64.
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w_router, dtype=np.float64)
    acc = x64 @ w64
    if router_bias is not None:
        acc = acc + np.asarray(router_bias, dtype=np.float64)[None, :]
    logits32 = acc.astype(np.float32)
    probs = softmax_fp64(logits32)
    # Stable sort of the negated logits: descending order, equal logits keep
    # ascending expert index.
    order = np.argsort(-logits32, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    gates = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    if renormalize:  # Mixtral-style (reading R8)
        gates = gates / np.sum(gates, axis=1, keepdims=True)
    return {"logits32": logits32, "probs": probs, "idx": idx, "gates": gates}


def near_tie_mask(probs: np.ndarray, k: int = 2, eps: float = 1e-6) -> dict:
    """Tokens whose routing is ambiguous at float32 rounding level.

    select: |p(k-th) - p(k+1-th)| < eps -> which experts are chosen may differ.
    order:  |p(1st) - p(2nd)| < eps     -> the slot order of the two may differ.
    """
    p = -np.sort(-np.asarray(probs, dtype=np.float64), axis=1)
    select = (p[:, k - 1] - p[:, k]) < eps
    order = (p[:, 0] - p[:, 1]) < eps
    return {"select": select, "order": order}


def route_alternatives(routing: dict, t: int, k: int = 2, eps: float = 1e-6) -> list:
    """All top-k orderings of token t that are correct within eps of probability:
    every pair (a, b) of distinct experts such that each chosen probability is
    within eps of the one at its rank and every unchosen one is not above the
    k-th by more than eps. Used to validate near-tie tokens (reading R4)."""
    p = np.asarray(routing["probs"][t], dtype=np.float64)
    srt = -np.sort(-p)
    out = []
    E = p.shape[0]
    for a in range(E):
        for b in range(E):
            if a == b:
                continue
            pair = (a, b)
            ok = all(abs(p[pair[r]] - srt[r]) < eps for r in range(k))
            rest = [p[e] for e in range(E) if e not in pair]
            ok = ok and all(v <= srt[k - 1] + eps for v in rest)
            if ok:
                out.append(pair)
    return out


def dispatch(idx: np.ndarray, E: int) -> dict:
    """Integer dispatch: per-expert counts, exclusive offsets, and the stable
    permutation of (token, slot) pairs sorted by (expert, token) (reading R5;
    no capacity, no drop, [ch10] §10.3.2).

    Returns counts [E], offsets [E+1], perm_token [T*k], perm_slot [T*k],
    slot_pos [T,k] (position of (t, s) in the permuted order)."""
    idx = np.asarray(idx)
    T, k = idx.shape
    for t in range(T):
        if len(set(int(v) for v in idx[t])) != k:
            raise ValueError(f"token {t} does not have {k} distinct experts")
    counts = np.zeros(E, dtype=np.int64)
    for e in range(E):
        counts[e] = np.count_nonzero(idx == e)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm_token = []
    perm_slot = []
    for e in range(E):
        # Row-major nonzero: tokens ascending; a token holds expert e in one slot only.
        tt, ss = np.nonzero(idx == e)
        perm_token.extend(int(v) for v in tt)
        perm_slot.extend(int(v) for v in ss)
    perm_token = np.asarray(perm_token, dtype=np.int64)
    perm_slot = np.asarray(perm_slot, dtype=np.int64)
    slot_pos = np.empty((T, k), dtype=np.int64)
    slot_pos[perm_token, perm_slot] = np.arange(T * k, dtype=np.int64)
    return {
        "counts": counts,
        "offsets": offsets,
        "perm_token": perm_token,
        "perm_slot": perm_slot,
        "slot_pos": slot_pos,
    }


def dequant_int8(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """W = q * s with one scale per output channel (last axis), float64 (reading R7)."""
    q64 = np.asarray(q).astype(np.float64)
    s64 = np.asarray(s, dtype=np.float64)
    return q64 * s64[..., None, :]


def expert_ffn(xrows, wg, wu, wd, gelu_mode: str = "tanh"):
    """One GeGLU expert on a block of rows, float64, no biases:
    h = GELU(x . wg) * (x . wu);  y = h . wd   ([ch10] §10.4 box; [ch1] §1.2; R2).

    xrows [n, d]; wg, wu [d, f]; wd [f, d]. Returns (y [n, d], h [n, f])."""
    x64 = np.asarray(xrows, dtype=np.float64)
    a = x64 @ np.asarray(wg, dtype=np.float64)
    b = x64 @ np.asarray(wu, dtype=np.float64)
    h = _gelu(a, gelu_mode) * b
    y = h @ np.asarray(wd, dtype=np.float64)
    return y, h


def _expert_getter(experts) -> Callable[[int], tuple]:
    if callable(experts):
        return experts
    wg, wu, wd = experts[:3]
    scales = experts[3] if len(experts) > 3 else None
    if scales is None:
        return lambda e: (wg[e], wu[e], wd[e])
    sg, su, sd = scales
    return lambda e: (
        dequant_int8(wg[e], sg[e]),
        dequant_int8(wu[e], su[e]),
        dequant_int8(wd[e], sd[e]),
    )


def forward_sparse(
    x,
    w_router,
    experts,
    *,
    E: int = 8,
    k: int = 2,
    router_bias=None,
    gelu_mode: str = "tanh",
    tokens: Sequence[int] | None = None,
    routing: dict | None = None,
    return_h: bool = False,
    renormalize: bool = False,
) -> dict:
    """Sparse evaluation, expert by expert: out[t] = sum_s g_s * FFN_{e_s}(x[t]).

    [blueprint] "MoE sublayer"; [ch10] §10.3.1 (no renormalisation), §10.4 (GeGLU).

    experts: (wg [E,d,f], wu [E,d,f], wd [E,f,d]) or (q_g, q_u, q_d, (s_g, s_u, s_d))
             for int8 weights, or a callable e -> (wg_e, wu_e, wd_e) that returns
             one expert's (already dequantised) matrices.
    tokens:  subset of token ids to evaluate (default: all). Routing is always
             computed for all tokens unless ``routing`` is given.
    Returns dict(out [n, d] float64, routing, and h [n, k, f] if return_h).
    """
    x = np.asarray(x)
    T = x.shape[0]
    if routing is None:
        routing = route(x, w_router, router_bias, k, renormalize)
    idx, gates = routing["idx"], routing["gates"]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    get = _expert_getter(experts)
    n = tok.shape[0]
    contrib = None
    h_all = None
    for e in range(E):
        rows, slots = np.nonzero(idx[tok] == e)  # rows index into tok
        if rows.size == 0:
            continue
        wg, wu, wd = get(e)
        y, h = expert_ffn(x[tok[rows]], wg, wu, wd, gelu_mode)
        if contrib is None:
            contrib = np.zeros((n, k, y.shape[1]), dtype=np.float64)
        contrib[rows, slots, :] = gates[tok[rows], slots][:, None] * y
        if return_h:
            if h_all is None:
                h_all = np.zeros((n, k, h.shape[1]), dtype=np.float64)
            h_all[rows, slots, :] = h
    if contrib is None:
        d = np.asarray(w_router).shape[0]
        contrib = np.zeros((n, k, d), dtype=np.float64)
    out = contrib[:, 0, :].copy()
    for s in range(1, k):
        out = out + contrib[:, s, :]
    res = {"out": out, "routing": routing, "tokens": tok}
    if return_h:
        res["h"] = h_all
    return res


def forward_dense_bruteforce(
    x, w_router, experts, *, E: int = 8, k: int = 2, router_bias=None,
    gelu_mode: str = "tanh", renormalize: bool = False,
) -> np.ndarray:
    """Dense brute force, the way the published code does it ([ch11] §11.3.1
    item 3): evaluate all E experts on every token, then keep the top-k with a
    gate-weighted one-hot mask and sum over experts. float64."""
    x = np.asarray(x)
    T = x.shape[0]
    routing = route(x, w_router, router_bias, k, renormalize)
    mask = np.zeros((T, E), dtype=np.float64)
    for t in range(T):
        for s in range(k):
            mask[t, routing["idx"][t, s]] = routing["gates"][t, s]
    get = _expert_getter(experts)
    out = None
    for e in range(E):
        wg, wu, wd = get(e)
        y, _ = expert_ffn(x, wg, wu, wd, gelu_mode)
        term = mask[:, e:e + 1] * y
        out = term if out is None else out + term
    return out
