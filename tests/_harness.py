"""Shared helpers of the parity tests: run the CUDA path through the C ABI and
compare with the oracle. The oracle only ever receives the generated inputs;
where several routings are correct (near ties) the GPU's choice is accepted
only if the oracle itself lists it among the valid alternatives."""

from __future__ import annotations

import numpy as np
import torch

import mixture_experts_ffn_14_b200 as moe
import oracle

ATOL, RTOL = 1e-2, 2e-2          # |gpu - ref| <= 1e-2 + 2e-2 |ref|
GATE_ATOL = 2e-6                 # fp32 softmax against the fp64 one
TIE_EPS = 1e-6                   # near-tie exclusion on probabilities


def np64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_gpu(inp: dict, *, path=moe.MOE_PATH_AUTO, activation=moe.MOE_ACT_GELU_TANH, down_splits=0, want_h=True,
            stream=None, renormalize=False, residual=None, post_norm_weight=None, norm_eps=1e-5,
            row_gather=False, separate_combine=False) -> dict:
    """One forward through moe_forward_ex with every debug output requested."""
    x = inp["x"]
    T, d = x.shape
    E, _, f = inp["w_gate"].shape
    dev = x.device
    dt = moe.dtype_code(x, inp["w_gate"])
    ws = torch.empty(moe.moe_workspace_size(T, d, f, E, 2, dt, path, down_splits), dtype=torch.uint8, device=dev)
    out = torch.empty((T, d), dtype=x.dtype, device=dev)
    dbg = {
        "idx": torch.empty((T, 2), dtype=torch.int32, device=dev),
        "gates": torch.empty((T, 2), dtype=torch.float32, device=dev),
        "counts": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "perm_token": torch.empty(2 * T, dtype=torch.int32, device=dev),
        "perm_slot": torch.empty(2 * T, dtype=torch.int32, device=dev),
    }
    if want_h:   # the int8-weight path keeps its intermediate in fp16
        h_dtype = torch.float16 if inp["w_gate"].dtype == torch.int8 else x.dtype
        dbg["h"] = torch.empty((2 * T, f), dtype=h_dtype, device=dev)
    scales = (inp["s_gate"], inp["s_up"], inp["s_down"]) if "s_gate" in inp else None
    moe.moe_forward_ex(x, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out, ws, scales=scales,
                       router_bias=inp.get("router_bias"), activation=activation, path=path, down_splits=down_splits,
                       renormalize=renormalize, residual=residual, post_norm_weight=post_norm_weight,
                       norm_eps=norm_eps, row_gather=row_gather, separate_combine=separate_combine,
                       debug=dbg, stream=stream)
    torch.cuda.synchronize()
    st, code = moe.moe_device_status(ws)
    assert st == 0 and code == 0, f"device status {st} code {code:#x}"
    res = {k: v.cpu().numpy() for k, v in dbg.items() if k != "h"}
    res["out"] = np64(out)
    if want_h:
        res["h"] = dbg["h"]
    return res


def expected_routing(x64, wr64, bias64, gpu_idx, renormalize=False) -> tuple:
    """Oracle routing; near-tie tokens take the GPU's pair only if the oracle
    lists it as valid. Returns (routing dict with idx/gates, n_excluded)."""
    r = oracle.route(x64, wr64, bias64)
    tie = oracle.near_tie_mask(r["probs"], eps=TIE_EPS)
    idx = r["idx"].copy()
    amb = np.nonzero(tie["select"] | tie["order"])[0]
    for t in amb:
        alts = oracle.route_alternatives(r, int(t), eps=TIE_EPS)
        g = tuple(int(v) for v in gpu_idx[t])
        if g in alts:
            idx[t] = g
    gates = np.take_along_axis(r["probs"], idx.astype(np.int64), axis=1)
    if renormalize:
        gates = gates / gates.sum(axis=1, keepdims=True)
    return {"idx": idx, "gates": gates, "probs": r["probs"], "logits32": r["logits32"]}, len(amb)


def check_routing_and_dispatch(gpu: dict, routing: dict):
    T = routing["idx"].shape[0]
    mism = np.nonzero((gpu["idx"] != routing["idx"]).any(1))[0]
    assert mism.size == 0, f"routing differs on {mism.size} tokens, e.g. {mism[:5]}"
    assert np.max(np.abs(gpu["gates"] - routing["gates"])) <= GATE_ATOL
    dsp = oracle.dispatch(routing["idx"], 8)
    assert (gpu["counts"] == dsp["counts"]).all()
    assert (gpu["offsets"] == dsp["offsets"]).all()
    assert (gpu["perm_token"] == dsp["perm_token"]).all()
    assert (gpu["perm_slot"] == dsp["perm_slot"]).all()
    assert gpu["counts"].sum() == 2 * T
    return dsp


def assert_close(got, ref, what="out"):
    err = np.abs(got - ref)
    lim = ATOL + RTOL * np.abs(ref)
    bad = err > lim
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                           f"max |err| {err.max():.3e}, worst ratio {(err / lim).max():.2f}")
    return float((err / lim).max())


def oracle_inputs(inp: dict) -> dict:
    """Exact float64 / int views of the generated inputs for the oracle."""
    o = {"x": np64(inp["x"]), "w_router": np64(inp["w_router"]),
         "bias": np64(inp["router_bias"]) if "router_bias" in inp else None}
    return o


def expert_getter(inp: dict):
    """Callable e -> one expert's float64 (dequantised) matrices, copied from
    the generated tensors one expert at a time."""
    def get(e):
        if "s_gate" in inp:
            return tuple(
                oracle.dequant_int8(inp[w][e].cpu().numpy(), np64(inp[s][e]))
                for w, s in (("w_gate", "s_gate"), ("w_up", "s_up"), ("w_down", "s_down")))
        return tuple(np64(inp[w][e]) for w in ("w_gate", "w_up", "w_down"))
    return get


def full_check(inp: dict, gpu: dict, tokens=None, check_h=True, gelu_mode="tanh", renormalize=False,
               residual=None, post_norm_weight=None, norm_eps=1e-5):
    """Routing + dispatch bit-exact, out (and h) within tolerance on `tokens`.
    With residual / post_norm_weight the oracle output is post-normed and added
    to the residual row by row, as the library's options ask for."""
    o = oracle_inputs(inp)
    routing, n_amb = expected_routing(o["x"], o["w_router"], o["bias"], gpu["idx"], renormalize)
    dsp = check_routing_and_dispatch(gpu, routing)
    T = o["x"].shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    res = oracle.forward_sparse(o["x"], o["w_router"], expert_getter(inp), routing=routing, tokens=tok,
                                return_h=check_h, gelu_mode=gelu_mode)
    ref = res["out"]
    if residual is not None or post_norm_weight is not None:
        ref = oracle.post_norm_residual(ref, None if residual is None else np64(residual)[tok],
                                        None if post_norm_weight is None else np64(post_norm_weight), norm_eps)
    worst = assert_close(gpu["out"][tok], ref, "out")
    if check_h:
        pos = dsp["slot_pos"][tok]               # [n, 2] permuted rows of each (token, slot)
        h_gpu = np64(gpu["h"][torch.as_tensor(pos.reshape(-1), device=gpu["h"].device)])
        h_gpu = h_gpu.reshape(len(tok), 2, -1)
        assert_close(h_gpu, res["h"], "h")
    return {"worst": worst, "ambiguous": n_amb}
