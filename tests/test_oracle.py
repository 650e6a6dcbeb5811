"""Pins for the CPU oracle: each test ties it to something other than itself
(values the pages print, closed forms, library routines, brute force,
invariants), so that a dropped term, a wrong sign or index, or a transposed
operand anywhere in the oracle fails at least one of them. CPU only."""

import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats
import torch

import oracle
from mixture_experts_ffn_14_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


def _rand_problem(T=12, d=24, f=40, E=8, seed=0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((d, E)) / math.sqrt(d)
    wg = rng.standard_normal((E, d, f)) / math.sqrt(d)
    wu = rng.standard_normal((E, d, f)) / math.sqrt(d)
    wd = rng.standard_normal((E, f, d)) / math.sqrt(f)
    return x, wr, wg, wu, wd


def _torch_geglu(x, wg, wu, wd, mode="tanh"):
    """Library evaluation (torch float64) of one GeGLU expert."""
    xt = torch.from_numpy(np.asarray(x, np.float64))
    a = xt @ torch.from_numpy(np.asarray(wg, np.float64))
    b = xt @ torch.from_numpy(np.asarray(wu, np.float64))
    act = torch.nn.functional.gelu(a, approximate="tanh" if mode == "tanh" else "none")
    return ((act * b) @ torch.from_numpy(np.asarray(wd, np.float64))).numpy()


# ---------------------------------------------------------------- shapes --

def test_ffn_size_and_param_counts_match_pages():
    g = _load("grok1_shapes.json")
    f = oracle.ffn_size(g["emb_size"], g["widening_factor"])
    assert f == g["ffn_size"]
    assert 3 * g["emb_size"] * f == g["params_per_expert"]
    assert round(3 * g["emb_size"] * f / 1e9, 3) == g["params_per_expert_rounded_billion"]
    assert round(g["num_experts"] * 3 * g["emb_size"] * f / 1e9, 2) == g["params_per_layer_rounded_billion"]
    w = workloads.WORKLOADS["prefill"]
    assert (w.d, w.f, w.E, w.k) == (g["emb_size"], g["ffn_size"], g["num_experts"],
                                   g["num_selected_experts"])


# ------------------------------------------------------------------ GELU --

def test_gelu_tanh_matches_library():
    z = np.linspace(-12, 12, 4001)
    ref = torch.nn.functional.gelu(torch.from_numpy(z), approximate="tanh").numpy()
    np.testing.assert_allclose(oracle.gelu_tanh(z), ref, rtol=1e-14, atol=1e-15)


def test_gelu_erf_matches_normal_cdf():
    z = np.linspace(-12, 12, 2001)
    np.testing.assert_allclose(oracle.gelu_erf(z), z * scipy.stats.norm.cdf(z),
                               rtol=1e-12, atol=1e-14)


def test_gelu_identities_and_tanh_vs_erf_bound():
    z = np.linspace(-8, 8, 1601)
    for fn in (oracle.gelu_tanh, oracle.gelu_erf):
        assert fn(np.array([0.0]))[0] == 0.0
        # Phi(-z) = 1 - Phi(z)  =>  gelu(z) - gelu(-z) = z (also for the tanh form)
        np.testing.assert_allclose(fn(z) - fn(-z), z, atol=1e-12)
        assert abs(fn(np.array([30.0]))[0] - 30.0) < 1e-12
        assert abs(fn(np.array([-30.0]))[0]) < 1e-12
    gap = np.max(np.abs(oracle.gelu_tanh(z) - oracle.gelu_erf(z)))
    assert 1e-5 < gap < 1e-3


# --------------------------------------------------------------- routing --

def test_softmax_matches_library():
    rng = np.random.default_rng(3)
    l = rng.standard_normal((50, 8)).astype(np.float32)
    np.testing.assert_allclose(oracle.softmax_fp64(l),
                               scipy.special.softmax(l.astype(np.float64), axis=1),
                               rtol=1e-13)


def test_route_closed_form_golden():
    g = _load("routing_closed_form.json")
    d = 8
    x = np.zeros((1, d))
    x[0, 0] = 1.0
    wr = np.zeros((d, 8))
    wr[0, :] = np.log(np.arange(1, 9, dtype=np.float64))
    r = oracle.route(x, wr)
    assert list(r["idx"][0]) == g["idx"]
    l32 = np.log(np.arange(1, 9, dtype=np.float64)).astype(np.float32).astype(np.float64)
    # The float32 rounding of log(i) perturbs the exact i/36 by ~1e-8 relative.
    np.testing.assert_allclose(r["gates"][0], np.array(g["gates_num"]) / g["gates_den"], rtol=1e-6)
    np.testing.assert_allclose(r["gates"][0], np.exp(l32[g["idx"]]) / np.exp(l32).sum(), rtol=1e-14)
    assert r["gates"][0].sum() < 1.0
    assert abs(r["gates"][0].sum() - g["gate_sum_num"] / g["gates_den"]) < 1e-6


def test_route_zero_router_tie_break():
    g = _load("routing_closed_form.json")["uniform_case"]
    x = np.random.default_rng(1).standard_normal((5, 16))
    r = oracle.route(x, np.zeros((16, 8)))
    assert (r["idx"] == np.array(g["idx"])).all()
    assert np.all(r["gates"] == g["gate"])


def test_route_matches_bruteforce_over_all_pairs():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((200, 32))
    wr = rng.standard_normal((32, 8)) / math.sqrt(32)
    r = oracle.route(x, wr)
    # Brute force: probabilities from the library softmax, every one of the 28
    # unordered pairs scored by its probability sum, best pair wins.
    p = scipy.special.softmax(r["logits32"].astype(np.float64), axis=1)
    for t in range(x.shape[0]):
        best = max(itertools.combinations(range(8), 2), key=lambda ab: p[t, ab[0]] + p[t, ab[1]])
        assert set(best) == set(int(v) for v in r["idx"][t])
        e0, e1 = r["idx"][t]
        assert p[t, e0] >= p[t, e1]
        np.testing.assert_allclose(r["gates"][t], p[t, [e0, e1]], rtol=1e-13)
        assert 0.0 < r["gates"][t].sum() <= 1.0


def test_route_logits_are_the_float32_rounding_of_the_exact_product():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((40, 64)).astype(np.float32)
    wr = (rng.standard_normal((64, 8)) / 8).astype(np.float32)
    r = oracle.route(x, wr)
    # Exact products of float32 values, summed with math.fsum (correctly rounded).
    for t in range(0, 40, 7):
        for e in range(8):
            exact = math.fsum(float(x[t, i]) * float(wr[i, e]) for i in range(64))
            assert r["logits32"][t, e] == np.float32(exact)


def test_router_bias_is_a_logit_shift():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 16))
    wr = rng.standard_normal((16, 8)) / 4
    bias = rng.standard_normal(8)
    r1 = oracle.route(x, wr, router_bias=bias)
    # Same logits through an extra constant input feature carrying the bias.
    r2 = oracle.route(np.concatenate([x, np.ones((64, 1))], 1), np.concatenate([wr, bias[None]], 0))
    np.testing.assert_allclose(r1["logits32"], r2["logits32"], rtol=1e-6, atol=1e-6)
    ok = ~oracle.near_tie_mask(r1["probs"])["select"]
    assert (np.sort(r1["idx"], 1)[ok] == np.sort(r2["idx"], 1)[ok]).all()


def test_near_tie_mask_and_alternatives():
    probs = np.array([[0.3, 0.2, 0.2 - 5e-7, 0.1, 0.1, 0.05, 0.03, 0.02 + 5e-7],
                      [0.4, 0.4 - 1e-7, 0.1, 0.05, 0.03, 0.01, 0.005, 0.005 + 1e-7]])
    m = oracle.near_tie_mask(probs)
    assert list(m["select"]) == [True, False]
    assert list(m["order"]) == [False, True]
    alts0 = oracle.route_alternatives({"probs": probs}, 0)
    assert set(alts0) == {(0, 1), (0, 2)}
    alts1 = oracle.route_alternatives({"probs": probs}, 1)
    assert set(alts1) == {(0, 1), (1, 0)}


# -------------------------------------------------------------- dispatch --

def test_dispatch_matches_sort_reference():
    rng = np.random.default_rng(2)
    T = 300
    idx = np.stack([rng.permutation(8)[:2] for _ in range(T)]).astype(np.int32)
    dsp = oracle.dispatch(idx, 8)
    tok = np.repeat(np.arange(T), 2)
    slot = np.tile(np.arange(2), T)
    exp = idx.reshape(-1)
    order = np.lexsort((tok, exp))          # primary key expert, then token
    assert (dsp["perm_token"] == tok[order]).all()
    assert (dsp["perm_slot"] == slot[order]).all()
    assert (dsp["counts"] == np.bincount(exp, minlength=8)).all()
    assert dsp["counts"].sum() == 2 * T
    assert dsp["offsets"][0] == 0 and dsp["offsets"][-1] == 2 * T
    # slot_pos is the inverse of the permutation
    assert (dsp["perm_token"][dsp["slot_pos"]] == np.arange(T)[:, None]).all()
    assert (dsp["perm_slot"][dsp["slot_pos"]] == np.arange(2)[None, :]).all()
    assert sorted(dsp["slot_pos"].reshape(-1)) == list(range(2 * T))


def test_dispatch_empty_and_full_experts():
    T = 9
    idx = np.array([[0, 3]] * T, dtype=np.int32)
    idx[4] = [3, 0]
    dsp = oracle.dispatch(idx, 8)
    assert list(dsp["counts"]) == [T, 0, 0, T, 0, 0, 0, 0]
    assert list(dsp["perm_token"][:T]) == list(range(T))
    assert list(dsp["perm_slot"][:T]) == [0, 0, 0, 0, 1, 0, 0, 0, 0]
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[1, 1]], dtype=np.int32), 8)


# ------------------------------------------------------------ expert math --

@pytest.mark.parametrize("mode", ["tanh", "erf"])
def test_sparse_equals_dense_one_hot_bruteforce(mode):
    x, wr, wg, wu, wd = _rand_problem()
    sp = oracle.forward_sparse(x, wr, (wg, wu, wd), gelu_mode=mode)["out"]
    dn = oracle.forward_dense_bruteforce(x, wr, (wg, wu, wd), gelu_mode=mode)
    np.testing.assert_allclose(sp, dn, rtol=1e-12, atol=1e-14)


def test_expert_ffn_matches_library():
    x, wr, wg, wu, wd = _rand_problem(T=7, d=20, f=36)
    for mode in ("tanh", "erf"):
        y, _ = oracle.expert_ffn(x, wg[3], wu[3], wd[3], mode)
        np.testing.assert_allclose(y, _torch_geglu(x, wg[3], wu[3], wd[3], mode), rtol=1e-12, atol=1e-14)


def test_identical_experts_reduce_to_one_dense_ffn():
    x, wr, wg, wu, wd = _rand_problem(T=10, d=16, f=24)
    wg[:] = wg[0]
    wu[:] = wu[0]
    wd[:] = wd[0]
    res = oracle.forward_sparse(x, wr, (wg, wu, wd))
    gsum = res["routing"]["gates"].sum(1, keepdims=True)
    np.testing.assert_allclose(res["out"], gsum * _torch_geglu(x, wg[0], wu[0], wd[0]),
                               rtol=1e-12, atol=1e-14)


def test_gelu_sits_on_the_gate_branch():
    x, wr, wg, wu, wd = _rand_problem(T=10, d=16, f=24)
    base = oracle.forward_sparse(x, wr, (wg, wu, wd))["out"]
    up2 = oracle.forward_sparse(x, wr, (wg, 2 * wu, wd))["out"]
    dn3 = oracle.forward_sparse(x, wr, (wg, wu, 3 * wd))["out"]
    gt2 = oracle.forward_sparse(x, wr, (2 * wg, wu, wd))["out"]
    np.testing.assert_allclose(up2, 2 * base, rtol=1e-12, atol=1e-14)   # linear in w_up
    np.testing.assert_allclose(dn3, 3 * base, rtol=1e-12, atol=1e-14)   # linear in w_down
    assert np.max(np.abs(gt2 - 2 * base)) > 1e-2                        # not linear in w_gate
    zero = oracle.forward_sparse(x, wr, (wg, 0 * wu, wd))["out"]
    assert np.all(zero == 0.0)


def test_permutation_invariances():
    x, wr, wg, wu, wd = _rand_problem(T=10, d=16, f=24)
    base = oracle.forward_sparse(x, wr, (wg, wu, wd))["out"]
    rng = np.random.default_rng(9)
    pf = rng.permutation(24)
    out_f = oracle.forward_sparse(x, wr, (wg[:, :, pf], wu[:, :, pf], wd[:, pf, :]))["out"]
    np.testing.assert_allclose(out_f, base, rtol=1e-12, atol=1e-14)
    pe = rng.permutation(8)
    out_e = oracle.forward_sparse(x, wr[:, pe], (wg[pe], wu[pe], wd[pe]))["out"]
    np.testing.assert_allclose(out_e, base, rtol=1e-12, atol=1e-14)
    pt = rng.permutation(10)
    out_t = oracle.forward_sparse(x[pt], wr, (wg, wu, wd))["out"]
    np.testing.assert_allclose(out_t, base[pt], rtol=1e-12, atol=1e-14)


def test_token_subset_and_callable_experts():
    x, wr, wg, wu, wd = _rand_problem(T=20)
    full = oracle.forward_sparse(x, wr, (wg, wu, wd), return_h=True)
    sub = [3, 17, 0, 8]
    part = oracle.forward_sparse(x, wr, lambda e: (wg[e], wu[e], wd[e]), tokens=sub, return_h=True)
    np.testing.assert_allclose(part["out"], full["out"][sub], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(part["h"], full["h"][sub], rtol=1e-12, atol=1e-15)


def test_scalar_case_d1_f1():
    # d = f = 1: each expert is y = gelu(x wg) (x wu) wd, by hand with math.tanh.
    rng = np.random.default_rng(4)
    x = rng.standard_normal((6, 1))
    wr = rng.standard_normal((1, 8))
    wg, wu, wd = (rng.standard_normal((8, 1, 1)) for _ in range(3))
    res = oracle.forward_sparse(x, wr, (wg, wu, wd))
    for t in range(6):
        l = [float(np.float32(x[t, 0] * wr[0, e])) for e in range(8)]
        m = max(l)
        z = sum(math.exp(v - m) for v in l)
        order = sorted(range(8), key=lambda e: (-l[e], e))[:2]
        acc = 0.0
        for e in order:
            a = x[t, 0] * wg[e, 0, 0]
            g = 0.5 * a * (1 + math.tanh(math.sqrt(2 / math.pi) * (a + 0.044715 * a ** 3)))
            acc += math.exp(l[e] - m) / z * g * (x[t, 0] * wu[e, 0, 0]) * wd[e, 0, 0]
        assert abs(res["out"][t, 0] - acc) < 1e-12


# ------------------------------------------------------------------ int8 --

def test_int8_unit_scales_equal_plain_weights():
    p = workloads.make_numpy_int8(T=8, d=32, f=48, seed=1)
    ones = (np.ones((8, 48)), np.ones((8, 48)), np.ones((8, 32)))
    a = oracle.forward_sparse(p["x"], p["w_router"], (p["w_gate"], p["w_up"], p["w_down"], ones))["out"]
    b = oracle.forward_sparse(p["x"], p["w_router"],
                              (p["w_gate"].astype(np.float64), p["w_up"].astype(np.float64),
                               p["w_down"].astype(np.float64)))["out"]
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=0)


def test_int8_scale_is_per_output_channel():
    p = workloads.make_numpy_int8(T=8, d=32, f=48, seed=2)
    s = (p["s_gate"].astype(np.float64), p["s_up"].astype(np.float64), p["s_down"].astype(np.float64))
    q = (p["w_gate"], p["w_up"], p["w_down"])
    base = oracle.forward_sparse(p["x"], p["w_router"], q + (s,), return_h=True)
    sd2 = s[2].copy()
    sd2[:, 5] *= 2
    r = oracle.forward_sparse(p["x"], p["w_router"], q + ((s[0], s[1], sd2),))["out"]
    np.testing.assert_allclose(r[:, 5], 2 * base["out"][:, 5], rtol=1e-13)
    np.testing.assert_allclose(np.delete(r, 5, 1), np.delete(base["out"], 5, 1), rtol=1e-14)
    su2 = s[1].copy()
    su2[:, 7] *= 2
    r = oracle.forward_sparse(p["x"], p["w_router"], q + ((s[0], su2, s[2]),), return_h=True)["h"]
    np.testing.assert_allclose(r[:, :, 7], 2 * base["h"][:, :, 7], rtol=1e-13)
    w = oracle.dequant_int8(p["w_down"][2], s[2][2])
    assert w[3, 4] == float(p["w_down"][2, 3, 4]) * s[2][2, 4]


def test_int8_sparse_equals_dense_bruteforce():
    p = workloads.make_numpy_int8(T=10, d=32, f=48, seed=3)
    ex = (p["w_gate"], p["w_up"], p["w_down"], (p["s_gate"], p["s_up"], p["s_down"]))
    np.testing.assert_allclose(oracle.forward_sparse(p["x"], p["w_router"], ex)["out"],
                               oracle.forward_dense_bruteforce(p["x"], p["w_router"], ex),
                               rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------- workloads --

def test_skew_bias_gives_the_stated_load_shares():
    rng = np.random.default_rng(0)
    d = 256
    x = rng.standard_normal((40000, d))
    wr = rng.standard_normal((d, 8)) / math.sqrt(d)
    r = oracle.route(x, wr, router_bias=np.array(workloads.SKEW_BIAS))
    share = np.bincount(r["idx"].reshape(-1), minlength=8) / r["idx"].size
    assert abs(share[0] - 0.50) < 0.01
    assert abs(share[1] - 0.15) < 0.02 and abs(share[2] - 0.15) < 0.02
    assert abs(share[3:].sum() - 0.20) < 0.02


def test_balanced_routing_is_near_uniform():
    p = workloads.make_numpy(T=4096, d=128, f=8, seed=0)
    r = oracle.route(p["x"], p["w_router"])
    share = np.bincount(r["idx"].reshape(-1), minlength=8) / r["idx"].size
    assert np.all(np.abs(share - 0.125) < 0.03)


def test_bf16_rounding_helper():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.14159], dtype=np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert (workloads.round_bf16_np(v) == ref).all()


# ------------------------------------------- next rows: Mixtral, post-norm --

def test_renormalized_routing_closed_form_and_softmax_of_selected_logits():
    g = _load("routing_closed_form.json")["renormalized_case"]
    x = np.zeros((1, 8))
    x[0, 0] = 1.0
    wr = np.zeros((8, 8))
    wr[0, :] = np.log(np.arange(1, 9, dtype=np.float64))
    r = oracle.route(x, wr, renormalize=True)
    assert list(r["idx"][0]) == g["idx"]
    np.testing.assert_allclose(r["gates"][0], np.array(g["gates_num"]) / g["gates_den"], rtol=1e-6)
    rng = np.random.default_rng(21)
    xs = rng.standard_normal((100, 16))
    wrs = rng.standard_normal((16, 8)) / 4
    rr = oracle.route(xs, wrs, renormalize=True)
    base = oracle.route(xs, wrs)
    assert (rr["idx"] == base["idx"]).all()
    sel = np.take_along_axis(rr["logits32"].astype(np.float64), rr["idx"].astype(np.int64), axis=1)
    np.testing.assert_allclose(rr["gates"], scipy.special.softmax(sel, axis=1), rtol=1e-12)
    np.testing.assert_allclose(rr["gates"].sum(1), 1.0, rtol=1e-14)


def test_silu_matches_library_and_mixtral_expert():
    z = np.linspace(-30, 30, 3001)
    ref = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    np.testing.assert_allclose(oracle.silu(z), ref, rtol=1e-13, atol=1e-15)
    x, wr, wg, wu, wd = _rand_problem(T=6, d=16, f=24)
    y, _ = oracle.expert_ffn(x, wg[1], wu[1], wd[1], "silu")
    xt = torch.from_numpy(x)
    lib = ((torch.nn.functional.silu(xt @ torch.from_numpy(wg[1])) * (xt @ torch.from_numpy(wu[1])))
           @ torch.from_numpy(wd[1])).numpy()
    np.testing.assert_allclose(y, lib, rtol=1e-12, atol=1e-14)
    dense = oracle.forward_dense_bruteforce(x, wr, (wg, wu, wd), gelu_mode="silu", renormalize=True)
    sparse = oracle.forward_sparse(x, wr, (wg, wu, wd), gelu_mode="silu", renormalize=True)["out"]
    np.testing.assert_allclose(sparse, dense, rtol=1e-12, atol=1e-14)


def test_post_norm_matches_library_rms_norm():
    rng = np.random.default_rng(22)
    y = rng.standard_normal((7, 64)) * 0.3
    w = rng.uniform(0.5, 1.5, 64)
    res = rng.standard_normal((7, 64))
    for eps in (1e-5, 1e-2):
        lib = torch.nn.functional.rms_norm(torch.from_numpy(y), (64,), torch.from_numpy(w), eps=eps).numpy()
        np.testing.assert_allclose(oracle.post_norm_residual(y, None, w, eps), lib, rtol=1e-12)
        np.testing.assert_allclose(oracle.post_norm_residual(y, res, w, eps), res + lib, rtol=1e-12)
    np.testing.assert_allclose(oracle.post_norm_residual(y, res), res + y, rtol=1e-15)
    # A constant row c normalises to w * sign(c) / sqrt(1 + eps / c^2).
    c = np.full((1, 64), -0.5)
    out = oracle.post_norm_residual(c, None, w, 1e-5)
    np.testing.assert_allclose(out[0], -w / np.sqrt(1 + 1e-5 / 0.25), rtol=1e-14)
