"""GPU parity: the CUDA path, called through the C ABI, against the oracle.

Routing indices, counts, offsets and the dispatch permutation must match
bit for bit (tokens within 1e-6 of a probability tie may take any ordering the
oracle lists as valid); gates within 2e-6; outputs and the GeGLU intermediate
within |gpu - ref| <= 1e-2 + 2e-2 |ref|."""

import numpy as np
import pytest
import torch

import mixture_experts_ffn_14_b200 as moe
from mixture_experts_ffn_14_b200 import workloads as W

from _harness import full_check, np64, run_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def small_bf16(T, d=512, f=384, seed=5, int8=False, skew=False):
    w = W.Workload("small", T, d, f, dtype="bf16_int8w" if int8 else "bf16", seed=seed, skew=skew)
    return W.make_torch(w, DEV)


def tiny_f32(seed=0, T=64, d=128, f=256):
    p = W.make_numpy(T, d, f, seed=seed)
    return {k: torch.from_numpy(v).to(DEV) for k, v in p.items()}


# ------------------------------------------------------------------ fp32 --

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_f32_full_parity(seed):
    inp = tiny_f32(seed)
    gpu = run_gpu(inp)
    full_check(inp, gpu)


@pytest.mark.parametrize("T", [1, 3, 33, 200])
def test_f32_ragged_token_counts(T):
    inp = tiny_f32(seed=T, T=T, d=128, f=192)
    full_check(inp, run_gpu(inp))


def test_f32_erf_gelu():
    inp = tiny_f32(seed=9)
    full_check(inp, run_gpu(inp, activation=moe.MOE_ACT_GELU_ERF), gelu_mode="erf")


# ------------------------------------------------------------------ bf16 --

PATHS = [moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE, moe.MOE_PATH_WEIGHT_STREAM]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 37, 300, 1000])
def test_bf16_parity_all_paths(T, path):
    inp = small_bf16(T)
    full_check(inp, run_gpu(inp, path=path))


@pytest.mark.parametrize("T", [128, 129, 200, 256, 257])
def test_bf16_automatic_form_boundary(T):
    # The automatic path runs bf16 weights in the weight-stream form up to 128
    # tokens and in token tiles above (both 128-row forms launched, one chosen
    # on the device; 256-row gate/up tiles from 512).
    inp = small_bf16(T, seed=70 + T)
    full_check(inp, run_gpu(inp, path=moe.MOE_PATH_AUTO))


# Row gather (moe_options_t.row_gather): token tiles read the gate/up operand
# rows from x with TMA four-row gathers instead of the dispatch stage's copy.
TT_PATHS = [moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE, moe.MOE_PATH_AUTO]


@pytest.mark.parametrize("path", TT_PATHS)
@pytest.mark.parametrize("T", [1, 37, 129, 257, 1000])
def test_row_gather_parity(T, path):
    inp = small_bf16(T, seed=31)
    full_check(inp, run_gpu(inp, path=path, row_gather=True))


@pytest.mark.parametrize("path", TT_PATHS)
def test_row_gather_from_an_offset_view_of_x(path):
    # x is a 16-byte aligned view three rows into a larger buffer whose other
    # rows hold 1000.0: reading any row outside the view would show in the output.
    inp = small_bf16(300, seed=21)
    T, d = inp["x"].shape
    big = torch.full((T + 7, d), 1000.0, dtype=inp["x"].dtype, device=DEV)
    big[3:3 + T] = inp["x"]
    view = big[3:3 + T]
    assert view.is_contiguous() and view.data_ptr() % 16 == 0
    inp2 = dict(inp, x=view)
    full_check(inp2, run_gpu(inp2, path=path, row_gather=True))


def test_row_gather_is_refused_for_int8_weights():
    # The int8-weight GEMMs run on fp16 operands from the dispatch copy.
    inp = small_bf16(5, seed=33, int8=True)
    T, d = inp["x"].shape
    E, _, f = inp["w_gate"].shape
    ws = torch.empty(moe.moe_workspace_size(T, d, f, E, 2, moe.MOE_BF16_INT8W), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(inp["x"])
    st = moe.moe_forward_ex(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out, ws,
                            scales=(inp["s_gate"], inp["s_up"], inp["s_down"]), row_gather=True,
                            raise_on_error=False)
    assert st == 2  # MOE_ERR_UNSUPPORTED


def test_row_gather_matches_copy_bitwise():
    # Same rows, same MMA order: the two ways of feeding A give identical bits.
    inp = small_bf16(700, seed=35)
    a = run_gpu(inp, path=moe.MOE_PATH_AUTO)
    b = run_gpu(inp, path=moe.MOE_PATH_AUTO, row_gather=True)
    assert np.array_equal(a["out"], b["out"])
    assert torch.equal(a["h"], b["h"])


def test_row_gather_skewed_with_empty_experts():
    inp = small_bf16(400, seed=37, skew=True)
    full_check(inp, run_gpu(inp, row_gather=True))


@pytest.mark.parametrize("T", [32768, 32800, 40000])
def test_dispatch_scan_threshold(T):
    # Up to 1024 router blocks (T = 32768) each dispatch CTA sums the block
    # histograms itself; above, a one-CTA scan computes the block offsets first.
    # Full dispatch against the oracle on both sides of the threshold; outputs on
    # a sample of tokens (first and last included).
    inp = small_bf16(T, d=256, f=128, seed=41)
    rng = np.random.default_rng(T)
    tok = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 64, replace=False)]))
    full_check(inp, run_gpu(inp, want_h=False), tokens=tok, check_h=False)


@pytest.mark.parametrize("splits", [1, 2, 3])
def test_bf16_weight_stream_split_k(splits):
    inp = small_bf16(90, d=256, f=384)
    full_check(inp, run_gpu(inp, path=moe.MOE_PATH_WEIGHT_STREAM, down_splits=splits))


@pytest.mark.parametrize("path", [moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE])
@pytest.mark.parametrize("splits", [2, 3])
def test_token_tile_split_k(path, splits):
    for int8 in (False, True):
        inp = small_bf16(400, d=512, f=384, seed=16, int8=int8)
        full_check(inp, run_gpu(inp, path=path, down_splits=splits))


@pytest.mark.parametrize("path", [moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE])
def test_bf16_long_k_pipeline_wrap(path):
    # K = 2048 (32 stages of 64) wraps the 4- and 6-deep rings many times; 3 n-tiles.
    inp = small_bf16(260, d=2048, f=384, seed=11)
    full_check(inp, run_gpu(inp, path=path))


@pytest.mark.parametrize("T", [1, 100, 129, 130, 255, 256, 257])
def test_bf16_pair_tile_boundaries(T):
    # Every token picks experts 0 and 1, so both hold T rows: the last 256-row
    # pair tile leaves 0..128 valid rows to the second CTA of the pair.
    inp = small_bf16(T, seed=15)
    inp["router_bias"] = torch.tensor([40.0, 30.0, 0, 0, 0, 0, 0, 0], device=DEV)
    for path in (moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE):
        gpu = run_gpu(inp, path=path)
        assert list(gpu["counts"][:2]) == [T, T]
        full_check(inp, gpu)


def test_bf16_skewed_with_empty_experts():
    inp = small_bf16(700, seed=12)
    # Router bias that sends every token to experts 0 and 1: six experts empty,
    # two experts with 700 rows each (6 m-tiles, ragged tail).
    inp["router_bias"] = torch.tensor([40.0, 30.0, 0, 0, 0, 0, 0, 0], device=DEV)
    gpu = run_gpu(inp, path=moe.MOE_PATH_TOKEN_TILE)
    assert list(gpu["counts"]) == [700, 700, 0, 0, 0, 0, 0, 0]
    full_check(inp, gpu)


def test_bf16_skew_bias_workload_small():
    inp = small_bf16(2048, d=256, f=256, seed=13, skew=True)
    gpu = run_gpu(inp)
    share = gpu["counts"] / gpu["counts"].sum()
    assert share[0] > 0.45
    full_check(inp, gpu, tokens=np.arange(0, 2048, 7))


def test_bf16_erf_gelu():
    inp = small_bf16(130, seed=14)
    full_check(inp, run_gpu(inp, activation=moe.MOE_ACT_GELU_ERF), gelu_mode="erf")


# ------------------------------------------------------------------ int8 --

@pytest.mark.parametrize("path", PATHS + [moe.MOE_PATH_AUTO])
@pytest.mark.parametrize("T", [5, 300])
def test_int8_parity_all_paths(T, path):
    inp = small_bf16(T, seed=21, int8=True)
    full_check(inp, run_gpu(inp, path=path))


def test_int8_power_of_two_scales_match_bf16_path():
    # With every scale 2^-7, q * 2^-7 is exact in bf16 and scaling by a power of
    # two commutes with fp32 rounding, so the int8 path (fp16 operands, scale in
    # the epilogue) and the bf16 path (weights q * 2^-7) form the same fp32
    # values; only H's final rounding differs (fp16 there, bf16 here).
    inp = small_bf16(150, seed=22, int8=True)
    for s in ("s_gate", "s_up", "s_down"):
        inp[s] = torch.full_like(inp[s], 2.0 ** -7)
    a = run_gpu(inp, path=moe.MOE_PATH_TOKEN_TILE)
    b_inp = dict(inp)
    for w in ("w_gate", "w_up", "w_down"):
        b_inp[w] = (inp[w].float() * 2.0 ** -7).to(torch.bfloat16)
    for s in ("s_gate", "s_up", "s_down"):
        del b_inp[s]
    b = run_gpu(b_inp, path=moe.MOE_PATH_TOKEN_TILE)
    assert a["h"].dtype == torch.float16 and b["h"].dtype == torch.bfloat16
    ha, hb = a["h"].float(), b["h"].float()
    assert bool(((ha - hb).abs() <= (2.0 ** -8 + 2.0 ** -10) * hb.abs() + 1e-6).all())
    # out sums f = 384 products of H with weights: independent H roundings of up
    # to 2^-9 relative move it by ~sqrt(f) * 2^-9 of a typical term (about 1 % of
    # its rms here, several times that in the tails), plus one bf16 ulp.
    rms = float(np.sqrt(np.mean(b["out"] ** 2)))
    diff = np.abs(a["out"] - b["out"])
    assert np.all(diff <= 5e-2 * rms + 2.0 ** -7 * np.abs(b["out"])), (diff.max(), rms)


@pytest.mark.parametrize("path", [moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE,
                                  moe.MOE_PATH_WEIGHT_STREAM])
def test_int8_every_code_converts_exactly(path):
    # W_up holds all 256 int8 codes, W_gate is 16 everywhere, x rows are one-hot
    # and the router ties (experts 0 and 1 for every token). Then the gate branch
    # is GELU(16) = 16 * (1 + erf(11.3)) / 2 = 16 exactly in fp32 (erf rounds to 1)
    # and H[row, n] = 16 * q_up[token, n]: an integer below 2048, exact in fp16.
    # Any code converted wrongly shows bitwise.
    T, d, f = 8, 256, 128
    codes = ((torch.arange(d * f).reshape(d, f) % 256) - 128).to(torch.int8)
    inp = {
        "x": torch.eye(T, d, dtype=torch.bfloat16, device=DEV),
        "w_router": torch.zeros((d, 8), dtype=torch.float32, device=DEV),
        "w_gate": torch.full((8, d, f), 16, dtype=torch.int8, device=DEV),
        "w_up": codes.to(DEV).expand(8, d, f).contiguous(),
        "w_down": torch.zeros((8, f, d), dtype=torch.int8, device=DEV),
        "s_gate": torch.ones((8, f), dtype=torch.bfloat16, device=DEV),
        "s_up": torch.ones((8, f), dtype=torch.bfloat16, device=DEV),
        "s_down": torch.ones((8, d), dtype=torch.bfloat16, device=DEV),
    }
    g = run_gpu(inp, path=path, activation=moe.MOE_ACT_GELU_ERF)
    assert (g["idx"] == np.array([0, 1])).all()
    tok = torch.as_tensor(g["perm_token"], device=DEV).long()
    want = 16.0 * codes.to(DEV).float()[tok]          # [2T, f]
    assert torch.equal(g["h"].float(), want)
    assert int(codes.min()) == -128 and int(codes.max()) == 127


# ------------------------------------------------------- determinism etc --

@pytest.mark.parametrize("T", [512, 1100, 2100])
def test_tall_bf16_gateup_tiles(T):
    # From 512 tokens the automatic path runs the bf16 gate/up GEMM in 256-row
    # tiles (two M = 128 MMAs per weight tile). Experts of 1-255 rows beyond
    # a multiple of 256 end in a partial tile: one MMA per step when it has at
    # most 128 rows. Each element of H accumulates the same 16-deep K steps in
    # the same order as in 128-row tiles, so H must equal the single-CTA
    # 128-row form bit for bit; H and out must match the oracle.
    inp = small_bf16(T, d=512, f=1024, seed=T)
    a = run_gpu(inp, path=moe.MOE_PATH_AUTO)
    b = run_gpu(inp, path=moe.MOE_PATH_TOKEN_TILE_SINGLE)
    assert torch.equal(a["h"], b["h"])
    full_check(inp, a, tokens=np.arange(0, T, 7))


def test_bitwise_determinism_and_streams():
    inp = small_bf16(333, seed=31)
    a = run_gpu(inp)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b = run_gpu(inp, stream=s)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["perm_token"], b["perm_token"])


@pytest.mark.parametrize("T,path,int8,splits,residual,skew", [
    (64, moe.MOE_PATH_AUTO, False, 0, False, False),           # weight-stream, split-K
    (100, moe.MOE_PATH_WEIGHT_STREAM, True, 3, True, False),
    (200, moe.MOE_PATH_WEIGHT_STREAM, False, 1, True, True),
    (300, moe.MOE_PATH_TOKEN_TILE, False, 1, False, False),
    (300, moe.MOE_PATH_TOKEN_TILE_SINGLE, False, 3, True, False),
    (1000, moe.MOE_PATH_AUTO, False, 0, False, False),
    (700, moe.MOE_PATH_AUTO, False, 2, True, True),
    (600, moe.MOE_PATH_AUTO, True, 2, True, False),
    (517, moe.MOE_PATH_TOKEN_TILE_SINGLE, True, 1, False, True),
])
def test_fused_combine_matches_combine_kernel_bitwise(T, path, int8, splits, residual, skew):
    # The down projection's epilogue sums each token's rows (whichever tile
    # finishes last, in a fixed order; token tiles and weight-stream tiles);
    # the separate combine kernel sums the same pieces in the same order:
    # outputs equal bit for bit, also with split-K pieces, the residual add,
    # int8 tiles and skewed loads.
    inp = small_bf16(T, seed=110 + T, int8=int8, skew=skew)
    kw = {}
    if residual:
        g = torch.Generator(device=DEV)
        g.manual_seed(T)
        kw["residual"] = torch.randn(inp["x"].shape, generator=g, device=DEV).to(torch.bfloat16)
    a = run_gpu(inp, path=path, down_splits=splits, want_h=False, **kw)
    b = run_gpu(inp, path=path, down_splits=splits, want_h=False, separate_combine=True, **kw)
    assert np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["out"], b["out"])
    okw = {"residual": kw["residual"]} if residual else {}
    full_check(inp, a, check_h=False, **okw)


def test_moe_forward_library_workspace_matches_ex():
    inp = small_bf16(257, seed=32)
    out = torch.empty_like(inp["x"])
    moe.moe_forward(inp["x"], inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out)
    torch.cuda.synchronize()
    ref = run_gpu(inp, want_h=False)
    assert np.array_equal(np64(out), ref["out"])
    assert moe.moe_device_status() == (0, 0)


def test_zero_tokens_is_a_noop():
    inp = small_bf16(4, seed=33)
    x0 = inp["x"][:0]
    out = torch.empty((0, inp["x"].shape[1]), dtype=torch.bfloat16, device=DEV)
    moe.moe_forward(x0, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out)


# ------------------------------------------- next rows: Mixtral, post-norm --

VARIANTS = [
    dict(renormalize=True),
    dict(activation=moe.MOE_ACT_SILU),
    dict(renormalize=True, activation=moe.MOE_ACT_SILU),
    dict(post_norm=True),
    dict(residual=True),
    dict(post_norm=True, residual=True, renormalize=True),
]


def _variant_args(inp, v, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    T, d = inp["x"].shape
    kw = {k: v[k] for k in ("renormalize", "activation") if k in v}
    if v.get("residual"):
        kw["residual"] = torch.randn((T, d), generator=g, device=DEV).to(inp["x"].dtype)
    if v.get("post_norm"):
        kw["post_norm_weight"] = (0.5 + torch.rand(d, generator=g, device=DEV)).float()
        kw["norm_eps"] = 1e-5
    return kw


def _oracle_kw(kw):
    okw = {k: kw[k] for k in ("renormalize", "residual", "post_norm_weight", "norm_eps") if k in kw}
    if kw.get("activation") == moe.MOE_ACT_SILU:
        okw["gelu_mode"] = "silu"
    return okw


@pytest.mark.parametrize("vi", range(len(VARIANTS)))
def test_variants_f32(vi):
    inp = tiny_f32(seed=40 + vi)
    kw = _variant_args(inp, VARIANTS[vi], vi)
    full_check(inp, run_gpu(inp, **kw), **_oracle_kw(kw))


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("vi", range(len(VARIANTS)))
def test_variants_bf16(vi, path):
    inp = small_bf16(300, seed=50 + vi)
    kw = _variant_args(inp, VARIANTS[vi], vi)
    full_check(inp, run_gpu(inp, path=path, **kw), **_oracle_kw(kw))


@pytest.mark.parametrize("vi", [2, 5])
def test_variants_int8(vi):
    inp = small_bf16(200, seed=60 + vi, int8=True)
    kw = _variant_args(inp, VARIANTS[vi], vi)
    full_check(inp, run_gpu(inp, **kw), **_oracle_kw(kw))


def test_renormalized_gates_sum_to_one():
    inp = small_bf16(64, seed=70)
    gpu = run_gpu(inp, renormalize=True, want_h=False)
    assert np.abs(gpu["gates"].sum(1) - 1.0).max() < 1e-6


@pytest.mark.parametrize("T", [1, 129, 256, 257, 300, 384, 385])
def test_int8_tile_boundaries(T):
    # Every token picks experts 0 and 1 (T rows each): full and ragged 128-row
    # tiles on the automatic path (weight-stream at T <= 256, token tiles above)
    # and on forced single-CTA token tiles.
    inp = small_bf16(T, seed=90, int8=True)
    inp["router_bias"] = torch.tensor([40.0, 30.0, 0, 0, 0, 0, 0, 0], device=DEV)
    for path in (moe.MOE_PATH_AUTO, moe.MOE_PATH_TOKEN_TILE_SINGLE):
        gpu = run_gpu(inp, path=path)
        assert list(gpu["counts"][:2]) == [T, T]
        full_check(inp, gpu)


@pytest.mark.parametrize("int8", [False, True])
@pytest.mark.parametrize("T", [64, 65, 100, 128])
def test_weight_stream_short_tiles_split_an_expert(T, int8):
    # Batches of at most 128 tokens take weight-stream tiles of at most 64
    # tokens; with every token on experts 0 and 1 those experts need one or two
    # tiles each (64 = one full tile, 65 = a full one and a single-token one).
    inp = small_bf16(T, seed=130 + T, int8=int8)
    inp["router_bias"] = torch.tensor([40.0, 30.0, 0, 0, 0, 0, 0, 0], device=DEV)
    gpu = run_gpu(inp)
    assert list(gpu["counts"][:2]) == [T, T]
    full_check(inp, gpu)


@pytest.mark.parametrize("T,skew", [(516, False), (1028, False), (700, True)])
def test_int8_tall_tiles_both_halves(T, skew):
    # int8 token tiles hold 256 rows as two MMAs on one converted weight tile;
    # the second (rows 128..255) runs only when the tile has more than 128 rows.
    # About 130 and 257 rows per expert, and a skewed load (one expert near half
    # of all slots), put tiles on both sides of 128 and 256.
    inp = small_bf16(T, seed=95 + T, int8=True, skew=skew)
    g = run_gpu(inp)
    counts = g["counts"]
    assert (counts % 256 > 128).any() or (counts > 256).any()
    full_check(inp, g)


@pytest.mark.parametrize("path", [moe.MOE_PATH_TOKEN_TILE, moe.MOE_PATH_TOKEN_TILE_SINGLE])
def test_grouped_tile_order_for_large_experts(path):
    # An expert whose intermediate rows exceed the L2 budget (here 2000 rows x
    # f = 32768 for the down projection: 8 pair or 16 single-CTA row tiles of
    # 16 / 8 MB) has its row tiles taken in groups; every token still routes to
    # experts 0 and 1, and the outputs match the oracle.
    w = W.Workload("grouped", 2000, 256, 32768, dtype="bf16", seed=140)
    inp = W.make_torch(w, DEV)
    inp["router_bias"] = torch.tensor([40.0, 30.0, 0, 0, 0, 0, 0, 0], device=DEV)
    gpu = run_gpu(inp, path=path, down_splits=1, want_h=False)
    assert list(gpu["counts"][:2]) == [2000, 2000]
    rng = np.random.default_rng(7)
    full_check(inp, gpu, tokens=np.sort(rng.choice(2000, size=48, replace=False)), check_h=False)


def _status_after(inp, x, path=moe.MOE_PATH_AUTO):
    T, d = x.shape
    f = inp["w_gate"].shape[2]
    ws = torch.empty(moe.moe_workspace_size(T, d, f, dtype=moe.MOE_BF16_INT8W, path=path), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty_like(x)
    moe.moe_forward_ex(x, inp["w_router"], inp["w_gate"], inp["w_up"], inp["w_down"], out, ws,
                       scales=(inp["s_gate"], inp["s_up"], inp["s_down"]), path=path)
    return moe.moe_device_status(ws)


@pytest.mark.parametrize("path", [moe.MOE_PATH_WEIGHT_STREAM, moe.MOE_PATH_TOKEN_TILE_SINGLE])
def test_int8_fp16_range_is_reported(path):
    # The int8-weight GEMMs take fp16 operands: a bf16 activation above 65504
    # in magnitude, or a GeGLU intermediate that large, cannot be represented.
    # The library flags it (status bit 0x20) instead of returning a silently
    # wrong output. An ordinary finite input triggers it; nothing faults.
    inp = small_bf16(300, seed=120, int8=True)
    assert _status_after(inp, inp["x"], path) == (0, 0)
    x = inp["x"].clone()
    x[150, 7] = 1e5                                   # finite in bf16, not in fp16
    st, code = _status_after(inp, x, path)
    assert st == moe.N.MOE_ERR_DEVICE_CHECK and code == 0x20
    # H overflow with in-range activations: unit scales and every code 127 make
    # x . w_gate about 127 * sqrt(d) * 4, so GELU(gate) * up is far above 65504.
    big = dict(inp)
    for w in ("w_gate", "w_up"):
        big[w] = torch.full_like(inp[w], 127)
    for s_ in ("s_gate", "s_up"):
        big[s_] = torch.ones_like(inp[s_])
    xs = torch.full_like(inp["x"], 4.0)
    st, code = _status_after(big, xs, path)
    assert st == moe.N.MOE_ERR_DEVICE_CHECK and code == 0x20
    assert _status_after(inp, inp["x"], path) == (0, 0)  # the next call starts clean


@pytest.mark.parametrize("splits", [2, 3])
def test_int8_token_tile_split_k(splits):
    inp = small_bf16(600, d=512, f=384, seed=91, int8=True)
    full_check(inp, run_gpu(inp, down_splits=splits))
