"""GPU parity: every kernel of the layer, called through the C ABI, against the CPU oracle.

Routing, capacity and the permutation are compared bit for bit; gates at 1e-5 relative;
expert outputs and the layer output at max|err| <= 2e-2 max|ref| for bf16 GEMMs (1e-4
absolute for the fp32 toy layer).  Sizes span several tiles with ragged tails.
"""
import time
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import (assert_close_layer, assert_route_equal, check_status, dev, err_stats,
                      explain_routing_differences, f64, forward_launches, fragile_tokens,
                      gpu_route, host)
from golden.reader import load
from mixture_experts_layer_50_b200 import _native as nat
from mixture_experts_layer_50_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _needs_cuda(cuda_dev):
    yield


# ---------------------------------------------------------------------------------------
# routing + capacity (moe_route with given fp32 logits): bit-exact
# ---------------------------------------------------------------------------------------
def test_route_capacity_trace_of_the_slides():
    g = load("p2_capacity_trace.txt")
    assign = [tuple(int(v) for v in p.split()) for p in g["assign"].split("|")]
    z = np.full((8, 4), 0.2, np.float32)
    for t, (a, b) in enumerate(assign):
        z[t, a], z[t, b] = 2.1, 1.8
    for cf, tag in ((Fraction(5, 4), "1.25"), (1, "1.0"), (2, "2.0")):
        C = O.capacity(8, 2, 4, cf)
        cfg = nat.make_config(8, 64, 4, 2, 64, capacity=C)
        got = gpu_route(cfg, z)
        assert_route_equal(got, z, 2, O.SOFTMAX, 1, None, None, 4, C)
        assert int(got["drop_mask"].sum()) == int(g.get(f"drops_{tag}", 1))
    got = gpu_route(nat.make_config(8, 64, 4, 2, 64, capacity=5), z)
    assert got["demand"].tolist() == [6, 4, 3, 3]
    t6 = 5
    assert got["drop_mask"][t6].tolist() == [1, 0]
    assert round(float(got["gates"][t6, 1]), 3) == 0.426


ROUTE_CASES = [
    # N, E, k, score_fn, renorm, n_bias_sets, capacity, quantum(ties)
    (1, 4, 2, 0, 1, 0, 0, 0.0),
    (7, 8, 2, 0, 1, 0, 0, 0.0),
    (129, 64, 6, 1, 1, 1, 0, 0.0),
    (1000, 8, 2, 0, 1, 0, 0, 0.0),
    (1000, 8, 1, 0, 0, 0, 0, 0.0),           # Switch: raw p
    (777, 384, 6, 1, 1, 2, 0, 0.0),          # per-modality bias sets
    (513, 256, 8, 1, 1, 1, 20, 0.0),         # capacity with sigmoid
    (300, 16, 4, 0, 1, 0, 0, 0.25),          # many exact ties
    (300, 16, 4, 1, 1, 0, 0, 0.25),
    (257, 33, 32, 0, 1, 0, 0, 0.0),          # k = 32, E not a multiple of 32
    (200, 1024, 8, 1, 1, 1, 0, 0.0),         # largest E
    (128, 5, 5, 0, 1, 0, 0, 0.0),            # k = E
    (1000, 4, 2, 0, 1, 0, 1, 0.0),           # capacity 1: one kept slot per expert
]


@pytest.mark.parametrize("N,E,k,sf,rn,nb,C,q", ROUTE_CASES)
def test_route_bit_exact(N, E, k, sf, rn, nb, C, q):
    seed = N * 7 + E
    z = W.random_logits(N, E, seed, scale=2.0, quantum=q)
    bias = W.random_bias(nb, E, seed + 1) if nb else None
    mod = W.random_modality(N, seed + 2) if nb > 1 else None
    cfg = nat.make_config(N, 64, E, k, 64, n_bias_sets=nb, score_fn=sf, renorm=rn, capacity=C)
    got = gpu_route(cfg, z, bias, mod)
    assert_route_equal(got, z, k, sf, rn, bias, mod, E, C)


def test_route_all_tokens_one_expert_and_capacity():
    N, E = 1000, 16
    z = W.random_logits(N, E, 3)
    z[:, 5] += 100.0
    C = O.capacity(N, 2, E, 1)
    got = gpu_route(nat.make_config(N, 64, E, 2, 64, capacity=C), z)
    assert_route_equal(got, z, 2, O.SOFTMAX, 1, None, None, E, C)
    assert got["counts"][5] == C and got["demand"][5] == N


def test_route_full_size_v41flash_and_zipf_capacity():
    # DeepSeek-V4.1-Flash routing shape: 16384 tokens, 384 experts, top-6, two bias sets
    N, E, k = 16384, 384, 6
    z = W.random_logits(N, E, 11, scale=1.4)
    bias = W.random_bias(2, E, 12)
    mod = W.random_modality(N, 13)
    got = gpu_route(nat.make_config(N, 64, E, k, 64, n_bias_sets=2, score_fn=1), z, bias, mod)
    assert_route_equal(got, z, k, O.SIGMOID, 1, bias, mod, E, 0)
    # skewed capacity workload: Zipf offsets on the logits, cf = 1 and 1.25, top-2 and k=1
    E = 64
    z = (W.random_logits(N, E, 14, scale=0.9) + W.zipf_logit_offsets(E)[None, :]).astype(np.float32)
    for k, rn, cf in ((2, 1, 1), (2, 1, Fraction(5, 4)), (1, 0, 1)):
        C = O.capacity(N, k, E, cf)
        got = gpu_route(nat.make_config(N, 64, E, k, 64, renorm=rn, capacity=C), z)
        _, _, d = assert_route_equal(got, z, k, O.SOFTMAX, rn, None, None, E, C)
        assert int(got["drop_mask"].sum()) > 0


@pytest.mark.parametrize("N,d,E", [(16, 256, 8), (300, 512, 160), (1000, 256, 384),
                                   (8192, 512, 256), (777, 136, 1024), (4096, 256, 8),
                                   (122, 272, 17), (300, 64, 5), (64, 128, 33)])
def test_router_gemm_logits(N, d, E):
    """z = x . W_g on the tensor cores (tile widths 32 to 256, split K for few tiles, E not a
    multiple of 4 so that logit rows are not 16-byte aligned) against float64, element by
    element, within an fp32 accumulation bound."""
    g = torch.Generator().manual_seed(N + E)
    x = torch.randn(N, d, generator=g).to(torch.bfloat16)
    W_g = (0.05 * torch.randn(E, d, generator=g)).to(torch.bfloat16)
    cfg = nat.make_config(N, d, E, 2, 64)
    ws = nat.alloc_workspace(cfg)
    z = torch.empty((N, E), dtype=torch.float32, device="cuda")
    out = dict(ids=torch.empty((N, 2), dtype=torch.int32, device="cuda"),
               gates=torch.empty((N, 2), dtype=torch.float32, device="cuda"),
               counts=torch.empty(E, dtype=torch.int32, device="cuda"),
               demand=torch.empty(E, dtype=torch.int32, device="cuda"),
               drop_mask=torch.empty((N, 2), dtype=torch.uint8, device="cuda"))
    nat.moe_route(cfg, x=x.cuda(), W_g=W_g.cuda(), logits_out=z, ws=ws, **out)
    check_status(ws)
    x64, w64 = f64(x), f64(W_g)
    z_o = O.router_logits(x64, w64)
    bound = 1e-4 * (np.abs(x64) @ np.abs(w64).T) + 1e-30
    err = np.abs(host(z).astype(np.float64) - z_o)
    assert (err <= bound).all(), float((err / bound).max())
    # the routing of those logits, bit for bit
    assert_route_equal({k_: host(v) for k_, v in out.items()}, host(z), 2, O.SOFTMAX, 1, None,
                       None, E, 0)


def test_route_reports_bad_modality_flag():
    N, E = 64, 8
    z = W.random_logits(N, E, 5)
    bias = W.random_bias(2, E, 6)
    mod = np.zeros(N, np.uint8)
    mod[7] = 9  # no such bias set: the kernel falls back to set 0 and reports it
    cfg = nat.make_config(N, 64, E, 2, 64, n_bias_sets=2, score_fn=1)
    ws = nat.alloc_workspace(cfg)
    ids = torch.empty((N, 2), dtype=torch.int32, device="cuda")
    gates = torch.empty((N, 2), dtype=torch.float32, device="cuda")
    nat.moe_route(cfg, logits=dev(z), bias=dev(bias), modality=dev(mod), ids=ids, gates=gates,
                  ws=ws)
    assert nat.moe_check_status(ws) == nat.MOE_ERR_INVALID_INPUT
    assert nat.moe_check_status(ws) == 0   # cleared by the read


# ---------------------------------------------------------------------------------------
# permutation (moe_permute): bit-exact
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("N,E,k,C,dt", [(300, 8, 2, 0, torch.bfloat16), (1000, 64, 6, 70, torch.bfloat16),
                                       (129, 5, 3, 0, torch.float32), (1, 4, 2, 0, torch.bfloat16),
                                       # >= 64 tokens per SM with small rows: the
                                       # warp-per-token scatter
                                       (9472, 16, 2, 0, torch.bfloat16),
                                       (12345, 64, 4, 700, torch.bfloat16),
                                       (10001, 8, 3, 0, torch.float32)])
def test_permute_bit_exact(N, E, k, C, dt):
    d = 72 if dt == torch.bfloat16 else 68
    z = W.random_logits(N, E, N + E)
    ids_o, _ = O.route(z, k)
    dsp = O.dispatch(ids_o, E, C)
    x = torch.randn(N, d, generator=torch.Generator().manual_seed(1)).to(dt).cuda()
    cfg = nat.make_config(N, d, E, k, 64, dtype=nat.BF16 if dt == torch.bfloat16 else nat.F32)
    ws = nat.alloc_workspace(cfg)
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_token = torch.full((N * k,), -7, dtype=torch.int32, device="cuda")
    slot_row = torch.empty((N, k), dtype=torch.int32, device="cuda")
    xp = torch.zeros((N * k, d), dtype=dt, device="cuda")
    nat.moe_permute(cfg, ids=dev(ids_o), drop_mask=dev(dsp["drop_mask"]), x=x, offsets=offsets,
                    row_token=row_token, slot_row=slot_row, xp=xp, ws=ws)
    check_status(ws)
    M = int(dsp["offsets"][-1])
    np.testing.assert_array_equal(host(offsets), dsp["offsets"])
    np.testing.assert_array_equal(host(slot_row), dsp["slot_row"])
    np.testing.assert_array_equal(host(row_token)[:M], dsp["row_token"])
    assert (host(row_token)[M:] == -7).all()
    assert torch.equal(xp[:M].cpu(), x.cpu()[torch.from_numpy(dsp["row_token"]).long()])


def test_permute_reports_bad_ids_without_touching_memory():
    N, E, k = 64, 8, 2
    ids = np.tile(np.array([[1, 2]], np.int32), (N, 1))
    ids[3] = [9, 1]      # out of range
    ids[4] = [5, 5]      # repeated within a token
    cfg = nat.make_config(N, 64, E, k, 64)
    ws = nat.alloc_workspace(cfg)
    x = torch.randn(N, 64, device="cuda").to(torch.bfloat16)
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    slot_row = torch.empty((N, k), dtype=torch.int32, device="cuda")
    xp = torch.zeros((N * k, 64), dtype=torch.bfloat16, device="cuda")
    nat.moe_permute(cfg, ids=dev(ids), x=x, offsets=offsets, slot_row=slot_row, xp=xp, ws=ws)
    assert nat.moe_check_status(ws) == nat.MOE_ERR_INVALID_INPUT
    sr = host(slot_row)
    assert sr[3, 0] == -1 and sr[4, 1] == -1 and sr[4, 0] >= 0
    assert host(offsets)[-1] == 2 * N - 2


# ---------------------------------------------------------------------------------------
# expert FFN (moe_expert_ffn): tcgen05 grouped GEMMs vs float64
# ---------------------------------------------------------------------------------------
FFN_CASES = [
    # N, d, E, k, F, n_shared, act, clamp
    (300, 256, 5, 2, 384, 1, W.SWIGLU, 0.0),
    (700, 512, 8, 2, 256, 0, W.SWIGLU, 0.0),
    (200, 136, 6, 3, 200, 1, W.SWIGLU, 0.0),     # ragged K, ragged columns, partial tiles
    (64, 256, 16, 4, 128, 1, W.SWIGLU, 0.5),     # clamp active on many pre-activations
    (333, 192, 4, 2, 320, 0, W.RELU, 0.0),
    (1, 128, 4, 2, 128, 1, W.SWIGLU, 0.0),
]


@pytest.mark.parametrize("path", ["1sm", "1sm128", "2sm", "swap", "1sm64", "tall"])
@pytest.mark.parametrize("N,d,E,k,F,S,act,clamp", FFN_CASES)
def test_expert_ffn(N, d, E, k, F, S, act, clamp, path, monkeypatch):
    # every grouped-GEMM variant (1-SM 128x256 and 128x128 tiles, 2-SM 256x256, the
    # token-in-N kernel with weights in M, the 1-SM kernel forced to 64-row tiles, and its
    # 256-row tall tiles) on every case
    _set_path(path, monkeypatch)
    shape = W.LayerShape("t", N=N, d=d, E=E, k=k, F=F, n_shared=S, act=act, clamp=clamp,
                         w_std=0.08, seed=N + d)
    t = W.make_inputs(shape, device="cuda")
    z = W.random_logits(N, E, N)
    z[:, 0] += 1.0   # a hot expert with several M tiles
    ids_o, _ = O.route(z, k)
    dsp = O.dispatch(ids_o, E, 0)
    M = int(dsp["offsets"][-1])
    xp = torch.zeros((N * k, d), dtype=torch.bfloat16, device="cuda")
    xp[:M] = t["x"][torch.from_numpy(dsp["row_token"]).long().cuda()]
    ye = torch.zeros((N * k + S * N, d), dtype=torch.bfloat16, device="cuda")
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    nat.moe_expert_ffn(cfg, xp=xp, offsets=dev(dsp["offsets"]), x=t["x"], W_gu=t["W_gu"],
                       W_down=t["W_down"], ye=ye, ws=ws)
    check_status(ws)
    x64, Wgu, Wd = f64(t["x"]), f64(t["W_gu"]), f64(t["W_down"])
    ref = np.zeros((N * k + S * N, d))
    for e in range(E):
        a, b = dsp["offsets"][e], dsp["offsets"][e + 1]
        if b > a:
            ref[a:b] = O.expert_ffn(x64[dsp["row_token"][a:b]], Wgu[e], Wd[e], act, clamp)
    if S:
        ref[N * k:] = O.expert_ffn(x64, Wgu[E], Wd[E], act, clamp)
    got = host(ye)
    rows = np.r_[0:M, N * k:N * k + S * N]
    assert_close_layer(got[rows], ref[rows])


def _set_path(path, monkeypatch):
    """MOE_B200_GEMM_PATH for one kernel variant; "1sm64" is the 1-SM kernel forced to
    64-row tiles (MOE_B200_DECODE_A64=2), which the layer otherwise takes for small groups."""
    if path == "1sm64":
        monkeypatch.setenv("MOE_B200_GEMM_PATH", "1sm")
        monkeypatch.setenv("MOE_B200_DECODE_A64", "2")
    else:
        monkeypatch.setenv("MOE_B200_GEMM_PATH", path)
        monkeypatch.setenv("MOE_B200_DECODE_A64", "0")


@pytest.mark.parametrize("path", ["1sm", "swap", "2sm", "1sm64", "tall"])
def test_expert_ffn_group_sizes_around_the_tile_edges(path, monkeypatch):
    """Groups of 0 ... 513 rows around every tile edge: the token-in-N kernel rounds a group's
    last row block up to 16 rows and loads it in 32-row boxes; the 1-SM kernel pads to
    128-row tiles (M = 64 for a last tile of at most 64 rows), or cuts groups into 64-row
    tiles, or 256-row tall tiles whose second half is skipped or runs M = 64; the 2-SM kernel
    pads to 256-row tiles (128 with a half tile for the down projection)."""
    _set_path(path, monkeypatch)
    sizes = [0, 1, 15, 16, 17, 31, 32, 33, 127, 128, 129, 255, 256, 257, 300, 383, 384, 385,
             511, 512, 513]
    E, k, d, F = len(sizes), 1, 256, 384
    N = sum(sizes)
    shape = W.LayerShape("t", N=N, d=d, E=E, k=k, F=F, n_shared=1, act=W.SWIGLU, clamp=0.0,
                         w_std=0.08, seed=11)
    t = W.make_inputs(shape, device="cuda")
    ids = np.repeat(np.arange(E, dtype=np.int32), sizes)[np.random.default_rng(3).permutation(N)]
    dsp = O.dispatch(ids[:, None], E, 0)
    np.testing.assert_array_equal(dsp["counts"], sizes)
    xp = t["x"][torch.from_numpy(dsp["row_token"]).long().cuda()].contiguous()
    ye = torch.zeros((N * k + N, d), dtype=torch.bfloat16, device="cuda")
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    nat.moe_expert_ffn(cfg, xp=xp, offsets=dev(dsp["offsets"]), x=t["x"], W_gu=t["W_gu"],
                       W_down=t["W_down"], ye=ye, ws=ws)
    check_status(ws)
    x64, Wgu, Wd = f64(t["x"]), f64(t["W_gu"]), f64(t["W_down"])
    ref = np.zeros((2 * N, d))
    for e in range(E):
        a, b = dsp["offsets"][e], dsp["offsets"][e + 1]
        if b > a:
            ref[a:b] = O.expert_ffn(x64[dsp["row_token"][a:b]], Wgu[e], Wd[e], W.SWIGLU, 0.0)
    ref[N:] = O.expert_ffn(x64, Wgu[E], Wd[E], W.SWIGLU, 0.0)
    assert_close_layer(host(ye), ref)


# ---------------------------------------------------------------------------------------
# combine (moe_combine)
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("N,d,E,k,S,C,dt", [(500, 264, 8, 2, 1, 100, torch.bfloat16),
                                           (129, 64, 4, 3, 0, 0, torch.float32)])
def test_combine(N, d, E, k, S, C, dt):
    z = W.random_logits(N, E, 21)
    ids_o, gates_o = O.route(z, k)
    dsp = O.dispatch(ids_o, E, C)
    ye = torch.randn(N * k + S * N, d, generator=torch.Generator().manual_seed(2)).to(dt).cuda()
    y = torch.empty((N, d), dtype=dt, device="cuda")
    cfg = nat.make_config(N, d, E, k, 64, n_shared=S, dtype=nat.BF16 if dt == torch.bfloat16 else nat.F32)
    g32 = gates_o.astype(np.float32)
    nat.moe_combine(cfg, ye=ye, slot_row=dev(dsp["slot_row"]), gates=dev(g32), y=y)
    torch.cuda.synchronize()
    ye64 = f64(ye)
    ref = np.zeros((N, d))
    for t in range(N):
        for j in range(k):
            r = dsp["slot_row"][t, j]
            if r >= 0:
                ref[t] += float(g32[t, j]) * ye64[r]
        if S:
            ref[t] += ye64[N * k + t]
    got = host(y).astype(np.float64)
    if dt == torch.bfloat16:
        assert (np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5 * np.abs(ref).max()).all()
    else:
        assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


# ---------------------------------------------------------------------------------------
# the whole layer (moe_forward)
# ---------------------------------------------------------------------------------------
def _run_forward(shape, t, C, N=None):
    N = shape.N if N is None else N
    cfg = nat.config_from_shape(shape, N=N, capacity=C)
    ws = nat.alloc_workspace(cfg)
    E, k = shape.E, shape.k
    ro = dict(logits=torch.empty((N, E), dtype=torch.float32, device="cuda"),
              ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
              gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
              counts=torch.empty(E, dtype=torch.int32, device="cuda"),
              demand=torch.empty(E, dtype=torch.int32, device="cuda"),
              drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"),
              offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"))
    y = torch.empty_like(t["x"])
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                    logit_offset=t.get("logit_offset"), bias=t.get("bias"),
                    modality=t.get("modality"), route_out=ro, ws=ws)
    check_status(ws)
    launches = nat.moe_last_launch_count()
    return y, {kk: host(v) for kk, v in ro.items()}, launches


def _oracle_kwargs(shape, t, C):
    return dict(k=shape.k, E=shape.E, score_fn=shape.score_fn, renorm=shape.renorm,
                act=shape.act, clamp=shape.clamp, n_shared=shape.n_shared,
                bias=None if "bias" not in t else host(t["bias"]),
                modality=None if "modality" not in t else host(t["modality"]),
                logit_offset=None if "logit_offset" not in t else host(t["logit_offset"]), C=C)


def test_forward_toy_fp32_page_config():
    """The dataistudio listing's layer: 1000 tokens, d=64, 8 ReLU experts 64->256->64, top-2."""
    shape = W.PRESETS["toy"]
    t = W.make_inputs(shape, device="cuda")
    y, ro, launches = _run_forward(shape, t, 0)
    ref, info = O.forward(host(t["x"]), host(t["W_g"]), host(t["W_gu"]), host(t["W_down"]),
                          **_oracle_kwargs(shape, t, 0))
    # logits in fp32 on both sides: routing must agree except at fp32 near-ties
    frag = fragile_tokens(info["logits"], ro["logits"], 2, O.SOFTMAX)
    same = (ro["ids"] == info["ids"]).all(1)
    assert same[~frag].all()
    assert_close_layer(host(y)[same], ref[same], bf16=False)
    # per-expert load fractions (bincount / N) sum to k
    assert ro["demand"].sum() / shape.N == pytest.approx(2.0)
    assert launches == forward_launches(shape.N, shape.k, shape.E, shape.n_shared, shape.dtype == W.BF16)


def tile_edge_tokens(route, N, n_shared, tile_rows=(128, 256)):
    """Tokens that sit at the edges of the grouped GEMMs' M tiles: for every expert with kept
    rows, the first and last row of its first tile and of its last tile (for 128- and
    256-row tiles), and for the shared expert (all N tokens in token order) the tokens at
    the same edges of its tiles."""
    off = np.asarray(route["offsets"], np.int64)
    row_token = np.asarray(route["row_token"], np.int64)
    toks = []
    for e in range(off.size - 1):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        cnt = r1 - r0
        for tr in tile_rows:
            last_base = (cnt - 1) // tr * tr
            for r in (0, min(tr, cnt) - 1, last_base, cnt - 1):
                toks.append(row_token[r0 + r])
    if n_shared:
        for tr in tile_rows:
            last_base = (N - 1) // tr * tr
            toks += [0, min(tr, N) - 1, last_base, N - 1]
    return np.unique(np.asarray(toks, np.int64))


def full_range_sample(route, N, n_shared, seed=0, n_random=96):
    """Tile-edge tokens plus a seeded uniform draw over the whole token range, the last
    tokens (the last arrivals, the first to be dropped under a capacity) included."""
    rng = np.random.default_rng(seed)
    extra = rng.integers(0, N, n_random) if N > 0 else np.zeros(0, np.int64)
    tail = np.arange(max(0, N - 8), N)
    return np.unique(np.r_[tile_edge_tokens(route, N, n_shared), extra, tail]).astype(np.int64)


def _forward_case(name, N=None, sample=None, full_range=False):
    shape = W.PRESETS[name]
    if N is not None:
        shape = shape.replace(N=N)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(shape.N, shape.k, shape.E, shape.capacity_factor)
    y, ro, launches = _run_forward(shape, t, C)
    # the GPU router logits against float64
    x64 = f64(t["x"])
    off = None if "logit_offset" not in t else host(t["logit_offset"])
    z_o = O.router_logits(x64, f64(t["W_g"]), off)
    zerr = np.abs(ro["logits"].astype(np.float64) - z_o).max()
    assert zerr <= 1e-3 * np.abs(z_o).max(), zerr
    kw = _oracle_kwargs(shape, t, C)
    kw_no_off = {k: v for k, v in kw.items() if k != "logit_offset"}
    if full_range:
        # routing of every token first (cheap), then the rows at every tile edge of the
        # oracle's own layout and a draw over the whole token range
        ids_o, _ = O.route(z_o, shape.k, shape.score_fn, shape.renorm, kw["bias"], kw["modality"])
        sample = full_range_sample(O.dispatch(ids_o, shape.E, C), shape.N, shape.n_shared,
                                   seed=shape.seed)
    tokens = np.arange(shape.N) if sample is None else np.asarray(sample, np.int64)
    ref, info = O.forward(x64, f64(t["W_g"]), _LazyF64(t["W_gu"]), _LazyF64(t["W_down"]),
                          tokens=tokens, logits=z_o, **kw_no_off)
    # Routing from the GPU's logits may differ from routing on float64 logits only where the
    # logit discrepancy can explain it (fragile tokens and their capacity knock-ons)
    same_tok, why = explain_routing_differences(ro, info, z_o, ro["logits"], shape.k,
                                                shape.score_fn, kw["bias"], kw["modality"], C)
    n_diff = int((~same_tok).sum())
    if n_diff == 0:
        np.testing.assert_array_equal(ro["counts"], info["counts"])
        np.testing.assert_array_equal(ro["offsets"], info["offsets"])
    keep = same_tok[tokens]
    assert keep.mean() > 0.9
    mx, rms = err_stats(host(y)[tokens][keep], ref[keep])
    print(f"PARITY {name} N={shape.N}: logit err {zerr:.2e}, routing differs on {n_diff} "
          f"tokens ({why}), {int(keep.sum())} sampled rows compared, token range "
          f"{int(tokens.min()) if tokens.size else -1}..{int(tokens.max()) if tokens.size else -1}, "
          f"output max err {mx:.2e} x max|ref|, rms {rms:.2e}")
    assert_close_layer(host(y)[tokens][keep], ref[keep])
    assert launches == forward_launches(shape.N, shape.k, shape.E, shape.n_shared, shape.dtype == W.BF16)
    return ro


class _LazyF64:
    """Per-expert float64 view of a bf16 weight tensor on the GPU (only the slices used)."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        # bf16 -> float64 is exact; widening on the device makes the copy the only host cost
        return self.t[e].to(torch.float64).cpu().numpy()


def test_forward_small_shapes_all_tokens():
    for name, N in (("mixtral-n16", 16), ("dsv3-n64", 64), ("v41flash-n64", 64)):
        _forward_case(name, N=N)


def test_forward_large_groups_take_the_2sm_kernel(monkeypatch):
    # 4096 tokens, 8 experts, top-2: about 1024 rows per expert, so the automatic choice
    # takes the 2-SM kernel for the down projection; the forced 1-SM run must give the same
    # layer within the bar
    monkeypatch.delenv("MOE_B200_GEMM_PATH", raising=False)
    _forward_case("mixtral-n4096", sample=np.r_[0:8, 4090:4096])
    monkeypatch.setenv("MOE_B200_GEMM_PATH", "1sm")
    _forward_case("mixtral-n4096", sample=np.r_[0:8, 4090:4096])


def test_forward_tall_tiles(monkeypatch):
    """The 1-SM kernel's 256-row tiles on whole layers: a ridge-shaped layer (about 256 rows
    per expert, skewed, most groups ending in a half or an M = 64 tile) and a Mixtral-shaped
    one (1024-row groups), sampled over the whole token range."""
    monkeypatch.setenv("MOE_B200_GEMM_PATH", "tall")
    _forward_case("dsv3-n8192", N=2048, full_range=True)
    _forward_case("mixtral-n4096", full_range=True)


def test_forward_capacity_configs_reduced():
    for name in ("capacity-cf1", "capacity-cf1.25", "capacity-cfinf", "switch-cf1"):
        shape = W.PRESETS[name]
        _forward_case(name, N=2048, sample=np.r_[0:64, 2000:2048])


@pytest.mark.parametrize("name", ["mixtral-n256", "mixtral-n16384", "dsv3-n8192",
                                  "v41flash-n16384", "capacity-cf1", "capacity-cf1.25",
                                  "capacity-cfinf", "switch-cf1", "switch-cf1.25",
                                  "switch-cfinf"])
def test_forward_full_size_sampled(name):
    """Each preset layer at its stated token count: rows at the edges of every expert's first
    and last M tile (128- and 256-row tiles), the shared expert's tile edges, the last tokens
    and a uniform draw over the whole token range, against the oracle."""
    _forward_case(name, full_range=True)


def test_forward_zero_tokens_is_a_no_op():
    shape = W.PRESETS["mixtral-n16"].replace(d=256, F=256)
    t = W.make_inputs(shape.replace(N=4), device="cuda")
    cfg = nat.config_from_shape(shape, N=0)
    ws = nat.alloc_workspace(nat.config_from_shape(shape, N=4))
    y = torch.empty((1, 256), dtype=torch.bfloat16, device="cuda")   # nothing is written
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y, ws=ws)
    check_status(ws)


def test_forward_host_buffers_match_device_call():
    shape = W.PRESETS["dsv3-n64"].replace(d=512, F=256, E=32, N=200)
    t = W.make_inputs(shape, device="cuda")
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                    bias=t["bias"], ws=ws)
    xh = t["x"].cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    nat.moe_forward_host(cfg, x_host=xh, W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"],
                         y_host=yh, bias=t["bias"], ws=ws)
    check_status(ws)
    assert torch.equal(yh, y.cpu())


def test_layer_class_and_determinism():
    shape = W.PRESETS["v41flash-n64"].replace(N=300, d=256, F=256, E=48)
    t = W.make_inputs(shape, device="cuda")
    from mixture_experts_layer_50_b200 import MoELayer
    layer = MoELayer.from_workload(shape, t)
    y1 = layer.forward(t["x"], modality=t["modality"]).clone()
    y2 = layer.forward(t["x"], modality=t["modality"])
    assert torch.equal(y1, y2)
    assert layer.check_status() == 0


def test_pipelined_host_batches_match_device_calls():
    shape = W.PRESETS["v41flash-n64"].replace(N=333, d=256, F=256, E=24)
    t = W.make_inputs(shape, device="cuda")
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    g = torch.Generator().manual_seed(4)
    xs = [torch.randn(shape.N, shape.d, generator=g).to(torch.bfloat16).pin_memory() for _ in range(5)]
    ys = [torch.empty_like(xs[0]).pin_memory() for _ in range(5)]
    nat.moe_forward_host_batches(cfg, x_host=xs, W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"],
                                 y_host=ys, bias=t["bias"], modality=[t["modality"]] * 5, ws=ws)
    check_status(ws)
    for xb, yb in zip(xs, ys):
        y = torch.empty((shape.N, shape.d), dtype=torch.bfloat16, device="cuda")
        nat.moe_forward(cfg, x=xb.cuda(), W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                        bias=t["bias"], modality=t["modality"], ws=ws)
        assert torch.equal(y.cpu(), yb)


@pytest.mark.parametrize("N,d,E,k,F,S,act,clamp", [(257, 96, 5, 2, 200, 1, W.SWIGLU, 0.3),
                                                   (100, 64, 8, 2, 256, 0, W.RELU, 0.0),
                                                   (33, 1000, 3, 1, 72, 1, W.RELU, 0.0)])
def test_expert_ffn_fp32(N, d, E, k, F, S, act, clamp):
    """The fp32 expert path (the toy layer's): ragged d and F, shared expert, clamp."""
    shape = W.LayerShape("t32", N=N, d=d, E=E, k=k, F=F, n_shared=S, act=act, clamp=clamp,
                         dtype=W.F32, w_std=0.1, seed=N + d)
    t = W.make_inputs(shape, device="cuda")
    ids_o, _ = O.route(W.random_logits(N, E, 3), k)
    dsp = O.dispatch(ids_o, E, 0)
    M = int(dsp["offsets"][-1])
    xp = torch.zeros((N * k, d), dtype=torch.float32, device="cuda")
    xp[:M] = t["x"][torch.from_numpy(dsp["row_token"]).long().cuda()]
    ye = torch.zeros((N * k + S * N, d), dtype=torch.float32, device="cuda")
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    nat.moe_expert_ffn(cfg, xp=xp, offsets=dev(dsp["offsets"]), x=t["x"], W_gu=t["W_gu"],
                       W_down=t["W_down"], ye=ye, ws=ws)
    check_status(ws)
    x64, Wgu, Wd = f64(t["x"]), f64(t["W_gu"]), f64(t["W_down"])
    got = host(ye)
    for e in range(E):
        a, b = dsp["offsets"][e], dsp["offsets"][e + 1]
        if b > a:
            ref = O.expert_ffn(x64[dsp["row_token"][a:b]], Wgu[e], Wd[e], act, clamp)
            assert np.abs(got[a:b] - ref).max() <= 1e-4
    if S:
        ref = O.expert_ffn(x64, Wgu[E], Wd[E], act, clamp)
        assert np.abs(got[N * k:] - ref).max() <= 1e-4


def test_graph_replay_matches_eager_forward():
    shape = W.PRESETS["mixtral-n16"].replace(d=512, F=512, N=48)
    t = W.make_inputs(shape, device="cuda")
    from mixture_experts_layer_50_b200 import MoELayer
    layer = MoELayer.from_workload(shape, t)
    y_eager = layer.forward(t["x"]).clone()
    y = torch.empty_like(y_eager)
    layer.forward_graphed(t["x"], y)
    assert torch.equal(y, y_eager)
    # new contents in the same buffer: the replay computes on them
    x2 = torch.randn(t["x"].shape, device="cuda").to(t["x"].dtype)
    t["x"].copy_(x2)
    layer.forward_graphed(t["x"], y)
    assert torch.equal(y, layer.forward(t["x"]))
    assert layer.check_status() == 0


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    """Failure detection without a fault: a device wait on a barrier that nothing completes
    gives up after 2 ms, the status word reports MOE_ERR_TIMEOUT, and the next layer call on
    the same context runs normally."""
    shape = W.PRESETS["mixtral-n16"].replace(d=256, F=256, N=64)
    t = W.make_inputs(shape, device="cuda")
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    t0 = time.perf_counter()
    nat.moe_selftest_wait_timeout(ws, 2_000_000)
    assert nat.moe_check_status(ws) == nat.MOE_ERR_TIMEOUT
    assert time.perf_counter() - t0 < 5.0
    assert nat.moe_check_status(ws) == 0          # cleared by the read
    y = torch.empty_like(t["x"])
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y, ws=ws)
    check_status(ws)
    assert torch.isfinite(y.float()).all()


def _random_shape(seed):
    r = np.random.default_rng(1000 + seed)
    E = int(r.integers(1, 80))
    k = int(r.integers(1, min(E, 8) + 1))
    act = W.SWIGLU if r.random() < 0.7 else W.RELU
    sf = int(r.random() < 0.4)
    nb = int(r.integers(0, 3)) if sf == 1 else 0
    cf = [None, Fraction(1), Fraction(5, 4), Fraction(1, 2)][int(r.integers(0, 4))]
    return W.LayerShape(f"random-{seed}", N=int(r.integers(1, 600)), d=8 * int(r.integers(4, 65)),
                        E=E, k=k, F=8 * int(r.integers(4, 65)), n_shared=int(r.random() < 0.5),
                        score_fn=sf, renorm=int(r.random() < 0.85) if k == 1 else 1, act=act,
                        clamp=float(r.choice([0.0, 0.0, 0.5, 3.0])), n_bias_sets=nb,
                        capacity_factor=cf, zipf_skew=bool(r.random() < 0.3), w_std=0.05,
                        seed=seed)


@pytest.mark.parametrize("seed", range(12))
def test_forward_random_configurations(seed):
    """Seeded random layers (d, E, k, F, shared expert, score function, renorm, bias sets,
    activation, clamp, capacity, skew): routing bit-exact and the output within the bar,
    against the oracle fed the GPU's logits."""
    shape = _random_shape(seed)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(shape.N, shape.k, shape.E, shape.capacity_factor)
    y, ro, launches = _run_forward(shape, t, C)
    kw = _oracle_kwargs(shape, t, C)
    kw.pop("logit_offset")
    ref, info = O.forward(f64(t["x"]), None, _LazyF64(t["W_gu"]), _LazyF64(t["W_down"]),
                          logits=ro["logits"], **kw)
    for name in ("ids", "drop_mask", "counts", "demand", "offsets"):
        np.testing.assert_array_equal(ro[name], info[name], err_msg=f"{shape} {name}")
    rel = np.abs(ro["gates"] - info["gates"]) / np.maximum(np.abs(info["gates"]), 1e-30)
    assert rel.max() <= 1e-5, (shape, rel.max())
    assert_close_layer(host(y), ref)
    assert launches == forward_launches(shape.N, shape.k, shape.E, shape.n_shared, shape.dtype == W.BF16)


def _random_shape_wide(seed):
    r = np.random.default_rng(5000 + seed)
    fp32 = r.random() < 0.2
    E = int(r.integers(1, 300))
    k = int(r.integers(1, min(E, 16) + 1))
    act = W.SWIGLU if r.random() < 0.7 else W.RELU
    sf = int(r.random() < 0.5)
    nb = int(r.integers(0, 3)) if sf == 1 else 0
    cf = [None, Fraction(1), Fraction(5, 4), Fraction(1, 2), Fraction(3, 1)][int(r.integers(0, 5))]
    step = 4 if fp32 else 8
    return W.LayerShape(f"wide-{seed}", N=int(r.integers(1, 2000)),
                        d=step * int(r.integers(2, 512 // step + 1)), E=E, k=k,
                        F=step * int(r.integers(2, 512 // step + 1)),
                        n_shared=int(r.random() < 0.5), score_fn=sf,
                        renorm=int(r.random() < 0.7) if k == 1 else 1, act=act,
                        clamp=float(r.choice([0.0, 0.0, 1.0, 10.0])), n_bias_sets=nb,
                        capacity_factor=cf, zipf_skew=bool(r.random() < 0.3), w_std=0.05,
                        dtype=W.F32 if fp32 else W.BF16, seed=seed)


@pytest.mark.parametrize("seed", range(16))
def test_forward_random_configurations_wide(seed):
    """Wider random layers: up to 300 experts and k = 16, up to 2000 tokens (a sample of rows
    checked), the fp32 path, and the "report" overflow policy on a third of the capacity
    cases; routing bit-exact and the output within the bar against the oracle."""
    shape = _random_shape_wide(seed)
    reroute = shape.capacity_factor is not None and np.random.default_rng(seed).random() < 0.4
    t = W.make_inputs(shape, device="cuda")
    N, E, k = shape.N, shape.E, shape.k
    C = O.capacity(N, k, E, shape.capacity_factor)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    ro = dict(logits=torch.empty((N, E), dtype=torch.float32, device="cuda"),
              ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
              gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
              counts=torch.empty(E, dtype=torch.int32, device="cuda"),
              demand=torch.empty(E, dtype=torch.int32, device="cuda"),
              drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"),
              offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"))
    y = torch.empty_like(t["x"])
    fwd = nat.moe_forward_reroute if reroute else nat.moe_forward
    fwd(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
        logit_offset=t.get("logit_offset"), bias=t.get("bias"), modality=t.get("modality"),
        route_out=ro, ws=ws)
    check_status(ws)
    ro = {kk: host(v) for kk, v in ro.items()}
    kw = _oracle_kwargs(shape, t, C)
    kw.pop("logit_offset")
    rows = np.arange(N) if N <= 400 else np.unique(np.r_[0:32, N - 32:N,
                                                          np.random.default_rng(seed).integers(0, N, 64)])
    ref, info = O.forward(f64(t["x"]), None, _LazyF64(t["W_gu"]), _LazyF64(t["W_down"]),
                          logits=ro["logits"], tokens=rows,
                          overflow="reroute" if reroute else "drop", **kw)
    for name in ("ids", "drop_mask", "counts", "demand", "offsets"):
        np.testing.assert_array_equal(ro[name], info[name], err_msg=f"{shape} {name}")
    rel = np.abs(ro["gates"] - info["gates"]) / np.maximum(np.abs(info["gates"]), 1e-30)
    assert rel.max() <= 1e-5, (shape, rel.max())
    got = host(y)[rows].astype(np.float64)
    if shape.dtype == W.F32:
        assert np.abs(got - ref).max() <= 1e-4, (shape, np.abs(got - ref).max())
    else:
        assert_close_layer(got, ref)


@pytest.mark.parametrize("sf,nb,cf", [(0, 0, None), (1, 2, Fraction(1, 2))])
def test_forward_largest_expert_count_and_k(sf, nb, cf):
    """E = 1024 routed experts with k = 32 (the largest the ABI takes), plus a shared expert."""
    shape = W.LayerShape("max", N=200, d=64, E=1024, k=32, F=64, n_shared=1, score_fn=sf,
                         n_bias_sets=nb, capacity_factor=cf, w_std=0.05, seed=77)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(shape.N, shape.k, shape.E, cf)
    y, ro, launches = _run_forward(shape, t, C)
    kw = _oracle_kwargs(shape, t, C)
    kw.pop("logit_offset")
    ref, info = O.forward(f64(t["x"]), None, _LazyF64(t["W_gu"]), _LazyF64(t["W_down"]),
                          logits=ro["logits"], **kw)
    for name in ("ids", "drop_mask", "counts", "demand", "offsets"):
        np.testing.assert_array_equal(ro[name], info[name], err_msg=name)
    assert_close_layer(host(y), ref)
    assert launches == forward_launches(shape.N, shape.k, shape.E, shape.n_shared, shape.dtype == W.BF16)


@pytest.mark.parametrize("seed", range(12))
def test_route_random_configurations_bit_exact(seed):
    """Random routing problems on given fp32 logits (up to 1024 experts, k up to 32, capacity
    or none, ties from quantised logits): ids, counts, demand and drop mask bit-exact, gates
    within 1e-5."""
    r = np.random.default_rng(9000 + seed)
    N = int(r.integers(1, 5000))
    E = int(r.integers(1, 1025))
    k = int(r.integers(1, min(E, 32) + 1))
    sf = int(r.random() < 0.5)
    rn = int(r.random() < 0.8) if k == 1 else 1
    nb = int(r.integers(0, 3))
    C = 0 if r.random() < 0.3 else int(r.integers(1, max(2, N * k // E + 2)))
    q = float(r.choice([0.0, 0.0, 0.25]))
    z = W.random_logits(N, E, seed + 31, scale=float(r.uniform(0.5, 3.0)), quantum=q)
    bias = W.random_bias(nb, E, seed + 32) if nb else None
    mod = W.random_modality(N, seed + 33) if nb > 1 else None
    cfg = nat.make_config(N, 64, E, k, 64, n_bias_sets=nb, score_fn=sf, renorm=rn, capacity=C)
    got = gpu_route(cfg, z, bias, mod)
    assert_route_equal(got, z, k, sf, rn, bias, mod, E, C)


def test_c_client_fused_forward_equals_split_calls(tmp_path):
    """A plain C program runs moe_forward and route -> permute -> expert_ffn -> combine on
    the same layer and finds the same routing and the same output bits."""
    import subprocess
    from test_abi import _build_c_client
    exe = _build_c_client(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "moe_forward == route/permute/expert_ffn/combine" in r.stdout
