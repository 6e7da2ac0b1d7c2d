"""GPU parity of the routing variants and of the balancing by-products: forced (replayed)
routing and the hash router ("Le groupe d'experts (MoE)", exercises "Hard" and "Medium"), the
Switch balance statistic and the aux-loss-free bias update per modality."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close_layer, check_status, dev, f64, host
from mixture_experts_layer_50_b200 import _native as nat
from mixture_experts_layer_50_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _needs_cuda(cuda_dev):
    yield


def _route_out(N, E, k):
    return dict(ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
                gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
                counts=torch.empty(E, dtype=torch.int32, device="cuda"),
                demand=torch.empty(E, dtype=torch.int32, device="cuda"),
                drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"),
                offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"))


def test_replayed_routing_reproduces_the_forward_bit_for_bit():
    shape = W.PRESETS["v41flash-n64"].replace(N=700, d=512, F=256, E=32, k=4)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(shape.N, shape.k, shape.E, 1)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    ro = _route_out(shape.N, shape.E, shape.k)
    y = torch.empty_like(t["x"])
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                    bias=t["bias"], modality=t["modality"], route_out=ro, ws=ws)
    check_status(ws)
    # record, then force the same routing
    y2 = torch.empty_like(y)
    ro2 = {k_: torch.empty_like(ro[k_]) for k_ in ("counts", "demand", "drop_mask", "offsets")}
    nat.moe_forward_routed(cfg, x=t["x"], ids=ro["ids"].clone(), gates=ro["gates"].clone(),
                           W_gu=t["W_gu"], W_down=t["W_down"], y=y2, route_out=ro2, ws=ws)
    check_status(ws)
    assert torch.equal(y2, y)
    for k_ in ro2:
        assert torch.equal(ro2[k_], ro[k_]), k_
    assert nat.moe_last_launch_count() == 6


@pytest.mark.parametrize("C", [0, 40])
def test_forced_routing_against_the_oracle(C):
    shape = W.PRESETS["dsv3-n64"].replace(N=300, d=256, F=384, E=16, k=3)
    t = W.make_inputs(shape, device="cuda")
    rng = np.random.default_rng(5)
    # arbitrary forced routing: k distinct experts per token, arbitrary positive gates
    ids = np.stack([rng.permutation(shape.E)[:shape.k] for _ in range(shape.N)]).astype(np.int32)
    gates = rng.uniform(0.1, 1.0, ids.shape).astype(np.float32)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    ro = {"drop_mask": torch.empty((shape.N, shape.k), dtype=torch.uint8, device="cuda")}
    y = torch.empty_like(t["x"])
    nat.moe_forward_routed(cfg, x=t["x"], ids=dev(ids), gates=dev(gates), W_gu=t["W_gu"],
                           W_down=t["W_down"], y=y, route_out=ro, ws=ws)
    check_status(ws)
    ref, info = O.forward(f64(t["x"]), None, f64(t["W_gu"]), f64(t["W_down"]), k=shape.k,
                          E=shape.E, n_shared=shape.n_shared, C=C, ids=ids,
                          gates=gates.astype(np.float64))
    np.testing.assert_array_equal(host(ro["drop_mask"]), info["drop_mask"])
    assert_close_layer(host(y), ref)


def test_forced_routing_reports_bad_ids():
    shape = W.PRESETS["dsv3-n64"].replace(N=64, d=256, F=256, E=8, k=2)
    t = W.make_inputs(shape, device="cuda")
    ids = np.tile(np.array([[1, 2]], np.int32), (64, 1))
    ids[5] = [8, 1]          # out of range: dropped
    cfg = nat.config_from_shape(shape)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    nat.moe_forward_routed(cfg, x=t["x"], ids=dev(ids), gates=dev(np.full((64, 2), 0.5, np.float32)),
                           W_gu=t["W_gu"], W_down=t["W_down"], y=y, ws=ws)
    assert nat.moe_check_status(ws) == nat.MOE_ERR_INVALID_INPUT


@pytest.mark.parametrize("N,E,k,C", [(1000, 64, 2, 0), (4097, 384, 6, 80), (33, 8, 1, 3)])
def test_hash_router_bit_exact(N, E, k, C):
    tok = np.random.default_rng(N).integers(0, 2**31 - 1, N).astype(np.int32)
    cfg = nat.make_config(N, 64, E, k, 64, capacity=C)
    ws = nat.alloc_workspace(cfg)
    out = dict(ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
               gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
               counts=torch.empty(E, dtype=torch.int32, device="cuda"),
               demand=torch.empty(E, dtype=torch.int32, device="cuda"),
               drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"))
    nat.moe_route_hash(cfg, token_ids=dev(tok), ws=ws, **out)
    check_status(ws)
    ids_o, gates_o = O.hash_route(tok, E, k)
    d_o = O.dispatch(ids_o, E, C)
    np.testing.assert_array_equal(host(out["ids"]), ids_o)
    np.testing.assert_array_equal(host(out["gates"]), gates_o.astype(np.float32))
    for name in ("counts", "demand", "drop_mask"):
        np.testing.assert_array_equal(host(out[name]), d_o[name])


@pytest.mark.parametrize("N,E,k,sf,nb", [(1000, 8, 2, 0, 0), (4096, 384, 6, 1, 2), (777, 64, 1, 0, 1)])
def test_balance_statistics_and_bias_update(N, E, k, sf, nb):
    z = W.random_logits(N, E, N + E, scale=1.5)
    bias = W.random_bias(max(nb, 1), E, 9) if nb else np.zeros((1, E), np.float32)
    mod = W.random_modality(N, 10) if nb > 1 else None
    ids, _ = O.route(z, k, sf, 1, bias if nb else None, mod)
    cfg = nat.make_config(N, 64, E, k, 64, n_bias_sets=nb, score_fn=sf)
    ws = nat.alloc_workspace(cfg)
    sets = max(nb, 1)
    f = torch.empty(E, device="cuda")
    P = torch.empty(E, device="cuda")
    aux = torch.empty(1, device="cuda")
    set_load = torch.empty((sets, E), dtype=torch.int32, device="cuda")
    b = dev(bias)
    nat.moe_balance(cfg, logits=dev(z), ids=dev(ids), modality=None if mod is None else dev(mod),
                    f=f, P=P, aux=aux, set_load=set_load, bias=b, gamma=0.001, ws=ws)
    check_status(ws)
    f_o, P_o, aux_o = O.balance_stats(z, ids, E, sf)
    load_o = O.per_set_load(ids, E, mod, sets)
    np.testing.assert_array_equal(host(f), f_o.astype(np.float32))
    np.testing.assert_allclose(host(P), P_o, rtol=1e-5)
    assert abs(float(aux.item()) - aux_o) <= 1e-5 * aux_o
    np.testing.assert_array_equal(host(set_load), load_o)
    np.testing.assert_array_equal(host(b), O.bias_update(bias, load_o, 0.001))


def test_padded_dispatch_buffer_matches_the_slides_table():
    """Capacity as a tensor dimension: the [E, C, d] buffer of the 8-token, 4-expert trace."""
    from golden.reader import ints, load
    g = load("p2_capacity_trace.txt")
    assign = [tuple(int(v) for v in p.split()) for p in g["assign"].split("|")]
    ids = np.array(assign, np.int32)
    E, C, d = 4, int(g["C_1.25"]), 64
    cfg = nat.make_config(8, d, E, 2, 64, capacity=C)
    ws = nat.alloc_workspace(cfg)
    x = torch.arange(8 * d, dtype=torch.float32).reshape(8, d).to(torch.bfloat16).cuda() + 1
    offsets_pad = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    row_token = torch.full((E * C,), 77, dtype=torch.int32, device="cuda")
    slot_row = torch.empty((8, 2), dtype=torch.int32, device="cuda")
    xp = torch.full((E * C, d), 5.0, dtype=torch.bfloat16, device="cuda")
    nat.moe_permute_padded(cfg, ids=dev(ids), x=x, offsets_pad=offsets_pad, counts=counts,
                           row_token_pad=row_token, slot_row=slot_row, xp_pad=xp, ws=ws)
    check_status(ws)
    p = O.dispatch_padded(ids, E, C)
    np.testing.assert_array_equal(host(row_token), p["row_token"])
    np.testing.assert_array_equal(host(slot_row), p["slot_row"])
    np.testing.assert_array_equal(host(counts), p["counts"])
    np.testing.assert_array_equal(host(offsets_pad), np.arange(E + 1) * C)
    for e in range(E):
        assert host(row_token)[e * C:e * C + len(ints(g[f"table_E{e}"]))].tolist() == ints(g[f"table_E{e}"])
    rt = host(row_token)
    xh = x.cpu()
    for r in range(E * C):
        if rt[r] >= 0:
            assert torch.equal(xp[r].cpu(), xh[rt[r]])
        else:
            assert (xp[r].cpu() == 0).all()


def test_padded_forward_equals_the_compact_forward():
    shape = W.PRESETS["capacity-cf1.25"].replace(N=3000, d=512, F=256)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(shape.N, shape.k, shape.E, shape.capacity_factor)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    yp = torch.empty_like(t["x"])
    off = torch.empty(shape.E + 1, dtype=torch.int32, device="cuda")
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                    logit_offset=t["logit_offset"], ws=ws)
    nat.moe_forward_padded(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"],
                           y=yp, logit_offset=t["logit_offset"], route_out={"offsets": off}, ws=ws)
    check_status(ws)
    np.testing.assert_array_equal(host(off), np.arange(shape.E + 1) * C)
    # the same kernels on the same rows: each output row is computed from the same operands
    # in the same order, so the two layouts agree to the bit
    assert torch.equal(yp, y)


# ---------------------------------------------------------------------------------------
# overflow policy "report" (slides, "Politiques de débordement", row "Report sur E2/E3")
# ---------------------------------------------------------------------------------------
def _gpu_reroute(cfg, z, bias=None, mod=None):
    N, E, k = cfg.N, cfg.E, cfg.k
    ws = nat.alloc_workspace(cfg)
    out = dict(ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
               gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
               counts=torch.empty(E, dtype=torch.int32, device="cuda"),
               demand=torch.empty(E, dtype=torch.int32, device="cuda"),
               drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"),
               rerouted=torch.empty((N, k), dtype=torch.uint8, device="cuda"))
    nat.moe_route_reroute(cfg, logits=dev(z), bias=None if bias is None else dev(bias),
                          modality=None if mod is None else dev(mod), ws=ws, **out)
    check_status(ws)
    return {k_: host(v) for k_, v in out.items()}


def _assert_reroute_equal(got, z, k, sf, rn, bias, mod, E, C):
    ids_o, gates_o, drop_o, rr_o, first = O.route_reroute(z, k, C, sf, rn, bias, mod)
    np.testing.assert_array_equal(got["ids"], ids_o)
    np.testing.assert_array_equal(got["drop_mask"], drop_o)
    np.testing.assert_array_equal(got["rerouted"], rr_o)
    np.testing.assert_array_equal(got["demand"], first["demand"])
    np.testing.assert_array_equal(got["counts"], O.dispatch_masked(ids_o, E, drop_o)["counts"])
    rel = np.abs(got["gates"] - gates_o) / np.maximum(np.abs(gates_o), 1e-30)
    assert rel.max() <= 1e-5, rel.max()
    return rr_o


@pytest.mark.parametrize("N,E,k,sf,rn,nb,cf", [
    (3000, 64, 2, 0, 1, 0, 1),            # Zipf-skewed softmax top-2, cf = 1: many moves
    (2000, 32, 4, 1, 1, 2, 1),            # sigmoid + two bias sets, top-4
    (4096, 64, 1, 0, 0, 0, 1),            # Switch: raw probability gates
    (1000, 8, 6, 0, 1, 0, 1),             # 2k > E: the last candidates do not exist
    (777, 40, 16, 1, 1, 1, 1),            # k = 16, the largest the policy takes
])
def test_reroute_routing_bit_exact(N, E, k, sf, rn, nb, cf):
    z = W.random_logits(N, E, N + k, scale=1.5)
    z = (z + W.zipf_logit_offsets(E)[None, :] * (sf == 0)).astype(np.float32)
    bias = W.random_bias(nb, E, N) if nb else None
    mod = W.random_modality(N, N + 1) if nb > 1 else None
    C = O.capacity(N, k, E, cf)
    cfg = nat.make_config(N, 64, E, k, 64, n_bias_sets=nb, score_fn=sf, renorm=rn, capacity=C)
    got = _gpu_reroute(cfg, z, bias, mod)
    rr = _assert_reroute_equal(got, z, k, sf, rn, bias, mod, E, C)
    assert rr.sum() > 0


def test_reroute_on_the_slides_trace():
    from golden.reader import load
    g = load("p2_capacity_trace.txt")
    assign = [tuple(int(v) for v in p.split()) for p in g["assign"].split("|")]
    z = np.full((8, 4), 0.2, np.float32)
    for t, (a, b) in enumerate(assign):
        z[t, a], z[t, b] = 2.1, 1.8
    z[5, 3] = -1.0
    cfg = nat.make_config(8, 64, 4, 2, 64, capacity=int(g["C_1.25"]))
    got = _gpu_reroute(cfg, z)
    assert got["ids"][5].tolist() == [int(g["report_t6_expert"]), 1]
    assert got["counts"].tolist() == [5, 4, 4, 3] and got["drop_mask"].sum() == 0
    _assert_reroute_equal(got, z, 2, O.SOFTMAX, 1, None, None, 4, int(g["C_1.25"]))


def test_reroute_forward_against_the_oracle():
    shape = W.PRESETS["capacity-cf1"].replace(N=2048, d=256, F=256)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(shape.N, shape.k, shape.E, shape.capacity_factor)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    N, k, E = shape.N, shape.k, shape.E
    ro = dict(logits=torch.empty((N, E), device="cuda"),
              ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
              drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"),
              counts=torch.empty(E, dtype=torch.int32, device="cuda"))
    rr = torch.empty((N, k), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["x"])
    nat.moe_forward_reroute(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                            logit_offset=t["logit_offset"], route_out=ro, rerouted=rr, ws=ws)
    check_status(ws)
    z = host(ro["logits"])
    sample = np.r_[0:40, 2000:2048]
    ref, info = O.forward(f64(t["x"]), None, _Lazy(t["W_gu"]), _Lazy(t["W_down"]), k=k, E=E,
                          n_shared=shape.n_shared, C=C, logits=z, tokens=sample,
                          overflow="reroute")
    np.testing.assert_array_equal(host(ro["ids"]), info["ids"])
    np.testing.assert_array_equal(host(ro["drop_mask"]), info["drop_mask"])
    np.testing.assert_array_equal(host(rr), info["rerouted"])
    np.testing.assert_array_equal(host(ro["counts"]), info["counts"])
    assert info["rerouted"].sum() > 0
    assert_close_layer(host(y)[sample], ref)


def test_reroute_without_capacity_is_the_plain_forward():
    shape = W.PRESETS["dsv3-n64"].replace(N=300, d=256, F=256, E=16, k=4)
    t = W.make_inputs(shape, device="cuda")
    cfg = nat.config_from_shape(shape, capacity=0)
    ws = nat.alloc_workspace(cfg)
    y1, y2 = torch.empty_like(t["x"]), torch.empty_like(t["x"])
    rr = torch.full((shape.N, shape.k), 7, dtype=torch.uint8, device="cuda")
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y1,
                    bias=t["bias"], ws=ws)
    nat.moe_forward_reroute(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"],
                            y=y2, bias=t["bias"], rerouted=rr, ws=ws)
    check_status(ws)
    assert torch.equal(y1, y2) and int(rr.sum()) == 0


def test_reroute_refuses_k_above_16():
    cfg = nat.make_config(64, 64, 40, 17, 64, capacity=10)
    ws = nat.alloc_workspace(cfg)
    with pytest.raises(nat.MoeError) as e:
        nat.moe_route_reroute(cfg, logits=dev(np.zeros((64, 40), np.float32)),
                              ids=torch.empty((64, 17), dtype=torch.int32, device="cuda"),
                              gates=torch.empty((64, 17), device="cuda"), ws=ws)
    assert e.value.status == nat.MOE_ERR_UNSUPPORTED


class _Lazy:
    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return f64(self.t[e])


def test_layer_with_reroute_policy_device_and_host_buffers():
    from mixture_experts_layer_50_b200 import MoELayer
    shape = W.PRESETS["switch-cf1"].replace(N=1024, d=256, F=256)
    t = W.make_inputs(shape, device="cuda")
    layer = MoELayer.from_workload(shape, t, overflow="reroute")
    C = layer.capacity(shape.N)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    y_ref = torch.empty_like(t["x"])
    nat.moe_forward_reroute(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"],
                            y=y_ref, logit_offset=t["logit_offset"], ws=ws)
    check_status(ws)
    assert torch.equal(layer.forward(t["x"]), y_ref)
    xh = t["x"].cpu().pin_memory()
    yh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    layer.forward_host(xh, yh[0])
    layer.forward_host_batches([xh, xh], yh)
    assert torch.equal(yh[0], y_ref.cpu()) and torch.equal(yh[1], y_ref.cpu())
    assert layer.check_status() == 0


@pytest.mark.parametrize("N,E,k,cf,sf,nb", [(1, 8, 2, None, 0, 0), (16, 8, 2, 1, 0, 0),
                                            (64, 256, 8, None, 1, 1), (64, 384, 6, 1.25, 1, 2),
                                            (48, 64, 2, 1, 0, 0), (64, 1024, 8, 2, 1, 1)])
def test_small_batch_dispatch_equals_the_three_passes(N, E, k, cf, sf, nb, monkeypatch):
    """A small batch takes the one-launch dispatch; it must give the three passes' results bit
    for bit (routing outputs, layout, layer output)."""
    shape = W.LayerShape("small", N=N, d=256, E=E, k=k, F=128, n_shared=1, score_fn=sf,
                         n_bias_sets=nb, capacity_factor=cf, w_std=0.05, seed=N + E)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(N, k, E, cf)
    cfg = nat.config_from_shape(shape, capacity=C)
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_B200_SMALL_DISPATCH", flag)
        ws = nat.alloc_workspace(cfg)
        ro = _route_out(N, E, k)
        y = torch.empty_like(t["x"])
        nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                        bias=t.get("bias"), modality=t.get("modality"), route_out=ro, ws=ws)
        check_status(ws)
        outs.append((y, ro, nat.moe_last_launch_count()))
    (y1, r1, l1), (y0, r0, l0) = outs
    side = 2 if k <= 2 else 0   # the shared expert's two GEMMs on the side stream
    assert (l1, l0) == (6 + side, 8 + side)
    assert torch.equal(y1, y0)
    for name in r1:
        assert torch.equal(r1[name], r0[name]), name


def test_small_batch_dispatch_reports_bad_ids_like_the_three_passes(monkeypatch):
    """Forced routing with an id out of range and an id repeated within a token: both dispatch
    forms drop them and report MOE_ERR_INVALID_INPUT, with the same layout otherwise."""
    N, E, k = 12, 6, 3
    shape = W.LayerShape("bad", N=N, d=128, E=E, k=k, F=64, w_std=0.05, seed=5)
    t = W.make_inputs(shape, device="cuda")
    ids = np.tile(np.array([0, 1, 2], np.int32), (N, 1))
    ids[3] = [4, 4, 5]          # repeated within the token
    ids[7] = [1, 9, 2]          # out of range
    gates = np.full((N, k), 1.0 / k, np.float32)
    cfg = nat.config_from_shape(shape, capacity=4)
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_B200_SMALL_DISPATCH", flag)
        ws = nat.alloc_workspace(cfg)
        ro = {n: v for n, v in _route_out(N, E, k).items() if n in ("counts", "demand",
                                                                    "drop_mask", "offsets")}
        y = torch.empty_like(t["x"])
        nat.moe_forward_routed(cfg, x=t["x"], ids=dev(ids), gates=dev(gates), W_gu=t["W_gu"],
                               W_down=t["W_down"], y=y, route_out=ro, ws=ws)
        assert nat.moe_check_status(ws) == nat.MOE_ERR_INVALID_INPUT
        outs.append((y, ro))
    (y1, r1), (y0, r0) = outs
    assert torch.equal(y1, y0)
    for name in r1:
        assert torch.equal(r1[name], r0[name]), name


@pytest.mark.parametrize("N,E,k,cf,sf,nb", [(3000, 384, 6, None, 1, 2), (4097, 64, 2, 1, 0, 0),
                                            (1000, 300, 32, 0.5, 1, 1), (300, 8, 1, 1.25, 0, 0)])
def test_topk_fused_with_the_rank_pass_equals_separate_launches(N, E, k, cf, sf, nb, monkeypatch):
    """Top-k fused with the rank pass (opt-in, MOE_B200_FUSED_TOPK_RANK=1): the outputs must
    be those of the separate launches, bit for bit."""
    shape = W.LayerShape("fused", N=N, d=128, E=E, k=k, F=64, n_shared=1, score_fn=sf,
                         renorm=1, n_bias_sets=nb, capacity_factor=cf, w_std=0.05, seed=N + k)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(N, k, E, cf)
    cfg = nat.config_from_shape(shape, capacity=C)
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_B200_FUSED_TOPK_RANK", flag)
        ws = nat.alloc_workspace(cfg)
        ro = _route_out(N, E, k)
        y = torch.empty_like(t["x"])
        nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                        bias=t.get("bias"), modality=t.get("modality"), route_out=ro, ws=ws)
        check_status(ws)
        outs.append((y, ro, nat.moe_last_launch_count()))
    (y1, r1, l1), (y0, r0, l0) = outs
    side = 2 if k <= 2 else 0   # the shared expert's two GEMMs on the side stream
    assert (l1, l0) == (7 + side, 8 + side)
    assert torch.equal(y1, y0)
    for name in r1:
        assert torch.equal(r1[name], r0[name]), name


@pytest.mark.parametrize("N,E,k,cf,reroute", [(16, 8, 2, None, False), (3000, 64, 2, 1, False),
                                              (700, 384, 6, 1.25, False), (900, 16, 2, 1, True)])
def test_debug_mode_checks_the_layout_of_every_call(N, E, k, cf, reroute, monkeypatch):
    """MOE_B200_DEBUG=1: the fused calls check their dispatch layout on the host (it holds),
    and moe_check_dispatch on the device outputs agrees."""
    monkeypatch.setenv("MOE_B200_DEBUG", "1")
    shape = W.LayerShape("dbg", N=N, d=128, E=E, k=k, F=64, n_shared=1, capacity_factor=cf,
                         w_std=0.05, seed=N)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(N, k, E, cf)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    ro = _route_out(N, E, k)
    y = torch.empty_like(t["x"])
    fwd = nat.moe_forward_reroute if reroute else nat.moe_forward
    fwd(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y, route_out=ro,
        ws=ws)
    check_status(ws)
    if not reroute:
        slot = torch.empty((N, k), dtype=torch.int32, device="cuda")
        xp = torch.empty((N * k, shape.d), dtype=torch.bfloat16, device="cuda")
        off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
        nat.moe_permute(cfg, ids=ro["ids"], drop_mask=ro["drop_mask"], x=t["x"], offsets=off,
                        slot_row=slot, xp=xp, ws=ws)
        nat.moe_check_dispatch(cfg, ids=ro["ids"], drop_mask=ro["drop_mask"], counts=ro["counts"],
                               demand=ro["demand"], offsets=off, slot_row=slot)


@pytest.mark.parametrize("N,d,E,k,F,S,cf,act", [(16, 256, 8, 2, 384, 0, None, W.SWIGLU),
                                                (64, 512, 48, 6, 256, 1, None, W.SWIGLU),
                                                (37, 136, 6, 3, 200, 1, 1.25, W.SWIGLU),
                                                (1, 128, 4, 2, 128, 1, None, W.SWIGLU),
                                                (50, 192, 8, 2, 320, 0, 1, W.RELU)])
def test_decode_batch_64_row_stages_equal_full_stages(N, d, E, k, F, S, cf, act, monkeypatch):
    """A batch of at most 64 tokens runs the 1-SM GEMMs with 64-row tiles (every group fits
    one); the layer output, compact and padded, must be the bits of the 128-row tiles (whose
    tiles of at most 64 rows run the same M = 64 MMAs)."""
    shape = W.LayerShape("a64", N=N, d=d, E=E, k=k, F=F, n_shared=S, act=act,
                         capacity_factor=cf, w_std=0.05, seed=N + d)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(N, k, E, cf)
    cfg = nat.config_from_shape(shape, capacity=C)
    names = []
    outs = []
    for flag in ("1", "0"):
        monkeypatch.setenv("MOE_B200_DECODE_A64", flag)
        names.append(nat.moe_ffn_kernels(cfg))
        ws = nat.alloc_workspace(cfg)
        ys = []
        for fwd in ([nat.moe_forward] + ([nat.moe_forward_padded] if C > 0 else [])):
            y = torch.empty_like(t["x"])
            fwd(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y, ws=ws)
            check_status(ws)
            ys.append(y)
        outs.append(ys)
    assert all("1-SM, 64x" in n for n in names[0]) and not any("64x" in n for n in names[1])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("name,N,k", [("capacity-cf1", 3000, 2), ("dsv3-n64", 64, 2),
                                      ("v41flash-n64", 300, 1), ("switch-cf1", 777, 1)])
def test_shared_expert_on_the_side_stream_gives_the_same_bits(name, N, k, monkeypatch):
    """The shared expert's GEMMs on the library's side stream (concurrent with the routing
    chain) give the bits of the shared group inside the routed GEMM launches, eagerly and
    replayed from a CUDA graph that captured the fork and the join."""
    shape = W.PRESETS[name].replace(N=N, d=256, F=256, k=k)
    t = W.make_inputs(shape, device="cuda")
    from mixture_experts_layer_50_b200 import MoELayer
    ys = []
    for flag in ("0", "1"):
        monkeypatch.setenv("MOE_B200_SHARED_STREAM", flag)
        layer = MoELayer.from_workload(shape, t)
        y = layer.forward(t["x"], modality=t.get("modality")).clone()
        assert layer.check_status() == 0
        launches = nat.moe_last_launch_count()
        yg = torch.empty_like(y)
        for _ in range(2):
            layer.forward_graphed(t["x"], yg, modality=t.get("modality"))
        torch.cuda.synchronize()
        assert torch.equal(yg, y)
        ys.append((y, launches))
    (y0, l0), (y1, l1) = ys
    assert l1 == l0 + 2
    assert torch.equal(y0, y1)
