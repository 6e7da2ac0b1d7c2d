"""Expert-parallel layer on one GPU: the library's kernels on the per-rank layouts.

"Mixture-of-Experts : routage et capacité" slides, "L'idée — Communication".  A run here has one
GPU, so several ranks are emulated in one process: each emulated rank has its own layer object
(its experts, its workspace) and the row exchange is ``loopback_exchange`` (plain copies between
the ranks' buffers, in the plan's runs).  No kernel waits on another rank.  The result must equal
the single-device layer over the concatenated batch: bit for bit against the fused call given
the same routing, and within the bf16 bar against the oracle.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
from gpu_util import assert_close_layer, check_status, f64, host
from mixture_experts_layer_50_b200 import _native as nat
from mixture_experts_layer_50_b200 import workloads as W
from mixture_experts_layer_50_b200.ep import EPMoELayer, loopback_exchange

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _needs_cuda(cuda_dev):
    yield


def _layers(shape, t, world, max_tokens, cf):
    return [EPMoELayer.from_full_weights(
        W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], k=shape.k, E=shape.E, world=world,
        rank=r, n_shared=shape.n_shared, score_fn=shape.score_fn, renorm=shape.renorm,
        act=shape.act, clamp=shape.clamp, bias=t.get("bias"), logit_offset=t.get("logit_offset"),
        capacity_factor=cf, max_tokens=max_tokens) for r in range(world)]


def emulate(layers, xs, mods):
    """Every phase of the layer for all emulated ranks, the exchanges by loopback copies."""
    world = len(layers)
    dem = [L.route(x, m) for L, x, m in zip(layers, xs, mods)]
    gathered = torch.stack(dem).cpu()
    plans = [L.set_plan(gathered) for L in layers]
    sends = [L.permute(x) for L, x in zip(layers, xs)]
    recv = [L.new_recv_buffer() for L in layers]
    loopback_exchange(sends, recv, [p["sends"] for p in plans], [p["recvs"] for p in plans])
    ys = [torch.empty_like(x) for x in xs]
    ye = [L.run_experts(r, x, y) for L, r, x, y in zip(layers, recv, xs, ys)]
    back = [L.new_return_buffer() for L in layers]
    loopback_exchange(ye, back, [p["recvs"] for p in plans], [p["sends"] for p in plans])
    for L, b, y in zip(layers, back, ys):
        L.combine(b, y)
        check_status(L.ws)
    return ys, plans


def _split(N, world, seed, empty_rank=None):
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.integers(N // 8, N - N // 8, world - 1)) if world > 1 else np.zeros(0, int)
    sizes = np.diff(np.r_[0, cuts, N]).astype(int)
    if empty_rank is not None and world > 1:
        other = (empty_rank + 1) % world
        sizes[other] += sizes[empty_rank]
        sizes[empty_rank] = 0
    return sizes


CASES = [
    # preset, N, d, E, F, k, cf
    ("capacity-cf1", 600, 256, 16, 256, 2, 1),
    ("dsv3-n64", 500, 256, 24, 128, 4, None),
    ("v41flash-n64", 700, 512, 30, 256, 3, 1.25),
    ("mixtral-n16", 400, 256, 8, 384, 2, None),
    ("switch-cf1", 512, 128, 12, 128, 1, 1),
]


@pytest.mark.parametrize("case", CASES)
def test_one_rank_equals_the_fused_layer_bit_for_bit(case):
    """world = 1: route, plan, permute, a local exchange, the experts and the combine give
    moe_forward's output bits (and moe_forward_padded's, with a capacity)."""
    name, N, d, E, F, k, cf = case
    shape = W.PRESETS[name].replace(N=N, d=d, E=E, F=F, k=k)
    t = W.make_inputs(shape, device="cuda")
    C = O.capacity(N, k, E, cf)
    (L,) = _layers(shape, t, 1, N, cf)
    (y_ep,), _ = emulate([L], [t["x"]], [t.get("modality")])
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    kw = dict(x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
              logit_offset=t.get("logit_offset"), bias=t.get("bias"), modality=t.get("modality"),
              ws=ws)
    nat.moe_forward(cfg, **kw)
    check_status(ws)
    assert torch.equal(y_ep, y)
    if C > 0:
        nat.moe_forward_padded(cfg, **kw)
        check_status(ws)
        assert torch.equal(y_ep, y)


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("case", CASES)
def test_emulated_ranks_equal_the_single_device_layer(world, case, monkeypatch):
    """Several emulated ranks (one without tokens in some cases): every rank's output equals,
    bit for bit, the fused layer over the concatenated batch given the same routing
    (moe_forward_routed: the ranks' own ids and gates, capacity in the concatenated token
    order), and the oracle within the bf16 bar; the drop masks equal the oracle's."""
    monkeypatch.setenv("MOE_B200_GEMM_PATH", "1sm")       # one GEMM kernel on both sides
    name, N, d, E, F, k, cf = case
    shape = W.PRESETS[name].replace(N=N, d=d, E=E, F=F, k=k)
    if world > E:
        pytest.skip("more ranks than experts")
    t = W.make_inputs(shape, device="cuda")
    sizes = _split(N, world, seed=world * 31 + E, empty_rank=1 if world == 3 else None)
    starts = np.r_[0, np.cumsum(sizes)]
    xs = [t["x"][starts[r]:starts[r + 1]] for r in range(world)]
    mod = t.get("modality")
    mods = [None if mod is None else mod[starts[r]:starts[r + 1]] for r in range(world)]
    layers = _layers(shape, t, world, int(sizes.max()) if sizes.max() > 0 else 1, cf)
    ys, plans = emulate(layers, xs, mods)
    y_ep = torch.cat(ys)
    ids = torch.cat([L.ids[:L.N] for L in layers])
    gates = torch.cat([L.gates[:L.N] for L in layers])
    drop = torch.cat([L.drop_mask[:L.N] for L in layers])
    C = O.capacity(N, k, E, cf)
    assert all(p["capacity"] == C for p in plans)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    ro = dict(drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"))
    nat.moe_forward_routed(cfg, x=t["x"], ids=ids, gates=gates, W_gu=t["W_gu"],
                           W_down=t["W_down"], y=y, route_out=ro, ws=ws)
    check_status(ws)
    assert torch.equal(drop, ro["drop_mask"])
    assert torch.equal(y_ep, y)
    # the oracle on the same routing (the ranks' ids and gates), capacity in token order
    ref, info = O.forward(f64(t["x"]), None, f64(t["W_gu"]), f64(t["W_down"]), k=k, E=E,
                          n_shared=shape.n_shared, act=shape.act, clamp=shape.clamp,
                          ids=host(ids), gates=host(gates).astype(np.float64), C=C)
    np.testing.assert_array_equal(host(drop), info["drop_mask"])
    assert_close_layer(host(y_ep), ref)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("transport", ["nccl", "p2p"])
def test_forward_over_a_one_rank_nccl_group(transport):
    """EPMoELayer.forward itself (NCCL all-gather of the demands, then the row exchange, or
    with the peer-memory transport the fused dispatch and combine around its stream-ordered
    NCCL barriers) on a one-rank NCCL group equals moe_forward bit for bit, twice in a row."""
    import torch.distributed as dist
    shape = W.PRESETS["v41flash-n64"].replace(N=300, d=256, E=16, F=128, k=4)
    t = W.make_inputs(shape, device="cuda")
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True,
                          timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        (L,) = [EPMoELayer.from_full_weights(
            W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], k=shape.k, E=shape.E, world=1,
            rank=0, n_shared=shape.n_shared, score_fn=shape.score_fn, renorm=shape.renorm,
            act=shape.act, clamp=shape.clamp, bias=t.get("bias"),
            logit_offset=t.get("logit_offset"), capacity_factor=1.25, max_tokens=shape.N,
            transport=transport)]
        y_first = L.forward(t["x"], modality=t["modality"]).clone()
        y_ep = L.forward(t["x"], modality=t["modality"])
        torch.cuda.synchronize()
        assert L.check_status() == 0
        assert torch.equal(y_first, y_ep)
        L.close()
    finally:
        dist.destroy_process_group()
    C = O.capacity(shape.N, shape.k, shape.E, 1.25)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    nat.moe_forward(cfg, x=t["x"], W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], y=y,
                    bias=t["bias"], modality=t["modality"], ws=ws)
    check_status(ws)
    assert torch.equal(y_ep, y)


# ---- the peer-memory transport (moe_ep_copy_runs, CUDA IPC) --------------------------------
@pytest.mark.parametrize("world", [2, 4])
def test_copy_runs_moves_the_rows_the_message_exchange_moves(world):
    """moe_ep_copy_runs with a table of destination buffers (local here, one per emulated
    rank) leaves every receive and return buffer bit for bit as the message exchange does;
    a run that points past its buffer is skipped and reported."""
    from mixture_experts_layer_50_b200.ep import all_plans, loopback_exchange, peer_runs
    N, d, E, k = 500, 264, 12, 3
    rng = np.random.default_rng(world)
    z = rng.normal(0, 1, (N, E)).astype(np.float32)
    z[:, 0] += 1.0
    ids, _ = O.route(z, k)
    C = O.capacity(N, k, E, 1.25)
    sizes = _split(N, world, seed=world)
    starts = np.r_[0, np.cumsum(sizes)]
    demand = np.stack([np.bincount(ids[starts[r]:starts[r + 1]].ravel(), minlength=E)
                       for r in range(world)]).astype(np.int32)
    plans = all_plans(world, E, C, demand)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    sends = [torch.randn(max(1, p["rows_kept"]), d, device="cuda").to(torch.bfloat16)
             for p in plans]
    want = [torch.zeros(max(1, p["rows_owned"]), d, **bf) for p in plans]
    loopback_exchange(sends, want, [p["sends"] for p in plans], [p["recvs"] for p in plans])
    got = [torch.zeros_like(w) for w in want]
    base = torch.tensor([g.data_ptr() for g in got], dtype=torch.int64, device="cuda")
    rows = torch.tensor([g.shape[0] for g in got], dtype=torch.int64, device="cuda")
    ws = nat.alloc_workspace(nat.make_config(16, d, E, k, 64))
    for r in range(world):
        nat.moe_ep_copy_runs(sends[r], dst_base=base, dst_rows=rows,
                             runs=peer_runs(r, plans, "dispatch"), ws=ws)
    check_status(ws)
    for g, w in zip(got, want):
        assert torch.equal(g, w)
    outs = [w.float().mul(0.5).to(torch.bfloat16) for w in want]
    want_back = [torch.zeros_like(s) for s in sends]
    loopback_exchange(outs, want_back, [p["recvs"] for p in plans], [p["sends"] for p in plans])
    got_back = [torch.zeros_like(s) for s in sends]
    base_b = torch.tensor([g.data_ptr() for g in got_back], dtype=torch.int64, device="cuda")
    rows_b = torch.tensor([g.shape[0] for g in got_back], dtype=torch.int64, device="cuda")
    for r in range(world):
        nat.moe_ep_copy_runs(outs[r], dst_base=base_b, dst_rows=rows_b,
                             runs=peer_runs(r, plans, "return"), ws=ws)
    check_status(ws)
    for g, w in zip(got_back, want_back):
        assert torch.equal(g, w)
    # out of range: a destination row past the buffer, a buffer index past the table
    before = [g.clone() for g in got]
    nat.moe_ep_copy_runs(sends[0], dst_base=base, dst_rows=rows,
                         runs=[(0, 0, int(rows[0]) - 1, 2), (0, world, 0, 1)], ws=ws)
    assert nat.moe_check_status(ws) == nat.MOE_ERR_INVALID_INPUT
    assert torch.equal(got[0][:-1], before[0][:-1])      # only the in-range row was written
    assert torch.equal(got[0][-1], sends[0][0])


def _p2p_worker(rank, world, port, case, out_dir):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      MOE_B200_GEMM_PATH="1sm")             # one GEMM kernel on both sides
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        from mixture_experts_layer_50_b200.ep import EPMoELayer
        name, N, d, E, F, k, cf, sizes = case
        shape = W.PRESETS[name].replace(N=N, d=d, E=E, F=F, k=k)
        t = W.make_inputs(shape, device="cuda")             # the same seed on every rank
        starts = np.r_[0, np.cumsum(sizes)]
        x = t["x"][starts[rank]:starts[rank + 1]].contiguous()
        mod = t.get("modality")
        mod = None if mod is None else mod[starts[rank]:starts[rank + 1]].contiguous()
        layer = EPMoELayer.from_full_weights(
            W_g=t["W_g"], W_gu=t["W_gu"], W_down=t["W_down"], k=k, E=E, world=world, rank=rank,
            n_shared=shape.n_shared, score_fn=shape.score_fn, renorm=shape.renorm,
            act=shape.act, clamp=shape.clamp, bias=t.get("bias"),
            logit_offset=t.get("logit_offset"), capacity_factor=cf,
            max_tokens=int(max(sizes)), transport="p2p")
        ys = []
        for _ in range(2):                                    # the buffers are reused
            ys.append(layer.forward(x, modality=mod).clone())
        torch.cuda.synchronize()
        assert layer.check_status() == 0
        n = x.shape[0]
        torch.save(dict(y=[v.cpu() for v in ys], ids=layer.ids[:n].cpu(),
                        gates=layer.gates[:n].cpu(), drop=layer.drop_mask[:n].cpu()),
                   os.path.join(out_dir, f"rank{rank}.pt"))
        dist.barrier()
        layer.close()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [
    ("capacity-cf1", 600, 256, 16, 256, 2, 1, (350, 250)),
    ("v41flash-n64", 700, 512, 30, 256, 3, 1.25, (200, 0, 500)),
])
def test_peer_transport_between_processes_equals_the_single_device_layer(case, tmp_path,
                                                                        monkeypatch):
    """Ranks as separate processes sharing the GPU: each maps the others' buffers with CUDA
    IPC, its dispatch passes write its rows into the owners' receive buffers and its combine
    reads the outputs from the owners' output buffers (no message passing for the rows; host
    barriers between the phases, no kernel waiting on another).  Every rank's output, on
    two consecutive calls, equals bit for bit the fused layer over the concatenated batch given
    the ranks' routing, and the drop masks equal the oracle's for it."""
    import torch.multiprocessing as tmp
    name, N, d, E, F, k, cf, sizes = case
    world = len(sizes)
    ctx = tmp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_p2p_worker, args=(r, world, port, case, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    monkeypatch.setenv("MOE_B200_GEMM_PATH", "1sm")
    shape = W.PRESETS[name].replace(N=N, d=d, E=E, F=F, k=k)
    t = W.make_inputs(shape, device="cuda")
    ids = torch.cat([r["ids"] for r in res]).cuda()
    gates = torch.cat([r["gates"] for r in res]).cuda()
    drop = torch.cat([r["drop"] for r in res])
    C = O.capacity(N, k, E, cf)
    cfg = nat.config_from_shape(shape, capacity=C)
    ws = nat.alloc_workspace(cfg)
    y = torch.empty_like(t["x"])
    ro = dict(drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"))
    nat.moe_forward_routed(cfg, x=t["x"], ids=ids, gates=gates, W_gu=t["W_gu"],
                           W_down=t["W_down"], y=y, route_out=ro, ws=ws)
    check_status(ws)
    assert torch.equal(drop, ro["drop_mask"].cpu())
    np.testing.assert_array_equal(drop.numpy(), O.dispatch(host(ids), E, C)["drop_mask"])
    for call in range(2):
        y_ep = torch.cat([r["y"][call] for r in res]).cuda()
        assert torch.equal(y_ep, y), call


@pytest.mark.parametrize("world,case,sizes", [
    (2, CASES[0], None), (3, CASES[2], None), (4, CASES[1], None),
    # ranks of at most 64 tokens: the one-launch dispatch
    (2, ("mixtral-n16", 64, 256, 8, 384, 2, None), (40, 24)),
    # 10000+ tokens a rank: the warp-per-token scatter
    (2, ("switch-cf1", 21000, 128, 12, 128, 2, 1.25), (10000, 11000)),
])
def test_dispatch_passes_writing_into_the_owners_buffers(world, case, sizes):
    """moe_permute_ep_p2p: the dispatch passes write each kept row straight into its owner's
    receive buffer (per-expert destinations from every rank's plan; local buffers here, one per
    emulated rank).  Receive buffers, slot rows, counts and drop masks equal moe_permute_ep
    followed by the message exchange, bit for bit; a destination too small is reported."""
    from mixture_experts_layer_50_b200.ep import all_plans
    name, N, d, E, F, k, cf = case
    shape = W.PRESETS[name].replace(N=N, d=d, E=E, F=F, k=k)
    t = W.make_inputs(shape, device="cuda")
    if sizes is None:
        sizes = _split(N, world, seed=world * 7 + E)
    sizes = np.asarray(sizes)
    starts = np.r_[0, np.cumsum(sizes)]
    xs = [t["x"][starts[r]:starts[r + 1]] for r in range(world)]
    mod = t.get("modality")
    mods = [None if mod is None else mod[starts[r]:starts[r + 1]] for r in range(world)]
    layers = _layers(shape, t, world, int(sizes.max()), cf)
    dem = [L.route(x, m) for L, x, m in zip(layers, xs, mods)]
    gathered = torch.stack(dem).cpu()
    plans = [L.set_plan(gathered) for L in layers]
    # the reference: send buffers and the message exchange
    sends = [L.permute(x) for L, x in zip(layers, xs)]
    want = [L.new_recv_buffer().zero_() for L in layers]
    loopback_exchange(sends, want, [p["sends"] for p in plans], [p["recvs"] for p in plans])
    ref = [dict(slot=L.slot_row[:L.N].clone(), counts=L.counts.clone(),
                drop=L.drop_mask[:L.N].clone()) for L in layers]
    # the dispatch passes writing into the owners' buffers
    got = [torch.zeros_like(w) for w in want]
    addr = [g.data_ptr() for g in got]
    nrows = [g.shape[0] for g in got]
    for r, L in enumerate(layers):
        base, row0, rows = [addr[r]] * E, [0] * E, [0] * E
        for peer, e, _, n in plans[r]["sends"]:
            dst = {(p_, ex): rr for p_, ex, rr, _ in plans[peer]["recvs"]}
            base[e], row0[e], rows[e] = addr[peer], dst[(r, e)], nrows[peer]
        if L.N == 0:
            continue
        L.slot_row.fill_(-7)
        nat.moe_permute_ep_p2p(
            L.config(L.N), ids=L.ids[:L.N], cap=L.cap, x=xs[r], offsets=L.offsets,
            slot_row=L.slot_row[:L.N],
            dst_base=torch.tensor(base, dtype=torch.int64, device="cuda"),
            dst_row0=torch.tensor(row0, dtype=torch.int32, device="cuda"),
            dst_rows=torch.tensor(rows, dtype=torch.int64, device="cuda"),
            counts=L.counts, drop_mask=L.drop_mask[:L.N], ws=L.ws)
        check_status(L.ws)
        assert torch.equal(L.slot_row[:L.N], ref[r]["slot"])
        assert torch.equal(L.counts, ref[r]["counts"])
        assert torch.equal(L.drop_mask[:L.N], ref[r]["drop"])
    for g, w in zip(got, want):
        assert torch.equal(g, w)
    # a destination one row too small: that row is skipped and reported
    r = next(i for i, L in enumerate(layers) if plans[i]["sends"])
    L = layers[r]
    peer, e, _, n = plans[r]["sends"][-1]
    dst = {(p_, ex): rr for p_, ex, rr, _ in plans[peer]["recvs"]}
    base, row0, rows = [addr[r]] * E, [0] * E, [0] * E
    for pp, ee, _, nn in plans[r]["sends"]:
        dd = {(p_, ex): rr for p_, ex, rr, _ in plans[pp]["recvs"]}
        base[ee], row0[ee], rows[ee] = addr[pp], dd[(r, ee)], nrows[pp]
    rows[e] = dst[(r, e)] + n - 1
    nat.moe_permute_ep_p2p(
        L.config(L.N), ids=L.ids[:L.N], cap=L.cap, x=xs[r], offsets=L.offsets,
        slot_row=L.slot_row[:L.N], dst_base=torch.tensor(base, dtype=torch.int64, device="cuda"),
        dst_row0=torch.tensor(row0, dtype=torch.int32, device="cuda"),
        dst_rows=torch.tensor(rows, dtype=torch.int64, device="cuda"), ws=L.ws)
    assert nat.moe_check_status(L.ws) == nat.MOE_ERR_INVALID_INPUT


@pytest.mark.parametrize("world,case,sizes", [
    (2, CASES[0], None), (3, CASES[2], None), (4, CASES[1], None), (2, CASES[3], None),
    # k = 8 and k = 12: the block-per-token kernel's 8-slot and any-k forms
    (2, ("dsv3-n64", 400, 256, 32, 128, 8, None), None),
    (3, ("dsv3-n64", 300, 256, 48, 128, 12, 1.25), None),
    # 10000+ tokens a rank, 256-byte rows: the warp-per-token kernel (2 and 8 slots)
    (2, ("switch-cf1", 21000, 128, 12, 128, 2, 1.25), (10000, 11000)),
    (2, ("switch-cf1", 21000, 128, 16, 128, 8, 1.25), (11000, 10000)),
])
def test_combine_reading_the_owners_outputs(world, case, sizes):
    """moe_ep_combine_p2p: each rank's combine reads its slots' expert outputs where their
    owners wrote them (per-expert sources from every rank's plan; local buffers here, one per
    emulated rank), with no return trip.  y equals, bit for bit, the return exchange followed
    by moe_ep_combine; a source one row too small drops that slot alone and is reported."""
    from mixture_experts_layer_50_b200.ep import loopback_exchange
    name, N, d, E, F, k, cf = case
    shape = W.PRESETS[name].replace(N=N, d=d, E=E, F=F, k=k)
    t = W.make_inputs(shape, device="cuda")
    if sizes is None:
        sizes = _split(N, world, seed=world * 13 + E)
    sizes = np.asarray(sizes)
    starts = np.r_[0, np.cumsum(sizes)]
    xs = [t["x"][starts[r]:starts[r + 1]] for r in range(world)]
    mod = t.get("modality")
    mods = [None if mod is None else mod[starts[r]:starts[r + 1]] for r in range(world)]
    layers = _layers(shape, t, world, int(sizes.max()), cf)
    dem = [L.route(x, m) for L, x, m in zip(layers, xs, mods)]
    gathered = torch.stack(dem).cpu()
    plans = [L.set_plan(gathered) for L in layers]
    sends = [L.permute(x) for L, x in zip(layers, xs)]
    recv = [L.new_recv_buffer() for L in layers]
    loopback_exchange(sends, recv, [p["sends"] for p in plans], [p["recvs"] for p in plans])
    shared = [torch.empty_like(x) for x in xs]
    outs = [L.run_experts(r, x, y) for L, r, x, y in zip(layers, recv, xs, shared)]
    # the reference: the return exchange and the local combine
    back = [L.new_return_buffer() for L in layers]
    loopback_exchange(outs, back, [p["recvs"] for p in plans], [p["sends"] for p in plans])
    want = [L.combine(b, s.clone()) for L, b, s in zip(layers, back, shared)]
    addr = [o.data_ptr() for o in outs]
    nrows = [o.shape[0] for o in outs]

    def tables(r):
        base, row0, rows = [addr[r]] * E, [0] * E, [0] * E
        for peer, e, _, n in plans[r]["sends"]:
            dst = {(p_, ex): rr for p_, ex, rr, _ in plans[peer]["recvs"]}
            base[e], row0[e], rows[e] = addr[peer], dst[(r, e)], nrows[peer]
        return base, row0, rows

    def combine_p2p(L, y, base, row0, rows):
        nat.moe_ep_combine_p2p(
            L.config(L.N), ids=L.ids[:L.N], slot_row=L.slot_row[:L.N], gates=L.gates[:L.N],
            offsets=L.offsets, src_base=torch.tensor(base, dtype=torch.int64, device="cuda"),
            src_row0=torch.tensor(row0, dtype=torch.int32, device="cuda"),
            src_rows=torch.tensor(rows, dtype=torch.int64, device="cuda"), y=y, ws=L.ws)

    for r, L in enumerate(layers):
        if L.N == 0:
            continue
        y = shared[r].clone()
        combine_p2p(L, y, *tables(r))
        check_status(L.ws)
        assert torch.equal(y, want[r]), r
    # a source one row too small: the slot of that last row contributes nothing
    r = next(i for i, L in enumerate(layers) if plans[i]["sends"] and L.N > 0)
    L = layers[r]
    peer, e, _, n = plans[r]["sends"][-1]
    base, row0, rows = tables(r)
    rows[e] = row0[e] + n - 1
    last = int(L.offsets[e].item()) + n - 1               # the send-layout row of that slot
    slot = (L.slot_row[:L.N] == last).nonzero()
    assert slot.shape[0] == 1
    tok, j = int(slot[0, 0]), int(slot[0, 1])
    y = shared[r].clone()
    combine_p2p(L, y, base, row0, rows)
    assert nat.moe_check_status(L.ws) == nat.MOE_ERR_INVALID_INPUT
    others = torch.ones(L.N, dtype=torch.bool, device="cuda")
    others[tok] = False
    assert torch.equal(y[others], want[r][others])
    # that token: the combine of its other slots alone
    sr = L.slot_row[:L.N].clone()
    sr[tok, j] = -1
    y1 = shared[r].clone()
    nat.moe_ep_combine(L.config(L.N), ye=back[r], slot_row=sr, gates=L.gates[:L.N], y=y1)
    assert torch.equal(y[tok], y1[tok])
