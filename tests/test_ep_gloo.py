"""Expert-parallel exchange on CPU ranks (gloo, world size 2 and 3) against the oracle's
single-device layer over the concatenated batch.

The plan (``moe_ep_plan``, host C) and the row exchange (``exchange_rows``, torch.distributed
grouped point-to-point) are the library's own; the per-rank arithmetic (routing, the layout of
the kept rows, the expert FFNs and the combine) is the oracle's, in float64, so that this test
runs without a GPU.  "Mixture-of-Experts : routage et capacité" slides, "L'idée —
Communication": rows go to their expert's device and the outputs come back.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer(seed, N, d, E, F, k, S):
    rng = np.random.default_rng(seed)
    x = rng.normal(0, 1, (N, d))
    W_g = rng.normal(0, 0.3, (E, d))
    W_gu = rng.normal(0, 0.2, (E + S, 2 * F, d))
    W_down = rng.normal(0, 0.2, (E + S, d, F))
    return x, W_g, W_gu, W_down


def _worker(rank, world, port, case, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as O
        from mixture_experts_layer_50_b200 import _native as nat
        from mixture_experts_layer_50_b200.ep import exchange_rows
        seed, N, d, E, F, k, S, cf, sizes = case
        x, W_g, W_gu, W_down = _layer(seed, N, d, E, F, k, S)
        starts = np.r_[0, np.cumsum(sizes)]
        mine = slice(starts[rank], starts[rank + 1])
        xr_ = x[mine]
        # this rank's routing (oracle) and its demand, all-gathered with the token count
        z = O.router_logits(xr_, W_g)
        ids, gates = O.route(z, k)
        dem = np.r_[np.bincount(ids.ravel(), minlength=E), len(xr_)].astype(np.int32)
        g = torch.empty(world * (E + 1), dtype=torch.int32)
        dist.all_gather_into_tensor(g, torch.from_numpy(dem))
        g = g.numpy().reshape(world, E + 1)
        C = O.capacity(int(g[:, E].sum()), k, E, cf)
        plan = nat.moe_ep_plan(world, rank, E, C, g[:, :E])
        # this rank's kept rows under its per-expert capacity, in the send layout
        loc = O.dispatch(ids, E, 0)
        rank_in = loc["slot_row"] - loc["offsets"][ids]
        drop = rank_in >= plan["cap"][ids]
        lay = O.dispatch_masked(ids, E, drop)
        xp = torch.from_numpy(np.ascontiguousarray(xr_[lay["row_token"]]))
        assert xp.shape[0] == plan["rows_kept"]
        recv = torch.zeros((plan["rows_owned"], d), dtype=torch.float64)
        exchange_rows(xp, recv, plan["sends"], plan["recvs"], rank)
        # the owner's experts on the received groups
        e0 = plan["first_expert"]
        off = plan["owned_offsets"]
        ye = torch.zeros_like(recv)
        for i in range(plan["n_owned"]):
            a, b = int(off[i]), int(off[i + 1])
            if b > a:
                ye[a:b] = torch.from_numpy(O.expert_ffn(recv[a:b].numpy(), W_gu[e0 + i],
                                                        W_down[e0 + i]))
        back = torch.zeros((plan["rows_kept"], d), dtype=torch.float64)
        exchange_rows(ye, back, plan["recvs"], plan["sends"], rank)
        y = np.zeros_like(xr_)
        for t in range(len(xr_)):
            for j in range(k):
                r = lay["slot_row"][t, j]
                if r >= 0:
                    y[t] += gates[t, j] * back[r].numpy()
        for s in range(S):
            y += O.expert_ffn(xr_, W_gu[E + s], W_down[E + s])
        q.put((rank, y, drop.astype(np.uint8), plan["kept_all"]))
    except Exception as exc:  # report instead of hanging the other rank's test
        q.put((rank, repr(exc), None, None))
        raise
    finally:
        dist.destroy_process_group()


CASES = [
    # seed, N, d, E, F, k, S, cf, sizes per rank
    (1, 96, 16, 6, 8, 2, 1, 1, (40, 56)),
    (2, 120, 8, 7, 4, 3, 0, 1.25, (0, 70, 50)),        # a rank without tokens
    (3, 64, 8, 4, 4, 2, 1, None, (30, 34)),            # no capacity
    (4, 90, 8, 9, 4, 1, 1, 0.5, (45, 20, 25)),         # Switch-like k = 1, heavy dropping
]


@pytest.mark.parametrize("case", CASES)
def test_expert_parallel_exchange_equals_single_device_layer(case):
    import oracle as O
    seed, N, d, E, F, k, S, cf, sizes = case
    world = len(sizes)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in procs:
        rank, y, drop, kept = q.get(timeout=180)
        assert drop is not None, f"rank {rank} failed: {y}"
        out[rank] = (y, drop, kept)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, W_g, W_gu, W_down = _layer(seed, N, d, E, F, k, S)
    C = O.capacity(N, k, E, cf)
    y_ref, info = O.forward(x, W_g, W_gu, W_down, k=k, E=E, n_shared=S, C=C)
    starts = np.r_[0, np.cumsum(sizes)]
    for r in range(world):
        y, drop, kept = out[r]
        mine = slice(starts[r], starts[r + 1])
        np.testing.assert_array_equal(drop, info["drop_mask"][mine])
        np.testing.assert_allclose(y, y_ref[mine], rtol=1e-12, atol=1e-12)
        assert kept.sum() == int(info["counts"].sum())
