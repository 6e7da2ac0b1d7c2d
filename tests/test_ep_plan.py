"""The expert-parallel plan (host C, no GPU) against the oracle's single-device dispatch.

"Mixture-of-Experts : routage et capacité" slides, "L'idée — Communication": experts live on
different devices and rows travel to their expert's device and back.  The plan must make the
ranks together keep exactly the assignments the single-device layer keeps on the concatenated
batch (capacity in token order, "L'idée — Capacité"), and lay every owner's receive buffer out
as that layer's groups.
"""
import numpy as np
import pytest

import oracle as O
from mixture_experts_layer_50_b200 import _native as nat


def _split(N, world, rng):
    cuts = np.sort(rng.integers(0, N + 1, world - 1))
    return np.diff(np.r_[0, cuts, N]).astype(int)


def _case(seed, world, N, E, k, cf, quantum=0.0):
    rng = np.random.default_rng(seed)
    z = rng.normal(0, 1, (N, E)).astype(np.float32)
    if quantum:
        z = (np.round(z / quantum) * quantum).astype(np.float32)
    z[:, 0] += 1.0                                        # a hot expert, so capacity bites
    ids, _ = O.route(z, k)
    C = O.capacity(N, k, E, cf)
    sizes = _split(N, world, rng)
    starts = np.r_[0, np.cumsum(sizes)]
    demand = np.stack([np.bincount(ids[starts[r]:starts[r + 1]].ravel(), minlength=E)
                       for r in range(world)]).astype(np.int32)
    return ids, C, sizes, starts, demand


@pytest.mark.parametrize("seed,world,N,E,k,cf", [
    (0, 2, 300, 8, 2, 1), (1, 3, 500, 7, 2, 1.25), (2, 4, 257, 16, 4, None),
    (3, 1, 100, 4, 1, 0.5), (4, 5, 999, 5, 3, 1), (5, 8, 64, 64, 8, 2), (6, 3, 40, 3, 3, 1)])
def test_plan_keeps_what_the_single_device_layer_keeps(seed, world, N, E, k, cf):
    ids, C, sizes, starts, demand = _case(seed, world, N, E, k, cf)
    ref = O.dispatch(ids, E, C)
    keep = ref["drop_mask"] == 0
    plans = [nat.moe_ep_plan(world, r, E, C, demand) for r in range(world)]
    for r, p in enumerate(plans):
        tr = slice(starts[r], starts[r + 1])
        want = np.zeros(E, np.int64)
        np.add.at(want, ids[tr][keep[tr]], 1)
        np.testing.assert_array_equal(p["kept_all"][r], want)
        np.testing.assert_array_equal(p["kept_all"], plans[0]["kept_all"])
        # the per-expert capacity reproduces the drop mask in the rank's own token order
        loc = O.dispatch(ids[tr], E, 0)                      # ranks among this rank's tokens
        rank_in = loc["slot_row"] - loc["offsets"][ids[tr]]
        np.testing.assert_array_equal(rank_in < p["cap"][ids[tr]], keep[tr])
        assert p["rows_kept"] == int(want.sum())
        # sends: this rank's compact layout, each expert's run to its owner
        e0 = nat.moe_ep_first_expert(world, r, E)
        assert p["first_expert"] == e0
        lay = O.dispatch_masked(ids[tr], E, ~keep[tr])
        runs = {e: (row, rows) for _, e, row, rows in p["sends"]}
        for e in range(E):
            c = int(lay["counts"][e])
            if c == 0:
                assert e not in runs
            else:
                assert runs[e] == (int(lay["offsets"][e]), c)
        for peer, e, _, _ in p["sends"]:
            assert nat.moe_ep_first_expert(world, peer, E) <= e < nat.moe_ep_first_expert(world, peer + 1, E)


@pytest.mark.parametrize("seed,world,N,E,k,cf", [
    (10, 2, 300, 8, 2, 1), (11, 3, 501, 10, 3, None), (12, 4, 128, 9, 2, 1.25), (13, 2, 50, 2, 2, 1)])
def test_owner_buffers_are_the_single_device_groups(seed, world, N, E, k, cf):
    """Concatenating the received runs of an owner gives, expert by expert, exactly the global
    token list of the single-device layout (row_token of the oracle's dispatch)."""
    ids, C, sizes, starts, demand = _case(seed, world, N, E, k, cf)
    ref = O.dispatch(ids, E, C)
    plans = [nat.moe_ep_plan(world, r, E, C, demand) for r in range(world)]
    # every rank's send layout in global token ids
    sent_tokens = []
    for r in range(world):
        tr = slice(starts[r], starts[r + 1])
        keep = ref["drop_mask"][tr] == 0
        lay = O.dispatch_masked(ids[tr], E, ~keep)
        sent_tokens.append(lay["row_token"] + starts[r])
    for o, p in enumerate(plans):
        e0, e1 = p["first_expert"], p["first_expert"] + p["n_owned"]
        recv = np.full(p["rows_owned"], -1, np.int64)
        for peer, e, row, rows in p["recvs"]:
            src = [c for c in plans[peer]["sends"] if c[0] == o and c[1] == e]
            assert len(src) == 1 and src[0][3] == rows
            recv[row:row + rows] = sent_tokens[peer][src[0][2]:src[0][2] + rows]
        want = ref["row_token"][ref["offsets"][e0]:ref["offsets"][e1]]
        np.testing.assert_array_equal(recv, want)
        np.testing.assert_array_equal(p["owned_offsets"],
                                      ref["offsets"][e0:e1 + 1] - ref["offsets"][e0])
    # every send run has exactly one receive run, same size, in the same per-peer order
    for r, p in enumerate(plans):
        for peer in range(world):
            out = [(e, rows) for q, e, _, rows in p["sends"] if q == peer]
            inn = [(e, rows) for q, e, _, rows in plans[peer]["recvs"] if q == r]
            assert out == inn


def test_plan_without_capacity_keeps_everything_and_edges():
    demand = np.array([[3, 0, 1], [0, 0, 0], [2, 5, 0]], np.int32)
    for r in range(3):
        p = nat.moe_ep_plan(3, r, 3, 0, demand)
        np.testing.assert_array_equal(p["kept_all"], demand)
        assert (p["cap"] == np.iinfo(np.int32).max).all()
        assert p["n_owned"] == 1
    # an idle rank sends nothing but still owns and receives
    p1 = nat.moe_ep_plan(3, 1, 3, 0, demand)
    assert p1["sends"] == [] and p1["rows_kept"] == 0
    assert [(q, e, rows) for q, e, _, rows in p1["recvs"]] == [(2, 1, 5)]
    # capacity below what rank 0 alone asks for: the later ranks keep nothing of that expert
    p2 = nat.moe_ep_plan(3, 2, 3, 2, demand)
    np.testing.assert_array_equal(p2["kept_all"], [[2, 0, 1], [0, 0, 0], [0, 2, 0]])
    np.testing.assert_array_equal(p2["cap"], [0, 2, 1])


def test_ownership_is_contiguous_and_covers_every_expert():
    for world, E in ((1, 5), (2, 5), (3, 7), (8, 384), (8, 8), (5, 1024)):
        firsts = [nat.moe_ep_first_expert(world, r, E) for r in range(world + 1)]
        assert firsts[0] == 0 and firsts[-1] == E
        sizes = np.diff(firsts)
        assert sizes.min() >= 1 and sizes.max() - sizes.min() <= 1


def test_plan_rejects_bad_arguments():
    d = np.zeros((2, 4), np.int32)
    with pytest.raises(nat.MoeError):
        nat.moe_ep_plan(2, 2, 4, 0, d)                      # rank out of range
    with pytest.raises(nat.MoeError):
        nat.moe_ep_plan(5, 0, 4, 0, np.zeros((5, 4), np.int32))   # more ranks than experts
    with pytest.raises(nat.MoeError):
        nat.moe_ep_plan(2, 0, 4, 0, np.array([[1, -1, 0, 0], [0, 0, 0, 0]], np.int32))
    assert nat.lib.moe_ep_first_expert(0, 0, 4) == -1


@pytest.mark.parametrize("seed,world,N,E,k,cf", [
    (0, 2, 300, 8, 2, 1), (1, 3, 500, 7, 2, 1.25), (2, 4, 257, 16, 4, None), (5, 8, 64, 64, 8, 2)])
def test_peer_runs_move_the_rows_the_message_exchange_moves(seed, world, N, E, k, cf):
    """The peer-memory transport's runs (each rank writes its rows straight into the peers'
    buffers): applied to tagged rows, in both directions, they leave every buffer exactly as
    the message exchange (``loopback_exchange``) does."""
    import torch
    from mixture_experts_layer_50_b200.ep import all_plans, loopback_exchange, peer_runs
    ids, C, sizes, starts, demand = _case(seed, world, N, E, k, cf)
    plans = all_plans(world, E, C, demand)
    rows = lambda n: max(1, n)
    sends = [torch.arange(rows(p["rows_kept"]) * 2, dtype=torch.float64).reshape(-1, 2) + 1000 * r
             for r, p in enumerate(plans)]
    # dispatch: send buffers -> owners' receive buffers
    want = [torch.full((rows(p["rows_owned"]), 2), -1.0, dtype=torch.float64) for p in plans]
    loopback_exchange(sends, want, [p["sends"] for p in plans], [p["recvs"] for p in plans])
    got = [torch.full_like(w, -1.0) for w in want]
    for r in range(world):
        for src_row, dst, dst_row, n in peer_runs(r, plans, "dispatch"):
            got[dst][dst_row:dst_row + n] = sends[r][src_row:src_row + n]
    for g, w in zip(got, want):
        assert torch.equal(g, w)
    # return: receive buffers (the expert outputs) -> the sources' return buffers
    outs = [w + 0.5 for w in want]
    want_back = [torch.full_like(s, -1.0) for s in sends]
    loopback_exchange(outs, want_back, [p["recvs"] for p in plans], [p["sends"] for p in plans])
    got_back = [torch.full_like(s, -1.0) for s in sends]
    for r in range(world):
        for src_row, dst, dst_row, n in peer_runs(r, plans, "return"):
            got_back[dst][dst_row:dst_row + n] = outs[r][src_row:src_row + n]
    for g, w in zip(got_back, want_back):
        assert torch.equal(g, w)
    kept = sum(p["rows_kept"] for p in plans)
    assert sum(n for r in range(world) for *_, n in peer_runs(r, plans, "dispatch")) == kept


@pytest.mark.parametrize("seed,world,N,E,k,cf", [
    (0, 2, 300, 8, 2, 1), (1, 3, 500, 7, 2, 1.25), (2, 4, 257, 16, 4, None), (5, 8, 64, 64, 8, 2)])
def test_expert_tables_address_the_rows_the_message_exchange_moves(seed, world, N, E, k, cf):
    """The per-expert tables of the fused peer-memory dispatch and combine (kept row i of
    expert e goes to, and its output comes back from, row row0[e] + i of the owner's buffers):
    writing every rank's tagged send rows through them leaves each owner's receive buffer as
    the message exchange does, and reading the owners' outputs through them gives each rank
    what the return exchange gives."""
    import torch
    from mixture_experts_layer_50_b200.ep import all_plans, expert_tables, loopback_exchange
    ids, C, sizes, starts, demand = _case(seed, world, N, E, k, cf)
    plans = all_plans(world, E, C, demand)
    rows = lambda n: max(1, n)
    sends = [torch.arange(rows(p["rows_kept"]) * 2, dtype=torch.float64).reshape(-1, 2) + 1000 * r
             for r, p in enumerate(plans)]
    want = [torch.full((rows(p["rows_owned"]), 2), -1.0, dtype=torch.float64) for p in plans]
    loopback_exchange(sends, want, [p["sends"] for p in plans], [p["recvs"] for p in plans])
    outs = [w + 0.5 for w in want]
    want_back = [torch.full_like(s, -1.0) for s in sends]
    loopback_exchange(outs, want_back, [p["recvs"] for p in plans], [p["sends"] for p in plans])
    # the buffers' "addresses" are rank numbers here
    ranks = list(range(world))
    sizes_owned = [w.shape[0] for w in want]
    got = [torch.full_like(w, -1.0) for w in want]
    for r in range(world):
        recv, out, row0, size = expert_tables(r, plans, E, ranks, ranks, sizes_owned)
        back = torch.full_like(sends[r], -1.0)
        for peer, e, row, n in plans[r]["sends"]:
            assert recv[e] == out[e] == peer and size[e] == sizes_owned[peer]
            assert 0 <= row0[e] and row0[e] + n <= size[e]
            got[peer][row0[e]:row0[e] + n] = sends[r][row:row + n]
            back[row:row + n] = outs[peer][row0[e]:row0[e] + n]
        assert torch.equal(back, want_back[r])
    for g, w in zip(got, want):
        assert torch.equal(g, w)
