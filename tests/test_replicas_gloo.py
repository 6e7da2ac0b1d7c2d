"""Multi-rank host logic of bench.py on CPU ranks (gloo, world size 2): every rank runs an
independent replica (same weights, own tokens), timing is the max over ranks, and the
reported value aggregates the tokens of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from mixture_experts_layer_50_b200 import workloads as W
        shape = W.PRESETS["v41flash-n64"].replace(N=32, d=64, F=64, E=8, k=2)
        t = bench.make_replica(shape, rank, device="cpu")
        mx = bench.max_over_ranks(10.0 + rank, world, device="cpu")
        gathered = [None] * world
        dist.all_gather_object(gathered, (t["W_gu"].float().sum().item(), t["x"].float().sum().item()))
        q.put((rank, mx, gathered))
    finally:
        dist.destroy_process_group()


def test_two_cpu_ranks_replicas_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, gathered in out:
        assert mx == 11.0                                   # the slowest rank's time
        (w0, x0), (w1, x1) = gathered
        assert w0 == w1                                     # same layer weights
        assert x0 != x1                                     # own tokens per replica


def test_aggregate_value():
    import bench
    assert bench.aggregate_tokens_per_s(16384, 4, 10.0) == pytest.approx(16384 * 4 / 0.01)
