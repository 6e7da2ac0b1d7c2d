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


def test_traffic_is_read_only_for_the_measured_kernel_source(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu summary of the workload, and only while
    the kernel source still hashes to the one the counters were taken on."""
    import hashlib
    import bench
    src = os.path.join(bench.ROOT, "mixture_experts_layer_50_b200", "csrc", "gemm_tc.cu")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (tmp_path / "mixture_experts_layer_50_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "mixture_experts_layer_50_b200" / "csrc" / "gemm_tc.cu").write_bytes(open(src, "rb").read())
    (prof / "gemm_gate_up_mixtral_n16384.md").write_text(
        f"x\ntraffic_bytes_per_launch: 3.1e9\nkernel_source_sha256: {digest}\n")
    (prof / "gemm_gate_up_mixtral_n4096.md").write_text(
        "traffic_bytes_per_launch: 2.0e9\nkernel_source_sha256: 00\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_traffic("gemm_gate_up", "mixtral-n16384") == 3.1e9
    assert bench.read_traffic("gemm_gate_up", "mixtral-n4096") is None    # stale counters
    assert bench.read_traffic("gemm_gate_up", "dsv3-n8192") is None       # no capture


def test_algorithmic_work_of_the_roofline():
    """F_alg and B_alg behind roofline and layer_roofline, against the closed forms:
    F = 2 (M + S N) 3 d F + 2 N d E and B = touched experts' weights + router + x and y."""
    import numpy as np
    import bench
    from mixture_experts_layer_50_b200 import workloads as W
    s = W.PRESETS["mixtral-n16384"]
    w = bench.algorithmic_work(s, np.full(8, 4096))
    assert w["M"] == 32768 and w["touched"] == 8
    assert w["flops_layer"] == 2 * 32768 * 3 * 4096 * 14336 + 2 * 16384 * 4096 * 8
    assert w["flops_gate_up"] == 2 * 32768 * 4096 * 2 * 14336
    assert w["bytes_layer"] == 2 * (8 * 3 * 4096 * 14336 + 8 * 4096 + 2 * 16384 * 4096)
    # the gate/up launch: W_gate|W_up of the touched experts, x rows in, h rows out
    assert w["bytes_gate_up"] == 2 * (8 * 2 * 14336 * 4096 + 32768 * 4096 + 32768 * 14336)
    # decode: 16 tokens touch 7 experts; the shared expert of a V3-shaped layer counts in
    w = bench.algorithmic_work(s.replace(N=16), np.array([5, 4, 6, 3, 5, 4, 5, 0]))
    assert w["touched"] == 7
    assert w["bytes_layer"] == 2 * (7 * 3 * 4096 * 14336 + 8 * 4096 + 2 * 16 * 4096)
    v3 = W.PRESETS["dsv3-n64"]
    counts = np.zeros(256, np.int64)
    counts[:200] = 2
    counts[200:256:4] = 1
    w = bench.algorithmic_work(v3, counts)
    rows = int(counts.sum()) + 64
    assert w["flops_gate_up"] == 2 * rows * 7168 * 2 * 2048
    assert w["bytes_layer"] == 2 * ((w["touched"] + 1) * 3 * 7168 * 2048 + 256 * 7168 + 2 * 64 * 7168)


def test_settle_power_waits_for_the_power_reading_with_a_fake_nvml(monkeypatch):
    """The sweep's settle step reads NVML only (no setting is changed): it waits while the
    board's power reading is at or above half its limit, returns once it falls below, gives up
    after its time limit, and returns at once when NVML is unavailable."""
    import sys
    import types
    import bench

    class FakeNvml(types.ModuleType):
        def __init__(self, readings_mw, limit_mw=1_000_000):
            super().__init__("pynvml")
            self.readings = list(readings_mw)
            self.limit = limit_mw
            self.calls = 0

        def nvmlInit(self):
            pass

        def nvmlDeviceGetHandleByIndex(self, i):
            return i

        def nvmlDeviceGetEnforcedPowerLimit(self, h):
            return self.limit

        def nvmlDeviceGetPowerUsage(self, h):
            self.calls += 1
            return self.readings[min(self.calls - 1, len(self.readings) - 1)]

    monkeypatch.setattr(bench.time, "sleep", lambda s: None)
    fake = FakeNvml([900_000, 700_000, 600_000, 400_000])    # 900 W ... 400 W, limit 1 kW
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    bench.settle_power(0, limit_s=5.0)
    assert fake.calls == 4                                   # stopped at the first reading < 500 W
    fake = FakeNvml([900_000])                                # never settles
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    waited = bench.settle_power(0, limit_s=0.05)
    assert 0.05 <= waited < 1.0 and fake.calls > 1
    broken = types.ModuleType("pynvml")                       # no NVML entry points
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    assert bench.settle_power(0) < 0.5
