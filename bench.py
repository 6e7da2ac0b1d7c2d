#!/usr/bin/env python
"""Throughput of the MoE FFN layer forward pass on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one ``moe_forward`` over one batch of tokens (router GEMM, top-k, capacity and
permutation, gate/up and down grouped GEMMs with the shared expert, combine).  Default
workload: the Mixtral-shaped layer (d=4096, 8 SwiGLU experts of d_ff=14336, top-2) at
16384 tokens.  With N > 1 (torchrun, one rank per GPU) each rank runs an independent replica
of the layer on its own tokens: there is no exchange on the data path.

``--impl reference`` times the CPU oracle (float64, numpy) on bounded samples of the same
workload on this machine's cores; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_50_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer fwd tokens/s and % of bf16 tensor (prefill) or HBM (decode) roofline"
LAUNCH_NAMES = ["router_gemm", "route_topk", "rank_local", "dispatch_scan", "scatter_gather",
                "gemm_gate_up", "gemm_down", "combine"]
# with the "report" overflow policy: the capacity pass, the offers and the final layout
LAUNCH_NAMES_REROUTE = ["router_gemm", "route_topk", "rank_local", "dispatch_scan",
                        "capacity_pass", "reroute_offer", "rank_offers", "scan_offers",
                        "reroute_accept", "rank_final", "scan_final", "scatter_gather",
                        "gemm_gate_up", "gemm_down", "combine"]
L2_BYTES = 128 << 20          # B200 L2: 126 MB
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="mixtral-n16384", choices=sorted(W.PRESETS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--overflow", default="drop", choices=["drop", "reroute"],
                   help="capacity overflow policy: drop, or the slides' 'report' (reroute)")
    p.add_argument("--tokens", type=int, default=None,
                   help="override the workload's token count (profiling a smaller case)")
    p.add_argument("--experts", type=int, default=None,
                   help="override the workload's routed expert count (profiling a smaller case)")
    return p.parse_args()


def workload_shape(args):
    shape = W.PRESETS[args.workload]
    if args.tokens is not None:
        shape = shape.replace(N=args.tokens)
    if args.experts is not None:
        shape = shape.replace(E=args.experts)
    return shape


# ------------------------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(shape):
    cf = shape.capacity_factor
    return (f"{shape.name}: N={shape.N} d={shape.d} E={shape.E}+{shape.n_shared} k={shape.k} "
            f"F={shape.F} {'sigmoid' if shape.score_fn else 'softmax'}"
            f"{' renorm' if shape.renorm else ' raw-gate'}"
            f"{' bias-sets=' + str(shape.n_bias_sets) if shape.n_bias_sets else ''}"
            f"{' clamp=' + str(shape.clamp) if shape.clamp > 0 else ''}"
            f"{' cf=' + str(cf) if cf is not None else ''}"
            f"{' zipf-skew' if shape.zipf_skew else ''} {'bf16' if shape.dtype == W.BF16 else 'fp32'}")


def algorithmic_work(shape, counts):
    """F_alg and B_alg of one layer call and of the gate/up launch, from the actual routing."""
    N, d, F, E, S = shape.N, shape.d, shape.F, shape.E, shape.n_shared
    el = 2 if shape.dtype == W.BF16 else 4
    gu = 2 if shape.act == W.SWIGLU else 1
    M = int(counts.sum())
    touched = int((counts > 0).sum())
    rows = M + S * N
    f_gate_up = 2.0 * rows * d * gu * F
    f_down = 2.0 * rows * F * d
    f_router = 2.0 * N * d * E
    w_gu = (touched + S) * gu * F * d * el
    w_down = (touched + S) * d * F * el
    b_layer = w_gu + w_down + E * d * el + 2 * N * d * el
    # gate/up launch: its weights, its activation rows in, its hidden rows out
    b_gate_up = w_gu + rows * d * el + rows * F * el
    return dict(M=M, touched=touched, flops_layer=f_gate_up + f_down + f_router,
                bytes_layer=b_layer, flops_gate_up=f_gate_up, bytes_gate_up=b_gate_up)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # NVML unavailable: report no clocks rather than fail the bench
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                get = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
                r = get(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def read_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if its kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload.replace('-', '_')}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_bytes = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    m_hash = re.search(r"^kernel_source_sha256:\s*([0-9a-f]+)", text, re.M)
    if not m_bytes or not m_hash:
        return None
    src = os.path.join(ROOT, "mixture_experts_layer_50_b200", "csrc", "gemm_tc.cu")
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_hash.group(1):
        return None
    return float(m_bytes.group(1))


# ------------------------------------------------------------------------------------------
def dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device="cuda"):
    """The slowest rank's time: every rank takes part in the same all-reduce."""
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank, world, ms_step_max):
    """Whole-job throughput: tokens of all ranks over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_step_max / 1e3)


def make_replica(shape, rank, device="cuda"):
    """The layer's inputs for one replica: the same weights everywhere, own tokens per rank."""
    t = W.make_inputs(shape, device=device)
    if rank > 0:
        g = torch.Generator(device=device)
        g.manual_seed(shape.seed * 1000 + rank)
        x = torch.empty(t["x"].shape, dtype=torch.float32, device=device).normal_(generator=g)
        t["x"] = x.to(t["x"].dtype)
        if "modality" in t:
            u = torch.empty(t["x"].shape[0], device=device).uniform_(generator=g)
            t["modality"] = (u < 0.3).to(torch.uint8)
    return t


def run_ours(args):
    from mixture_experts_layer_50_b200 import build as _build
    if int(os.environ.get("LOCAL_RANK", "0")) == 0:
        _build.ensure_built()
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        # the other ranks wait for the library local rank 0 builds
        lib = _build.LIB
        for _ in range(6000):
            if os.path.exists(lib):
                break
            time.sleep(0.1)
    from mixture_experts_layer_50_b200 import _native as nat
    from mixture_experts_layer_50_b200.layer import MoELayer

    world, rank, local = dist_init(args.gpus)
    torch.cuda.set_device(local)
    shape = workload_shape(args)
    t = make_replica(shape, rank)
    layer = MoELayer.from_workload(shape, t, overflow=args.overflow)
    x, mod = t["x"], t.get("modality")
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()
    names = LAUNCH_NAMES_REROUTE if args.overflow == "reroute" and shape.capacity_factor else LAUNCH_NAMES

    # routing statistics of this batch (untimed), for the algorithmic work
    counts = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    layer.forward(x, modality=mod, y=y, route_out={"counts": counts})
    assert layer.check_status() == 0
    work = algorithmic_work(shape, counts.cpu().numpy())

    for _ in range(args.warmup):
        layer.forward(x, modality=mod, y=y)
    torch.cuda.synchronize()
    per_step_launches = nat.moe_last_launch_count()
    # the step as a CUDA graph: the eight launches captured once, replayed each step
    layer.forward_graphed(x, y, modality=mod)
    for _ in range(args.warmup):
        layer.forward_graphed(x, y, modality=mod)

    # timed region: K replays of the whole layer.  A layer whose weights and tokens fit in
    # L2 (the fp32 toy) gets L2 flushed before every step (a 256 MB write) and only the
    # replays themselves are timed; every other layer streams more than L2 per step.
    l2_resident = shape.weight_bytes() + 2 * x.numel() * x.element_size() < L2_BYTES
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if l2_resident else None
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if flush is None:
            ev0.record(stream)
            h0 = time.perf_counter()
            for _ in range(args.steps):
                layer.forward_graphed(x, y, modality=mod)
            host_us = (time.perf_counter() - h0) * 1e6 / args.steps
            ev1.record(stream)
            torch.cuda.synchronize()
            timed_ms = ev0.elapsed_time(ev1)
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            h0 = time.perf_counter()
            for a, b in evs:
                flush.fill_(1)
                a.record(stream)
                layer.forward_graphed(x, y, modality=mod)
                b.record(stream)
            host_us = (time.perf_counter() - h0) * 1e6 / args.steps
            torch.cuda.synchronize()
            timed_ms = sum(a.elapsed_time(b) for a, b in evs)
    barrier(world)
    assert layer.check_status() == 0

    # the same K steps launched one kernel at a time, with a CUDA event recorded on the
    # launching stream between the kernels: the per-kernel durations behind the roofline
    barrier(world)
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    nat.moe_profile_begin(args.steps)
    p0.record(stream)
    for _ in range(args.steps):
        layer.forward(x, modality=mod, y=y)
    p1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    launch_ms, calls = nat.moe_profile_end(16)
    eager_ms = max_over_ranks(p0.elapsed_time(p1), world) / args.steps
    assert layer.check_status() == 0
    ms_total = max_over_ranks(timed_ms, world)
    ms_step = ms_total / args.steps
    value = aggregate_tokens_per_s(shape.N, world, ms_step)

    # end to end through the public API with host buffers: every step copies its tokens in
    # from pinned host memory and its result back out.  moe_forward_host_batches overlaps
    # step b+1's copy-in and step b-1's copy-out with step b's layer; the serial call
    # (copy in, layer, copy out, synchronise) is reported beside it.
    xh = x.cpu().pin_memory()
    yhs = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    layer.forward_host_batches([xh] * 3, [yhs[0], yhs[1], yhs[0]], modality=mod)
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    layer.forward_host_batches([xh] * args.steps, [yhs[i % 2] for i in range(args.steps)],
                               modality=mod)
    e2e_ms = max_over_ranks((time.perf_counter() - w0) * 1e3, world) / args.steps
    layer.forward_host(xh, yhs[0], modality=mod)
    barrier(world)
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    for _ in range(args.steps):
        layer.forward_host(xh, yhs[0], modality=mod)
    serial_ms = max_over_ranks((time.perf_counter() - w0) * 1e3, world) / args.steps
    el = x.element_size()

    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    # cuBLAS reached bf16_tflops at full clock (burst) and bf16_tflops_sustained once the
    # power cap pulled the clock down: compare against the regime this run's clock shows
    burst = (clocks.get("sm_mhz") or 0) >= 0.95 * (clocks.get("sm_max_mhz") or 1e9)
    per_launch = {n: launch_ms[i] / max(calls, 1) for i, n in enumerate(names)
                  if i < len(launch_ms)}
    gu_ms = per_launch.get("gemm_gate_up")
    gu_kernel, down_kernel = nat.moe_ffn_kernels(layer.config(shape.N))
    # a short run has few clock samples: a gate/up launch faster than the sustained peak
    # allows ran at burst clocks, whatever the samples say
    if gu_ms and work["flops_gate_up"] / (gu_ms / 1e3) / 1e12 > peaks["bf16_tflops_sustained"]:
        burst = True
    tensor_key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    tensor_peak = peaks[tensor_key]
    ridge = tensor_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    intensity = work["flops_gate_up"] / work["bytes_gate_up"]
    roof = None
    if gu_ms:
        if intensity >= ridge:
            ach = work["flops_gate_up"] / (gu_ms / 1e3) / 1e12
            peak = tensor_peak
            roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": peak, "unit": "TFLOP/s"}
        else:
            ach = work["bytes_gate_up"] / (gu_ms / 1e3) / 1e9
            peak = peaks["hbm_gbs"]
            roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s"}
        roof["frac"] = round(ach / peak, 4)
        roof["traffic"] = read_traffic("gemm_gate_up", args.workload)
        act = "SwiGLU" if shape.act == W.SWIGLU else "ReLU"
        roof["kernel"] = f"gemm_gate_up: {gu_kernel}, {act} epilogue"
        roof["ms_per_launch"] = round(gu_ms, 4)
        roof["peak_source"] = f"{peak_src} ({tensor_key if roof['bound'] == 'tensor' else 'hbm_gbs'})"
    # whole-layer roofline: time bound = max(F / P, B / BW)
    t_bound = max(work["flops_layer"] / (tensor_peak * 1e12),
                  work["bytes_layer"] / (peaks["hbm_gbs"] * 1e9))
    layer_roof = {"flops": work["flops_layer"], "bytes": work["bytes_layer"],
                  "bound_ms": round(t_bound * 1e3, 4), "frac": round(t_bound * 1e3 / ms_step, 4),
                  "tflops": round(work["flops_layer"] / (ms_step / 1e3) / 1e12, 1),
                  "gbs": round(work["bytes_layer"] / (ms_step / 1e3) / 1e9, 1),
                  "kept_assignments": work["M"], "experts_touched": work["touched"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shape, t, sample_tokens=384)

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if shape.dtype == W.BF16 else "f32",
        "data": f"synthetic (seeded N(0,{shape.w_std:g}) weights, N(0,1) tokens)",
        "config": {"workload": workload_desc(shape)
                   + (" overflow=reroute" if args.overflow == "reroute" else ""),
                   "tokens_per_gpu": shape.N, "global_batch": shape.N * world,
                   "l2": ("L2 flushed before every step (256 MB write; the layer's "
                          f"{shape.weight_bytes() / 1e6:.1f} MB of weights fit in L2)"
                          if l2_resident else
                          f"inputs larger than L2 ({shape.weight_bytes() / 1e9:.2f} GB of weights per step)"),
                   "parallelism": f"replicas x{world} (no data-path collective)"},
        "roofline": roof, "layer_roofline": layer_roof,
        "launch_ms": {k: round(v, 4) for k, v in per_launch.items()},
        "ffn_kernels": {"gate_up": gu_kernel, "down": down_kernel},
        "e2e": {"value": round(shape.N * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": shape.N * shape.d * el,
                "d2h_bytes_per_step": shape.N * shape.d * el,
                "method": "moe_forward_host_batches (copies overlapped), wall clock"
                if args.overflow == "drop" else
                "pinned-host copies + moe_forward_reroute + copy back, one stream, wall clock",
                "serial_ms_per_step": round(serial_ms, 4)},
        "gpu_launches": per_step_launches * args.steps,
        "host_enqueue_us_per_step": round(host_us, 1),
        "eager_profiled_ms_per_step": round(eager_ms, 4),
        "timing": "timed region: K replays of the layer captured as one CUDA graph (8 kernels); "
                  "launch_ms and roofline: the same K steps launched eagerly with CUDA events "
                  "between the kernels on the launching stream",
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------------------
class _HostExperts:
    """Per-expert host views of device weights, handed to the oracle as it asks for them."""

    def __init__(self, t):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].float().cpu().numpy()


def _oracle_inputs(shape, t):
    x64 = W.bf16_to_f64(t["x"])
    return dict(x=x64, W_g=W.bf16_to_f64(t["W_g"]), W_gu=_HostExperts(t["W_gu"]),
                W_down=_HostExperts(t["W_down"]),
                kw=dict(k=shape.k, E=shape.E, score_fn=shape.score_fn, renorm=shape.renorm,
                        act=shape.act, clamp=shape.clamp, n_shared=shape.n_shared,
                        bias=None if "bias" not in t else t["bias"].cpu().numpy(),
                        modality=None if "modality" not in t else t["modality"].cpu().numpy(),
                        logit_offset=None if "logit_offset" not in t else t["logit_offset"].cpu().numpy()))


def _oracle_capacity(shape):
    import oracle as O
    return O.capacity(shape.N, shape.k, shape.E, shape.capacity_factor)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count()


def cpu_baseline(shape, t, sample_tokens=64):
    """The oracle as it stands on this host: full routing, expert math for a token sample."""
    import oracle as O
    inp = _oracle_inputs(shape, t)
    C = _oracle_capacity(shape)
    rng = np.random.default_rng(0)
    tokens = np.sort(rng.choice(shape.N, size=min(sample_tokens, shape.N), replace=False))
    t0 = time.perf_counter()
    O.forward(inp["x"], inp["W_g"], inp["W_gu"], inp["W_down"], C=C, tokens=tokens, **inp["kw"])
    dt = time.perf_counter() - t0
    return {"value": round(len(tokens) / dt, 3), "unit": "tokens/s", "cores": _blas_threads(),
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"routing of all {shape.N} tokens + expert FFNs and combine of "
                      f"{len(tokens)} sampled tokens; tokens/s = sampled tokens / wall time"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape = workload_shape(args)
    t = W.make_inputs(shape, device="cuda" if torch.cuda.is_available() else "cpu")
    import oracle as O
    inp = _oracle_inputs(shape, t)
    C = _oracle_capacity(shape)
    per_step = 8
    rng = np.random.default_rng(1)
    times, ntok = [], 0
    for s in range(args.warmup + args.steps):
        tokens = np.sort(rng.choice(shape.N, size=min(per_step, shape.N), replace=False))
        t0 = time.perf_counter()
        O.forward(inp["x"], inp["W_g"], inp["W_gu"], inp["W_down"], C=C, tokens=tokens, **inp["kw"])
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
            ntok += len(tokens)
    total = sum(times)
    value = ntok / total
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(shape), "tokens_per_gpu": shape.N},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": _blas_threads(),
                         "kind": "oracle",
                         "sample": f"per step: routing of all {shape.N} tokens + expert FFNs of "
                                   f"{per_step} sampled tokens"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
