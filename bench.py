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
# with top-k fused with the rank pass (opt-in, MOE_B200_FUSED_TOPK_RANK=1)
LAUNCH_NAMES_FUSED = ["router_gemm", "route_topk_rank", "dispatch_scan", "scatter_gather",
                      "gemm_gate_up", "gemm_down", "combine"]
# with the "report" overflow policy: the capacity pass, the offers and the final layout
LAUNCH_NAMES_REROUTE = ["router_gemm", "route_topk", "rank_local", "dispatch_scan",
                        "capacity_pass", "reroute_offer", "rank_offers", "scan_offers",
                        "reroute_accept", "rank_final", "scan_final", "scatter_gather",
                        "gemm_gate_up", "gemm_down", "combine"]
# a small batch (N <= 64, N k <= 1024) runs the three dispatch passes as one launch
LAUNCH_NAMES_SMALL = ["router_gemm", "route_topk", "dispatch_small", "gemm_gate_up",
                      "gemm_down", "combine"]
LAUNCH_NAMES_REROUTE_SMALL = ["router_gemm", "route_topk", "capacity_pass", "reroute_offer",
                              "rank_offers", "scan_offers", "reroute_accept", "dispatch_final",
                              "gemm_gate_up", "gemm_down", "combine"]
# fp32 layers: SIMT router, and the two SIMT FFN kernels timed as one stage
LAUNCH_NAMES_F32 = ["router_gemm", "route_topk", "rank_local", "dispatch_scan",
                    "scatter_gather", "ffn_up_down_f32", "combine"]
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
    p.add_argument("--no-sweep", action="store_true",
                   help="skip the secondary sweep of decode and ridge-point layers")
    p.add_argument("--cpu-sample", type=int, default=256,
                   help="tokens whose expert math the oracle runs per CPU measurement")
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


def l2_note(shape):
    l2_resident = shape.weight_bytes() + 2 * shape.N * shape.d * (2 if shape.dtype == W.BF16 else 4) < L2_BYTES
    return l2_resident, ("L2 flushed before every step (256 MB write; the layer's "
                         f"{shape.weight_bytes() / 1e6:.1f} MB of weights fit in L2)"
                         if l2_resident else
                         f"inputs larger than L2 ({shape.weight_bytes() / 1e9:.2f} GB of weights per step)")


def bench_config(shape, world, overflow="drop"):
    """The ``config`` object of the JSON line: the same in both arms."""
    return {"workload": workload_desc(shape) + (" overflow=reroute" if overflow == "reroute" else ""),
            "tokens_per_gpu": shape.N, "global_batch": shape.N * world,
            "seed": shape.seed, "l2": l2_note(shape)[1],
            "parallelism": f"replicas x{world} (no data-path collective)"}


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
    # the down launch: its weights, the hidden rows in, the expert outputs out
    b_down = w_down + rows * F * el + rows * d * el
    return dict(M=M, touched=touched, flops_layer=f_gate_up + f_down + f_router,
                bytes_layer=b_layer, flops_gate_up=f_gate_up, bytes_gate_up=b_gate_up,
                flops_down=f_down, bytes_down=b_down)


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        self.power = []
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
                self.power.append(self.nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
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
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples),
                "power_w": round(statistics.median(self.power), 1) if self.power else None}


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


def pick_tensor_peak(peaks, clocks, flops=None, ms=None):
    """cuBLAS reached bf16_tflops at full clock (burst) and bf16_tflops_sustained once the
    power cap pulled the clock down: compare against the regime this run's clock shows.  A
    short run has few clock samples: a launch faster than the sustained peak allows ran at
    burst clocks, whatever the samples say."""
    burst = (clocks.get("sm_mhz") or 0) >= 0.95 * (clocks.get("sm_max_mhz") or 1e9)
    if flops and ms and flops / (ms / 1e3) / 1e12 > peaks["bf16_tflops_sustained"]:
        burst = True
    key = "bf16_tflops" if burst else "bf16_tflops_sustained"
    return key, peaks[key]


def layer_roofline(work, ms_step, peaks, tensor_peak):
    """Whole-layer roofline: time bound = max(F / P, B / BW); the binding roof is the larger."""
    t_tensor = work["flops_layer"] / (tensor_peak * 1e12)
    t_hbm = work["bytes_layer"] / (peaks["hbm_gbs"] * 1e9)
    t_bound = max(t_tensor, t_hbm)
    return {"flops": work["flops_layer"], "bytes": work["bytes_layer"],
            "bound": "tensor" if t_tensor >= t_hbm else "hbm",
            "bound_ms": round(t_bound * 1e3, 4), "frac": round(t_bound * 1e3 / ms_step, 4),
            "tflops": round(work["flops_layer"] / (ms_step / 1e3) / 1e12, 1),
            "gbs": round(work["bytes_layer"] / (ms_step / 1e3) / 1e9, 1),
            "kept_assignments": work["M"], "experts_touched": work["touched"]}


def time_graphed(layer, x, y, mod, steps, warmup, world, local, l2_resident):
    """K replays of the layer captured as one CUDA graph, timed with CUDA events on the
    launching stream between a barrier + synchronize on both sides.  A layer whose weights
    and tokens fit in L2 gets L2 flushed before every step (a 256 MB write) and only the
    replays are timed.  Returns (device ms of all K steps, host enqueue us per step, clocks)."""
    stream = torch.cuda.current_stream()
    layer.forward_graphed(x, y, modality=mod)
    for _ in range(warmup):
        layer.forward_graphed(x, y, modality=mod)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if l2_resident else None
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if flush is None:
            ev0.record(stream)
            h0 = time.perf_counter()
            for _ in range(steps):
                layer.forward_graphed(x, y, modality=mod)
            host_us = (time.perf_counter() - h0) * 1e6 / steps
            ev1.record(stream)
            torch.cuda.synchronize()
            timed_ms = ev0.elapsed_time(ev1)
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
            h0 = time.perf_counter()
            for a, b in evs:
                flush.fill_(1)
                a.record(stream)
                layer.forward_graphed(x, y, modality=mod)
                b.record(stream)
            host_us = (time.perf_counter() - h0) * 1e6 / steps
            torch.cuda.synchronize()
            timed_ms = sum(a.elapsed_time(b) for a, b in evs)
    barrier(world)
    return timed_ms, host_us, clk.summary()


def route_counts(layer, shape, x, mod):
    """Kept rows per expert of this batch (untimed), for the algorithmic work."""
    counts = torch.empty(shape.E, dtype=torch.int32, device="cuda")
    layer.forward(x, modality=mod, route_out={"counts": counts})
    assert layer.check_status() == 0
    return counts.cpu().numpy()


# decode-sized and ridge-point layers measured beside the headline (same timing rules)
# lightest first: a layer timed right after a ~1 kW one inherits the power-cap governor's
# low clock for a second or so (see settle_power)
SWEEP = ["capacity-cf1", "switch-cf1", "mixtral-n16", "dsv3-n64", "v41flash-n64", "dsv3-n8192",
         "v41flash-n16384"]


def settle_power(index, limit_s=3.0):
    """Wait (at most limit_s, idle) until the board's power reading falls below half its
    limit.  NVML reports a moving average, and while it stays high after a heavy layer the
    power-cap governor holds the clock down: a short layer timed then would measure that
    layer's leftover state, not its own.  Returns the seconds waited."""
    t0 = time.perf_counter()
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(index)
        lim = pynvml.nvmlDeviceGetEnforcedPowerLimit(h) / 1000.0
        while time.perf_counter() - t0 < limit_s:
            if pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0 < 0.5 * lim:
                break
            time.sleep(0.1)
    except Exception:  # no NVML: nothing to wait for
        pass
    return time.perf_counter() - t0


def sweep_entry(name, args, world, rank, local, peaks):
    from mixture_experts_layer_50_b200.layer import MoELayer
    shape = W.PRESETS[name]
    t = make_replica(shape, rank)
    layer = MoELayer.from_workload(shape, t)
    x, mod = t["x"], t.get("modality")
    y = torch.empty_like(x)
    work = algorithmic_work(shape, route_counts(layer, shape, x, mod))
    l2_resident, _ = l2_note(shape)
    torch.cuda.synchronize()
    waited = settle_power(local)
    timed_ms, _, clocks = time_graphed(layer, x, y, mod, args.steps, args.warmup, world, local,
                                       l2_resident)
    assert layer.check_status() == 0
    ms_step = max_over_ranks(timed_ms, world) / args.steps
    key, tensor_peak = pick_tensor_peak(peaks, clocks)
    lr = layer_roofline(work, ms_step, peaks, tensor_peak)
    if lr["bound"] == "tensor":
        achieved, peak, unit = lr["tflops"], tensor_peak, "TFLOP/s"
    else:
        achieved, peak, unit = lr["gbs"], peaks["hbm_gbs"], "GB/s"
    out = {"workload": workload_desc(shape), "ms_per_step": round(ms_step, 4),
           "tokens_per_s": round(shape.N * world / (ms_step / 1e3), 1),
           "bound": lr["bound"], "achieved": achieved, "peak": peak, "unit": unit,
           "frac": lr["frac"], "peak_key": key if lr["bound"] == "tensor" else "hbm_gbs",
           "kept_assignments": lr["kept_assignments"], "experts_touched": lr["experts_touched"],
           "clocks": {k: clocks.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "power_w")},
           "settle_s": round(waited, 2)}
    del layer, t, x, y
    torch.cuda.empty_cache()
    return out


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
    work = algorithmic_work(shape, route_counts(layer, shape, x, mod))
    for _ in range(args.warmup):
        layer.forward(x, modality=mod, y=y)
    torch.cuda.synchronize()
    per_step_launches = nat.moe_last_launch_count()


    # timed region: K replays of the whole layer (the eight launches captured once as a
    # CUDA graph)
    l2_resident, _ = l2_note(shape)
    timed_ms, host_us, clocks = time_graphed(layer, x, y, mod, args.steps, args.warmup, world,
                                             local, l2_resident)
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
    # the profiled calls run every launch on the launching stream (the shared expert inside
    # the routed GEMMs), in this order
    names = {8: LAUNCH_NAMES,
             7: LAUNCH_NAMES_FUSED if shape.dtype == W.BF16 else LAUNCH_NAMES_F32,
             6: LAUNCH_NAMES_SMALL, 15: LAUNCH_NAMES_REROUTE,
             11: LAUNCH_NAMES_REROUTE_SMALL}.get(len(launch_ms),
                                                 [f"launch_{i}" for i in range(len(launch_ms))])
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
    per_launch = {n: launch_ms[i] / max(calls, 1) for i, n in enumerate(names)
                  if i < len(launch_ms)}
    gu_ms = per_launch.get("gemm_gate_up")
    gu_kernel, down_kernel = nat.moe_ffn_kernels(layer.config(shape.N))
    roof_name = "gemm_gate_up"
    if gu_ms is None and "ffn_up_down_f32" in per_launch:
        # fp32 layers: the two SIMT FFN kernels are timed as one stage; its work is both
        gu_ms = per_launch["ffn_up_down_f32"]
        work = dict(work, flops_gate_up=work["flops_gate_up"] + work["flops_down"],
                    bytes_gate_up=work["bytes_gate_up"] + work["bytes_down"])
        roof_name = "ffn_up_down_f32"
    tensor_key, tensor_peak = pick_tensor_peak(peaks, clocks, work["flops_gate_up"], gu_ms)
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
        roof["traffic"] = read_traffic(roof_name, args.workload)
        act = "SwiGLU" if shape.act == W.SWIGLU else "ReLU"
        roof["kernel"] = (f"gemm_gate_up: {gu_kernel}, {act} epilogue" if roof_name == "gemm_gate_up"
                          else f"ffn_up_down_f32: {gu_kernel} + {down_kernel} (one stage)")
        roof["ms_per_launch"] = round(gu_ms, 4)
        roof["peak_source"] = f"{peak_src} ({tensor_key if roof['bound'] == 'tensor' else 'hbm_gbs'})"
    layer_roof = layer_roofline(work, ms_step, peaks, tensor_peak)

    # the headline layer's buffers go before the sweep allocates its own layers
    del layer, t, x, y, xh, yhs
    torch.cuda.empty_cache()
    sweep = None
    if not args.no_sweep and args.tokens is None and args.experts is None \
            and args.overflow == "drop":
        sweep = {}
        for name in SWEEP:
            if name != args.workload:
                sweep[name] = sweep_entry(name, args, world, rank, local, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(shape, args.cpu_sample)

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
        if shape.dtype == W.BF16 else "f32",
        "data": f"synthetic (seeded N(0,{shape.w_std:g}) weights, N(0,1) tokens)",
        "config": bench_config(shape, world, args.overflow),
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
        "timing": f"timed region: K replays of the layer captured as one CUDA graph "
                  f"({per_step_launches} kernels); "
                  "launch_ms and roofline: the same K steps launched eagerly with CUDA events "
                  "between the kernels on the launching stream",
        "clocks": clocks,
        "sweep": sweep,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ------------------------------------------------------------------------------------------
# the CPU oracle timed on this host (the cpu_baseline leg and the reference arm)
# ------------------------------------------------------------------------------------------
HOST_F64_BUDGET = 24 << 30      # float64 expert weights kept on the host between measurements


class _HostExperts:
    """float64 host copies of the per-expert device weights, made on first use and kept while
    they fit a host budget.  The time spent making them is counted apart (``fetch_s``) so that
    it can be taken out of the oracle's own time."""

    def __init__(self, t, cache):
        self.t, self.cache, self.fetch_s = t, cache, 0.0

    def __getitem__(self, e):
        key = (self.t.data_ptr(), e)
        a = self.cache.get(key)
        if a is None:
            t0 = time.perf_counter()
            a = self.t[e].to(torch.float64).cpu().numpy()     # bf16 -> float64 is exact
            self.fetch_s += time.perf_counter() - t0
            if sum(v.nbytes for v in self.cache.values()) + a.nbytes <= HOST_F64_BUDGET:
                self.cache[key] = a
        return a


class OracleTimer:
    """Times the oracle as it stands on one layer instance: the routing of all N tokens
    (router projection, scores, top-k, capacity and layout) and the expert math and combine
    of a seeded token sample, in separate clocks.  The full-layer time per token is
    extrapolated from the two: t_route / N + t_expert / |sample|."""

    def __init__(self, shape, t):
        self.shape = shape
        dev = t["x"].device
        self.x64 = t["x"].to(torch.float64).cpu().numpy() if dev.type == "cuda" else W.bf16_to_f64(t["x"])
        self.Wg64 = t["W_g"].to(torch.float64).cpu().numpy()
        cache = {}
        self.W_gu, self.W_down = _HostExperts(t["W_gu"], cache), _HostExperts(t["W_down"], cache)
        self.kw = dict(k=shape.k, E=shape.E, score_fn=shape.score_fn, renorm=shape.renorm,
                       act=shape.act, clamp=shape.clamp, n_shared=shape.n_shared,
                       bias=None if "bias" not in t else t["bias"].cpu().numpy(),
                       modality=None if "modality" not in t else t["modality"].cpu().numpy())
        self.offset = None if "logit_offset" not in t else t["logit_offset"].cpu().numpy()
        import oracle as O
        self.O = O
        self.C = O.capacity(shape.N, shape.k, shape.E, shape.capacity_factor)

    def prefetch(self, tokens):
        """Host float64 weights of the experts the sample touches (outside any clock)."""
        O, kw = self.O, self.kw
        z = O.router_logits(self.x64[tokens], self.Wg64, self.offset)
        ids, _ = O.route(z, kw["k"], kw["score_fn"], kw["renorm"], kw["bias"],
                         None if kw["modality"] is None else kw["modality"][tokens])
        for e in sorted(set(ids.ravel().tolist())) + list(range(self.shape.E, self.shape.G)):
            self.W_gu[e], self.W_down[e]

    def measure(self, tokens):
        O, kw = self.O, self.kw
        t0 = time.perf_counter()
        z = O.router_logits(self.x64, self.Wg64, self.offset)
        ids, _ = O.route(z, kw["k"], kw["score_fn"], kw["renorm"], kw["bias"], kw["modality"])
        O.dispatch(ids, self.shape.E, self.C)
        t_route = time.perf_counter() - t0
        f0 = self.W_gu.fetch_s + self.W_down.fetch_s
        t1 = time.perf_counter()
        O.forward(self.x64, None, self.W_gu, self.W_down, logits=z, tokens=tokens, C=self.C, **kw)
        fetched = self.W_gu.fetch_s + self.W_down.fetch_s - f0
        t_expert = time.perf_counter() - t1 - fetched
        return t_route, t_expert

    def sample(self, rng, n):
        return np.sort(rng.choice(self.shape.N, size=min(n, self.shape.N), replace=False))


def _host_info():
    cpu_model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    cpu_model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        blas = max(n) if n else 1
    except Exception:
        blas = None
    return {"nproc": len(os.sched_getaffinity(0)), "cpu_model": cpu_model, "blas_threads": blas}


def oracle_runs(shape, t, sample_tokens, steps, warmup, seed):
    """Per-token full-layer seconds of the oracle over ``steps`` measurements (each on a
    fresh seeded sample of ``sample_tokens`` tokens) after ``warmup`` untimed ones."""
    ot = OracleTimer(shape, t)
    rng = np.random.default_rng(seed)
    per_token, wall = [], []
    for s in range(warmup + steps):
        tokens = ot.sample(rng, sample_tokens)
        ot.prefetch(tokens)
        t_route, t_expert = ot.measure(tokens)
        if s >= warmup:
            per_token.append(t_route / shape.N + t_expert / len(tokens))
            wall.append(t_route + t_expert)
    return per_token, wall, len(tokens)


def _oracle_sample_note(shape, n):
    return (f"per measurement: routing of all {shape.N} tokens (router projection, scores, "
            f"top-k, capacity, layout) + expert FFNs and combine of {n} seeded sampled tokens, "
            f"timed apart; value = 1 / (t_route/{shape.N} + t_expert/{n}), the full-layer "
            "throughput extrapolated from the sample (host float64 weight copies made "
            "outside the clocks)")


def cpu_baseline(shape, sample_tokens):
    """The oracle as it stands on this host, the same measurement as the reference arm."""
    t = W.make_inputs(shape, device="cuda" if torch.cuda.is_available() else "cpu")
    per_token, wall, n = oracle_runs(shape, t, sample_tokens, steps=2, warmup=0, seed=1)
    info = _host_info()
    return {"value": round(1.0 / statistics.mean(per_token), 3), "unit": "tokens/s",
            "cores": info["blas_threads"] or info["nproc"], "kind": "oracle",
            "seconds": round(sum(wall), 2), "host": info,
            "sample": "2 measurements; " + _oracle_sample_note(shape, n)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    shape = workload_shape(args)
    t = W.make_inputs(shape, device="cuda" if torch.cuda.is_available() else "cpu")
    per_token, wall, n = oracle_runs(shape, t, args.cpu_sample, args.steps, args.warmup, seed=1)
    value = 1.0 / statistics.mean(per_token)
    info = _host_info()
    out = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * shape.N / value, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(shape, world, args.overflow),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s",
                         "cores": info["blas_threads"] or info["nproc"], "kind": "oracle",
                         "seconds": round(sum(wall), 2), "host": info,
                         "sample": f"{args.steps} measurements after {args.warmup} untimed; "
                                   + _oracle_sample_note(shape, n)
                                   + "; ms_per_step = N / value, the extrapolated full layer"},
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
