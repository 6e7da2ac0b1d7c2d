"""ctypes binding of ``libmoe_b200.so`` (the C ABI of include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
Functions keep the C names and take torch tensors (device memory) plus the current torch
CUDA stream.  There is no fallback: if the library is missing, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os
from fractions import Fraction
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_50_b200.build` "
        "(nvcc, sm_100a). There is no non-CUDA implementation of this layer.")

lib = ctypes.CDLL(LIB_PATH)

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_INVALID_INPUT, \
    MOE_ERR_TIMEOUT = range(6)
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_CUDA", 4: "MOE_ERR_INVALID_INPUT", 5: "MOE_ERR_TIMEOUT"}
SOFTMAX, SIGMOID = 0, 1
SWIGLU, RELU = 0, 1
BF16, F32 = 0, 1


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.moe_last_error().decode("utf-8", "replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


class moe_config(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("F", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("n_bias_sets", ctypes.c_int32), ("score_fn", ctypes.c_int32),
                ("renorm", ctypes.c_int32), ("act", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("clamp", ctypes.c_float), ("capacity", ctypes.c_int64)]


class moe_route_out(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("logits", "ids", "gates", "counts", "demand", "drop_mask", "offsets")]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_cfgp = ctypes.POINTER(moe_config)
lib.moe_workspace_size.argtypes = [_cfgp]
lib.moe_workspace_size.restype = _sz
lib.moe_workspace_init.argtypes = [_vp, _vp]
lib.moe_capacity.argtypes = [_i64, _i32, _i32, _i64, _i64]
lib.moe_capacity.restype = _i64
lib.moe_route.argtypes = [_cfgp] + [_vp] * 14
lib.moe_permute.argtypes = [_cfgp] + [_vp] * 9
lib.moe_expert_ffn.argtypes = [_cfgp] + [_vp] * 8
lib.moe_combine.argtypes = [_cfgp] + [_vp] * 5
lib.moe_forward.argtypes = [_cfgp] + [_vp] * 11
lib.moe_forward_host.argtypes = [_cfgp] + [_vp] * 10
lib.moe_check_status.argtypes = [_vp, _vp]
lib.moe_route_static.argtypes = [_cfgp] + [_vp] * 10
lib.moe_forward_routed.argtypes = [_cfgp] + [_vp] * 9
lib.moe_route_hash.argtypes = [_cfgp] + [_vp] * 8
lib.moe_balance.argtypes = [_cfgp] + [_vp] * 8 + [ctypes.c_float, _vp, _vp]
lib.moe_permute_padded.argtypes = [_cfgp] + [_vp] * 10
lib.moe_forward_padded.argtypes = [_cfgp] + [_vp] * 11
lib.moe_forward_host_batches.argtypes = [_cfgp, _i32] + [_vp] * 10
lib.moe_route_reroute.argtypes = [_cfgp] + [_vp] * 15
lib.moe_selftest_wait_timeout.argtypes = [_vp, _i64, _vp]
lib.moe_forward_reroute.argtypes = [_cfgp] + [_vp] * 12
lib.moe_ffn_kernels.argtypes = [_cfgp, ctypes.c_char_p, ctypes.c_char_p, ctypes.c_size_t]


class moe_ep_chunk(ctypes.Structure):
    _fields_ = [("peer", ctypes.c_int32), ("expert", ctypes.c_int32), ("row", ctypes.c_int64),
                ("rows", ctypes.c_int64)]


lib.moe_ep_first_expert.argtypes = [_i32, _i32, _i32]
lib.moe_ep_first_expert.restype = _i32
lib.moe_ep_plan.argtypes = [_i32, _i32, _i32, _i64] + [_vp] * 10
lib.moe_ep_workspace_size.argtypes = [_cfgp, _i32]
lib.moe_ep_workspace_size.restype = _sz
lib.moe_permute_ep.argtypes = [_cfgp] + [_vp] * 11
lib.moe_ep_expert_ffn.argtypes = [_cfgp, _i32, _i32, _i64, _i64] + [_vp] * 9
lib.moe_ep_combine.argtypes = [_cfgp] + [_vp] * 5
lib.moe_ep_copy_runs.argtypes = [_vp, _i64, _vp, _vp, _i32, _vp, _vp, _i32, _i64, _i64, _vp, _vp]
lib.moe_permute_ep_p2p.argtypes = [_cfgp] + [_vp] * 12
lib.moe_ep_combine_p2p.argtypes = [_cfgp] + [_vp] * 10
lib.moe_ipc_handle.argtypes = [_vp, _vp, ctypes.POINTER(_i64)]
lib.moe_ipc_open.argtypes = [_vp, ctypes.POINTER(_vp)]
lib.moe_ipc_close.argtypes = [_vp]
lib.moe_check_dispatch_host.argtypes = [_i64, _i32, _i32, _i64] + [_vp] * 8 + [_sz]
lib.moe_check_dispatch.argtypes = [_cfgp] + [_vp] * 8
lib.moe_profile_begin.argtypes = [_i32]
lib.moe_profile_begin.restype = ctypes.c_int
lib.moe_profile_end.argtypes = [ctypes.POINTER(ctypes.c_float), _i32, ctypes.POINTER(_i32)]
lib.moe_profile_end.restype = _i32
lib.moe_last_error.restype = ctypes.c_char_p
lib.moe_last_launch_count.restype = _i32
for _f in ("moe_workspace_init", "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine",
           "moe_forward", "moe_forward_host", "moe_check_status", "moe_route_static",
           "moe_forward_routed", "moe_route_hash", "moe_balance", "moe_permute_padded",
           "moe_forward_padded", "moe_forward_host_batches", "moe_route_reroute",
           "moe_forward_reroute", "moe_selftest_wait_timeout", "moe_ffn_kernels", "moe_ep_plan",
           "moe_permute_ep", "moe_ep_expert_ffn", "moe_ep_combine", "moe_check_dispatch_host",
           "moe_check_dispatch", "moe_ep_copy_runs", "moe_ipc_handle", "moe_ipc_open",
           "moe_ipc_close", "moe_permute_ep_p2p", "moe_ep_combine_p2p"):
    getattr(lib, _f).restype = ctypes.c_int

EXPORTED = ("moe_workspace_size", "moe_workspace_init", "moe_capacity", "moe_route",
            "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward", "moe_forward_host",
            "moe_check_status", "moe_profile_begin", "moe_profile_end", "moe_last_error",
            "moe_last_launch_count", "moe_route_static", "moe_forward_routed",
            "moe_route_hash", "moe_balance", "moe_permute_padded", "moe_forward_padded",
            "moe_forward_host_batches", "moe_route_reroute", "moe_forward_reroute",
            "moe_selftest_wait_timeout", "moe_ffn_kernels", "moe_ep_first_expert",
            "moe_ep_plan", "moe_ep_workspace_size", "moe_permute_ep", "moe_ep_expert_ffn",
            "moe_ep_combine", "moe_check_dispatch_host", "moe_check_dispatch",
            "moe_ep_copy_runs", "moe_ipc_handle", "moe_ipc_open", "moe_ipc_close",
            "moe_permute_ep_p2p", "moe_ep_combine_p2p")


def make_config(N, d, E, k, F, n_shared=0, n_bias_sets=0, score_fn=SOFTMAX, renorm=1,
                act=SWIGLU, dtype=BF16, clamp=0.0, capacity=0) -> moe_config:
    return moe_config(int(N), int(d), int(E), int(k), int(F), int(n_shared), int(n_bias_sets),
                      int(score_fn), int(renorm), int(act), int(dtype), float(clamp),
                      int(capacity))


def config_from_shape(shape, N: Optional[int] = None, capacity: int = 0) -> moe_config:
    """moe_config for a workloads.LayerShape."""
    return make_config(shape.N if N is None else N, shape.d, shape.E, shape.k, shape.F,
                       shape.n_shared, shape.n_bias_sets, shape.score_fn, shape.renorm,
                       shape.act, shape.dtype, shape.clamp, capacity)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"expected a torch tensor, got {type(t)}")
    if not t.is_cuda:
        raise ValueError("tensors passed to the MoE library must live in CUDA memory")
    if not t.is_contiguous():
        raise ValueError("tensors passed to the MoE library must be contiguous")
    return t.data_ptr()


def _host_ptr(t) -> int:
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("host buffers must be contiguous CPU tensors (pinned for speed)")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def moe_workspace_size(cfg: moe_config) -> int:
    return int(lib.moe_workspace_size(ctypes.byref(cfg)))


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _check(lib.moe_workspace_init(_ptr(ws), _stream(stream)), "moe_workspace_init")


def alloc_workspace(cfg: moe_config, device="cuda") -> torch.Tensor:
    """A zero-initialised workspace (uint8 tensor) for calls with this configuration."""
    size = moe_workspace_size(cfg)
    if size == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    ws = torch.empty(size + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + size]
    moe_workspace_init(ws)
    return ws


def moe_capacity(T: int, k: int, E: int, cf) -> int:
    """C = ceil(T k / E * cf); cf None (no limit) gives 0."""
    if cf is None:
        return 0
    f = Fraction(cf)
    return int(lib.moe_capacity(int(T), int(k), int(E), f.numerator, f.denominator))


def moe_route(cfg, *, logits=None, x=None, W_g=None, logit_offset=None, bias=None,
              modality=None, ids=None, gates=None, counts=None, demand=None, drop_mask=None,
              logits_out=None, ws, stream=None):
    st = lib.moe_route(ctypes.byref(cfg), _ptr(logits), _ptr(x), _ptr(W_g), _ptr(logit_offset),
                       _ptr(bias), _ptr(modality), _ptr(ids), _ptr(gates), _ptr(counts),
                       _ptr(demand), _ptr(drop_mask), _ptr(logits_out), _ptr(ws),
                       _stream(stream))
    _check(st, "moe_route")


def moe_route_static(cfg, *, logits, bias=None, modality=None, ids, gates, counts, demand,
                     drop_mask, status=None, stream=None):
    """moe_route on given logits without a workspace (scratch in the library's fixed array)."""
    st = lib.moe_route_static(ctypes.byref(cfg), _ptr(logits), _ptr(bias), _ptr(modality),
                              _ptr(ids), _ptr(gates), _ptr(counts), _ptr(demand),
                              _ptr(drop_mask), _ptr(status), _stream(stream))
    _check(st, "moe_route_static")


def moe_permute(cfg, *, ids, drop_mask=None, x, offsets, row_token=None, slot_row, xp, ws,
                stream=None):
    st = lib.moe_permute(ctypes.byref(cfg), _ptr(ids), _ptr(drop_mask), _ptr(x), _ptr(offsets),
                         _ptr(row_token), _ptr(slot_row), _ptr(xp), _ptr(ws), _stream(stream))
    _check(st, "moe_permute")


def moe_expert_ffn(cfg, *, xp, offsets, x=None, W_gu, W_down, ye, ws, stream=None):
    st = lib.moe_expert_ffn(ctypes.byref(cfg), _ptr(xp), _ptr(offsets), _ptr(x), _ptr(W_gu),
                            _ptr(W_down), _ptr(ye), _ptr(ws), _stream(stream))
    _check(st, "moe_expert_ffn")


def moe_combine(cfg, *, ye, slot_row, gates, y, stream=None):
    st = lib.moe_combine(ctypes.byref(cfg), _ptr(ye), _ptr(slot_row), _ptr(gates), _ptr(y),
                         _stream(stream))
    _check(st, "moe_combine")


def moe_forward(cfg, *, x, W_g, W_gu, W_down, y, logit_offset=None, bias=None, modality=None,
                route_out: Optional[dict] = None, ws, stream=None):
    ro = None
    if route_out:
        ro = moe_route_out(*[_ptr(route_out.get(n)) for n, _ in moe_route_out._fields_])
    st = lib.moe_forward(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(logit_offset), _ptr(bias),
                         _ptr(modality), _ptr(W_gu), _ptr(W_down), _ptr(y),
                         ctypes.byref(ro) if ro is not None else None, _ptr(ws),
                         _stream(stream))
    _check(st, "moe_forward")


def moe_route_reroute(cfg, *, logits=None, x=None, W_g=None, logit_offset=None, bias=None,
                      modality=None, ids=None, gates=None, counts=None, demand=None,
                      drop_mask=None, rerouted=None, logits_out=None, ws, stream=None):
    """Routing with the "report" overflow policy: a dropped slot goes to the token's next-best
    expert while that expert has room."""
    st = lib.moe_route_reroute(ctypes.byref(cfg), _ptr(logits), _ptr(x), _ptr(W_g),
                               _ptr(logit_offset), _ptr(bias), _ptr(modality), _ptr(ids),
                               _ptr(gates), _ptr(counts), _ptr(demand), _ptr(drop_mask),
                               _ptr(rerouted), _ptr(logits_out), _ptr(ws), _stream(stream))
    _check(st, "moe_route_reroute")


def moe_forward_reroute(cfg, *, x, W_g, W_gu, W_down, y, logit_offset=None, bias=None,
                        modality=None, route_out: Optional[dict] = None, rerouted=None, ws,
                        stream=None):
    """The layer with the "report" overflow policy instead of dropping."""
    ro = None
    if route_out:
        ro = moe_route_out(*[_ptr(route_out.get(n)) for n, _ in moe_route_out._fields_])
    st = lib.moe_forward_reroute(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(logit_offset),
                                 _ptr(bias), _ptr(modality), _ptr(W_gu), _ptr(W_down), _ptr(y),
                                 ctypes.byref(ro) if ro is not None else None, _ptr(rerouted),
                                 _ptr(ws), _stream(stream))
    _check(st, "moe_forward_reroute")


def moe_forward_routed(cfg, *, x, ids, gates, W_gu, W_down, y, route_out: Optional[dict] = None,
                       ws, stream=None):
    """The layer with caller-supplied (forced or replayed) ids and gates."""
    ro = None
    if route_out:
        ro = moe_route_out(*[_ptr(route_out.get(n)) for n, _ in moe_route_out._fields_])
    st = lib.moe_forward_routed(ctypes.byref(cfg), _ptr(x), _ptr(ids), _ptr(gates), _ptr(W_gu),
                                _ptr(W_down), _ptr(y),
                                ctypes.byref(ro) if ro is not None else None, _ptr(ws),
                                _stream(stream))
    _check(st, "moe_forward_routed")


def moe_route_hash(cfg, *, token_ids, ids, gates, counts=None, demand=None, drop_mask=None, ws,
                   stream=None):
    """Deterministic hash routing of token ids, then capacity and counts."""
    st = lib.moe_route_hash(ctypes.byref(cfg), _ptr(token_ids), _ptr(ids), _ptr(gates),
                            _ptr(counts), _ptr(demand), _ptr(drop_mask), _ptr(ws),
                            _stream(stream))
    _check(st, "moe_route_hash")


def moe_balance(cfg, *, logits, ids, modality=None, f=None, P=None, aux=None, set_load=None,
                bias=None, gamma=0.001, ws, stream=None):
    """Balance statistics (f, P, E sum f P, loads per bias set) and the +-gamma bias update."""
    st = lib.moe_balance(ctypes.byref(cfg), _ptr(logits), _ptr(ids), _ptr(modality), _ptr(f),
                         _ptr(P), _ptr(aux), _ptr(set_load), _ptr(bias), float(gamma), _ptr(ws),
                         _stream(stream))
    _check(st, "moe_balance")


def moe_permute_padded(cfg, *, ids, drop_mask=None, x, offsets_pad, counts, row_token_pad=None,
                       slot_row, xp_pad, ws, stream=None):
    """The padded [E][C][d] dispatch buffer (capacity as a tensor dimension)."""
    st = lib.moe_permute_padded(ctypes.byref(cfg), _ptr(ids), _ptr(drop_mask), _ptr(x),
                                _ptr(offsets_pad), _ptr(counts), _ptr(row_token_pad),
                                _ptr(slot_row), _ptr(xp_pad), _ptr(ws), _stream(stream))
    _check(st, "moe_permute_padded")


def moe_forward_padded(cfg, *, x, W_g, W_gu, W_down, y, logit_offset=None, bias=None,
                       modality=None, route_out: Optional[dict] = None, ws, stream=None):
    """The layer through the padded dispatch layout (needs a capacity)."""
    ro = None
    if route_out:
        ro = moe_route_out(*[_ptr(route_out.get(n)) for n, _ in moe_route_out._fields_])
    st = lib.moe_forward_padded(ctypes.byref(cfg), _ptr(x), _ptr(W_g), _ptr(logit_offset),
                                _ptr(bias), _ptr(modality), _ptr(W_gu), _ptr(W_down), _ptr(y),
                                ctypes.byref(ro) if ro is not None else None, _ptr(ws),
                                _stream(stream))
    _check(st, "moe_forward_padded")


def moe_forward_host(cfg, *, x_host, W_g, W_gu, W_down, y_host, logit_offset=None, bias=None,
                     modality=None, ws, stream=None):
    st = lib.moe_forward_host(ctypes.byref(cfg), _host_ptr(x_host), _ptr(W_g),
                              _ptr(logit_offset), _ptr(bias), _ptr(modality), _ptr(W_gu),
                              _ptr(W_down), _host_ptr(y_host), _ptr(ws), _stream(stream))
    _check(st, "moe_forward_host")


def moe_forward_host_batches(cfg, *, x_host: list, W_g, W_gu, W_down, y_host: list,
                             logit_offset=None, bias=None, modality: Optional[list] = None, ws,
                             stream=None):
    """Pipelined host-to-host layer over several batches (copies overlap the layer)."""
    n = len(x_host)
    if len(y_host) != n:
        raise ValueError("x_host and y_host must have the same number of batches")
    xs = (ctypes.c_void_p * n)(*[_host_ptr(t) for t in x_host])
    ys = (ctypes.c_void_p * n)(*[_host_ptr(t) for t in y_host])
    mods = None
    if modality is not None:
        mods = (ctypes.c_void_p * n)(*[_ptr(t) for t in modality])
    st = lib.moe_forward_host_batches(ctypes.byref(cfg), n, xs, _ptr(W_g), _ptr(logit_offset),
                                      _ptr(bias), mods, _ptr(W_gu), _ptr(W_down), ys, _ptr(ws),
                                      _stream(stream))
    _check(st, "moe_forward_host_batches")


def moe_ffn_kernels(cfg) -> tuple:
    """Names of the kernels the gate/up and the down projections of cfg launch (host only)."""
    gu = ctypes.create_string_buffer(256)
    dn = ctypes.create_string_buffer(256)
    _check(lib.moe_ffn_kernels(ctypes.byref(cfg), gu, dn, 256), "moe_ffn_kernels")
    return gu.value.decode(), dn.value.decode()


def moe_selftest_wait_timeout(ws, limit_ns: int, stream=None):
    """A bounded device wait on a barrier nothing completes: records MOE_ERR_TIMEOUT."""
    _check(lib.moe_selftest_wait_timeout(_ptr(ws), int(limit_ns), _stream(stream)),
           "moe_selftest_wait_timeout")


def moe_check_status(ws, stream=None) -> int:
    """Synchronise and return the device status (0 = MOE_OK); clears it."""
    return int(lib.moe_check_status(_ptr(ws), _stream(stream)))


def moe_last_launch_count() -> int:
    return int(lib.moe_last_launch_count())


def moe_profile_begin(max_calls: int):
    _check(lib.moe_profile_begin(int(max_calls)), "moe_profile_begin")


def moe_profile_end(max_launches: int = 16):
    """(per-launch total ms over the recorded calls, number of recorded calls)."""
    buf = (ctypes.c_float * max_launches)()
    calls = _i32(0)
    n = lib.moe_profile_end(buf, max_launches, ctypes.byref(calls))
    if n < 0:
        raise MoeError(MOE_ERR_CUDA, "moe_profile_end")
    return [float(buf[i]) for i in range(min(n, max_launches))], int(calls.value)


# ---- expert parallelism --------------------------------------------------------------------
def moe_ep_first_expert(world: int, rank: int, E: int) -> int:
    """First expert owned by ``rank`` (``rank == world`` gives E)."""
    v = int(lib.moe_ep_first_expert(int(world), int(rank), int(E)))
    if v < 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_ep_first_expert")
    return v


def moe_ep_plan(world: int, rank: int, E: int, capacity: int, demand_all) -> dict:
    """The exchange plan of one rank (host only).  ``demand_all``: int32 [world][E] (numpy or
    CPU tensor).  Returns cap [E], kept_all [world][E], owned_offsets [E_own + 1] (numpy
    int32), sends / recvs as lists of (peer, expert, row, rows), rows_kept, rows_owned."""
    import numpy as np
    dem = np.ascontiguousarray(np.asarray(demand_all, dtype=np.int32).reshape(world, E))
    e_own = moe_ep_first_expert(world, rank + 1, E) - moe_ep_first_expert(world, rank, E)
    cap = np.zeros(E, np.int32)
    kept = np.zeros((world, E), np.int32)
    owned = np.zeros(e_own + 1, np.int32)
    sends = (moe_ep_chunk * E)()
    recvs = (moe_ep_chunk * max(1, world * e_own))()
    ns, nr = _i32(0), _i32(0)
    rk, ro = _i64(0), _i64(0)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    st = lib.moe_ep_plan(int(world), int(rank), int(E), int(capacity), p(dem), p(cap), p(kept),
                         p(owned), sends, ctypes.byref(ns), recvs, ctypes.byref(nr),
                         ctypes.byref(rk), ctypes.byref(ro))
    _check(st, "moe_ep_plan")
    as_list = lambda arr, n: [(c.peer, c.expert, c.row, c.rows) for c in arr[:n]]
    return dict(cap=cap, kept_all=kept, owned_offsets=owned, sends=as_list(sends, ns.value),
                recvs=as_list(recvs, nr.value), rows_kept=int(rk.value),
                rows_owned=int(ro.value), first_expert=moe_ep_first_expert(world, rank, E),
                n_owned=e_own)


def moe_ep_workspace_size(cfg: moe_config, world: int) -> int:
    return int(lib.moe_ep_workspace_size(ctypes.byref(cfg), int(world)))


def alloc_ep_workspace(cfg: moe_config, world: int, device="cuda") -> torch.Tensor:
    size = moe_ep_workspace_size(cfg, world)
    if size == 0:
        raise MoeError(MOE_ERR_INVALID_ARG, "moe_ep_workspace_size")
    ws = torch.empty(size + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + size]
    moe_workspace_init(ws)
    return ws


def moe_permute_ep(cfg, *, ids, cap, x, offsets, row_token=None, slot_row, xp, counts=None,
                   drop_mask=None, ws, stream=None):
    """Permutation with a per-expert capacity (device int32 [E]) into the send layout."""
    st = lib.moe_permute_ep(ctypes.byref(cfg), _ptr(ids), _ptr(cap), _ptr(x), _ptr(offsets),
                            _ptr(row_token), _ptr(slot_row), _ptr(xp), _ptr(counts),
                            _ptr(drop_mask), _ptr(ws), _stream(stream))
    _check(st, "moe_permute_ep")


def moe_ep_expert_ffn(cfg, world: int, rank: int, n_tokens: int, rows: int, *, xr,
                      owned_offsets, x=None, W_gu, W_down, ye, y=None, ws, stream=None):
    """The owner's experts on the received rows (and the shared expert on its own tokens).
    ``cfg`` is the configuration the workspace was sized with (N = most tokens per rank)."""
    st = lib.moe_ep_expert_ffn(ctypes.byref(cfg), int(world), int(rank), int(n_tokens),
                               int(rows), _ptr(xr),
                               _ptr(owned_offsets), _ptr(x), _ptr(W_gu), _ptr(W_down), _ptr(ye),
                               _ptr(y), _ptr(ws), _stream(stream))
    _check(st, "moe_ep_expert_ffn")


def moe_ep_combine(cfg, *, ye, slot_row, gates, y, stream=None):
    """The combine on the token's rank (adds to the shared rows already in y)."""
    st = lib.moe_ep_combine(ctypes.byref(cfg), _ptr(ye), _ptr(slot_row), _ptr(gates), _ptr(y),
                            _stream(stream))
    _check(st, "moe_ep_combine")


def moe_ep_copy_runs(src, *, dst_base, dst_rows, runs, ws=None, stream=None):
    """Copy row runs of ``src`` [rows][d] into the buffers ``dst_base`` (device int64 tensor
    of addresses, as from ``ipc_open`` or ``tensor.data_ptr()``) of sizes ``dst_rows`` (device
    int64 tensor, rows): ``runs`` is a list of (src_row, dst_buf, dst_row, rows)."""
    runs = [tuple(int(v) for v in r) for r in runs if int(r[3]) > 0]
    if not runs:
        return
    dev = src.device
    run_t = torch.tensor(runs, dtype=torch.int32).to(dev, non_blocking=True)
    start = [0]
    for r in runs:
        start.append(start[-1] + r[3])
    start_t = torch.tensor(start, dtype=torch.int32).to(dev, non_blocking=True)
    row_bytes = src.shape[1] * src.element_size()
    st = lib.moe_ep_copy_runs(_ptr(src), src.shape[0], _ptr(dst_base), _ptr(dst_rows),
                              dst_base.numel(), _ptr(run_t), _ptr(start_t), len(runs),
                              start[-1], row_bytes, _ptr(ws), _stream(stream))
    _check(st, "moe_ep_copy_runs")


def moe_permute_ep_p2p(cfg, *, ids, cap, x, offsets, slot_row, dst_base, dst_row0, dst_rows,
                       counts=None, drop_mask=None, ws, stream=None):
    """moe_permute_ep with expert e's kept rows written into rows dst_row0[e]... of the
    buffer at dst_base[e] (device int64 [E] addresses, int32 [E] first rows, int64 [E] sizes)."""
    st = lib.moe_permute_ep_p2p(ctypes.byref(cfg), _ptr(ids), _ptr(cap), _ptr(x), _ptr(offsets),
                                _ptr(slot_row), _ptr(dst_base), _ptr(dst_row0), _ptr(dst_rows),
                                _ptr(counts), _ptr(drop_mask), _ptr(ws), _stream(stream))
    _check(st, "moe_permute_ep_p2p")


def moe_ep_combine_p2p(cfg, *, ids, slot_row, gates, offsets, src_base, src_row0, src_rows, y,
                       ws, stream=None):
    """moe_ep_combine reading slot (t, j)'s expert output (expert e = ids[t, j], send-layout
    row r) at row src_row0[e] + r - offsets[e] of the buffer at src_base[e] (device int64 [E]
    addresses, int32 [E] first rows, int64 [E] sizes)."""
    st = lib.moe_ep_combine_p2p(ctypes.byref(cfg), _ptr(ids), _ptr(slot_row), _ptr(gates),
                                _ptr(offsets), _ptr(src_base), _ptr(src_row0), _ptr(src_rows),
                                _ptr(y), _ptr(ws), _stream(stream))
    _check(st, "moe_ep_combine_p2p")


def ipc_handle(t: torch.Tensor):
    """(64-byte CUDA IPC handle of the allocation holding ``t``, ``t``'s byte offset in it)."""
    h = ctypes.create_string_buffer(64)
    off = _i64(0)
    _check(lib.moe_ipc_handle(_ptr(t), h, ctypes.byref(off)), "moe_ipc_handle")
    return bytes(h.raw), int(off.value)


def ipc_open(handle: bytes) -> int:
    """Map another process's allocation; returns its base address in this process."""
    if len(handle) != 64:
        raise ValueError("a CUDA IPC handle is 64 bytes")
    base = _vp()
    _check(lib.moe_ipc_open(ctypes.create_string_buffer(handle, 64), ctypes.byref(base)),
           "moe_ipc_open")
    return int(base.value)


def ipc_close(base: int) -> None:
    _check(lib.moe_ipc_close(_vp(base)), "moe_ipc_close")


# ---- debugging aid -------------------------------------------------------------------------
def moe_check_dispatch_host(N, k, E, capacity, *, ids, drop_mask, counts, offsets, slot_row,
                            demand=None, row_token=None):
    """Invariants of a dispatch layout, on host (numpy) arrays.  Returns (status, message)."""
    import numpy as np
    a = lambda v, dt: None if v is None else np.ascontiguousarray(np.asarray(v, dtype=dt))
    arrs = [a(ids, np.int32), a(drop_mask, np.uint8), a(counts, np.int32), a(demand, np.int32),
            a(offsets, np.int32), a(slot_row, np.int32), a(row_token, np.int32)]
    p = [None if v is None else v.ctypes.data_as(ctypes.c_void_p) for v in arrs]
    msg = ctypes.create_string_buffer(256)
    st = lib.moe_check_dispatch_host(int(N), int(k), int(E), int(capacity), *p, msg, 256)
    return int(st), msg.value.decode()


def moe_check_dispatch(cfg, *, ids, drop_mask, counts, offsets, slot_row, demand=None,
                       row_token=None, stream=None):
    """The same check on device tensors (synchronises); raises MoeError on a broken one."""
    st = lib.moe_check_dispatch(ctypes.byref(cfg), _ptr(ids), _ptr(drop_mask), _ptr(counts),
                                _ptr(demand), _ptr(offsets), _ptr(slot_row), _ptr(row_token),
                                _stream(stream))
    _check(st, "moe_check_dispatch")
