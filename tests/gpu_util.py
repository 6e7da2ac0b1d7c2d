"""Helpers of the GPU parity tests: run the C ABI on torch tensors, compare with the oracle."""
import numpy as np
import torch

import oracle as O
from mixture_experts_layer_50_b200 import _native as nat
from mixture_experts_layer_50_b200 import workloads as W


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t):
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy()


def f64(t):
    return W.bf16_to_f64(t)


def check_status(ws):
    st = nat.moe_check_status(ws)
    assert st == 0, f"device status {nat.STATUS_NAMES.get(st, st)}"


def gpu_route(cfg, logits, bias=None, modality=None):
    """moe_route on given fp32 logits; returns numpy outputs."""
    N, E, k = cfg.N, cfg.E, cfg.k
    ws = nat.alloc_workspace(cfg)
    out = dict(ids=torch.empty((N, k), dtype=torch.int32, device="cuda"),
               gates=torch.empty((N, k), dtype=torch.float32, device="cuda"),
               counts=torch.empty(E, dtype=torch.int32, device="cuda"),
               demand=torch.empty(E, dtype=torch.int32, device="cuda"),
               drop_mask=torch.empty((N, k), dtype=torch.uint8, device="cuda"))
    nat.moe_route(cfg, logits=dev(logits), bias=None if bias is None else dev(bias),
                  modality=None if modality is None else dev(modality), ws=ws, **out)
    check_status(ws)
    return {kk: host(v) for kk, v in out.items()}


def assert_route_equal(got, logits, k, score_fn, renorm, bias, modality, E, C):
    ids_o, gates_o = O.route(logits, k, score_fn, renorm, bias, modality)
    d_o = O.dispatch(ids_o, E, C)
    np.testing.assert_array_equal(got["ids"], ids_o)
    np.testing.assert_array_equal(got["demand"], d_o["demand"])
    np.testing.assert_array_equal(got["counts"], d_o["counts"])
    np.testing.assert_array_equal(got["drop_mask"], d_o["drop_mask"])
    rel = np.abs(got["gates"] - gates_o) / np.maximum(np.abs(gates_o), 1e-30)
    assert rel.max() <= 1e-5, rel.max()
    return ids_o, gates_o, d_o


def err_stats(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    scale = np.abs(ref).max()
    rms_rel = np.sqrt((err ** 2).mean()) / max(np.sqrt((ref ** 2).mean()), 1e-300)
    return err.max() / max(scale, 1e-300), rms_rel


def assert_close_layer(got, ref, bf16=True):
    """Layer-output bar: max|err| <= 2e-2 max|ref| (bf16 GEMMs) or <= 1e-4 absolute (fp32)."""
    if bf16:
        mx, rms = err_stats(got, ref)
        assert mx <= 2e-2, f"max err {mx:.3e} x max|ref|"
        assert rms <= 1e-2, f"rms relative error {rms:.3e}"
    else:
        err = np.abs(np.asarray(got, np.float64) - ref).max()
        assert err <= 1e-4, err


def fragile_tokens(logits_o, logits_g, k, score_fn, bias=None, modality=None):
    """Tokens whose top-k set could change under the observed logit discrepancy."""
    eps = 8 * float(np.abs(logits_g.astype(np.float64) - logits_o.astype(np.float64)).max()) + 1e-6
    keys = O.selection_keys(logits_o, score_fn, bias, modality).astype(np.float64)
    if score_fn == O.SIGMOID:
        eps = eps * 0.25 + 1e-6          # |d sigma / dz| <= 1/4
    srt = -np.sort(-keys, axis=1)
    if k >= keys.shape[1]:
        return np.zeros(keys.shape[0], bool)
    gap = srt[:, k - 1] - srt[:, k]
    return gap <= 2 * eps
