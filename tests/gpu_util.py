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


def small_dispatch(N, k):
    """Whether the library takes its one-launch dispatch for a batch of N tokens (the rule of
    moe::use_small_dispatch: N <= 64 and N * k <= 1024)."""
    return 0 < N <= 64 and N * k <= 1024


def forward_launches(N, k, E=8, S=0, bf16=True):
    """Kernel launches of one moe_forward: router GEMM, top-k, the rank, scan and scatter
    passes (one launch for all three in a small batch), gate/up and down GEMMs, combine; with
    a shared expert (bf16) its own gate/up and down GEMMs on the side stream."""
    n = 6 if small_dispatch(N, k) else 8
    return n + (2 if S and bf16 and N > 0 and k <= 2 else 0)


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


def _key_gaps(logits_o, logits_g, score_fn, bias, modality):
    eps = 8 * float(np.abs(logits_g.astype(np.float64) - logits_o.astype(np.float64)).max()) + 1e-6
    keys = O.selection_keys(logits_o, score_fn, bias, modality).astype(np.float64)
    if score_fn == O.SIGMOID:
        eps = eps * 0.25 + 1e-6          # |d sigma / dz| <= 1/4
    srt = -np.sort(-keys, axis=1)
    return srt[:, :-1] - srt[:, 1:], eps


def fragile_tokens(logits_o, logits_g, k, score_fn, bias=None, modality=None):
    """Tokens whose top-k set could change under the observed logit discrepancy: the k-th
    and (k+1)-th largest keys lie within twice the largest possible key error."""
    if k >= logits_o.shape[1]:
        return np.zeros(logits_o.shape[0], bool)
    gaps, eps = _key_gaps(logits_o, logits_g, score_fn, bias, modality)
    return gaps[:, k - 1] <= 2 * eps


def order_fragile_tokens(logits_o, logits_g, k, score_fn, bias=None, modality=None):
    """Tokens whose slot order (descending key) could change: two of the k largest keys lie
    within twice the largest possible key error."""
    if k < 2:
        return np.zeros(logits_o.shape[0], bool)
    gaps, eps = _key_gaps(logits_o, logits_g, score_fn, bias, modality)
    return (gaps[:, :k - 1] <= 2 * eps).any(axis=1)


def explain_routing_differences(route_g, info, logits_o, logits_g, k, score_fn, bias=None,
                                modality=None, capacity=0):
    """Checks that every token routed differently from independently computed logits is
    explained by the logit discrepancy, and returns the mask of tokens routed alike.

    * a token whose expert *set* differs must be fragile (its k-th and (k+1)-th keys within
      the key error);
    * a token with the same set in another slot order must be order-fragile;
    * a token with the same ids but another drop mask is a capacity knock-on: an expert that
      a token leaves (and the one it joins instead) sees every later token's rank move by
      one, which moves its keep/drop boundary by one token, so there are at most two such
      tokens per expert exchanged (none without a capacity).  Ranks count demand, not kept
      rows, so knock-ons do not chain.
    """
    ids_g, ids_o = np.asarray(route_g["ids"]), np.asarray(info["ids"])
    same_ids = (ids_g == ids_o).all(1)
    same_set = (np.sort(ids_g, 1) == np.sort(ids_o, 1)).all(1)
    same_drop = (np.asarray(route_g["drop_mask"]) == np.asarray(info["drop_mask"])).all(1)
    frag = fragile_tokens(logits_o, logits_g, k, score_fn, bias, modality)
    ofrag = order_fragile_tokens(logits_o, logits_g, k, score_fn, bias, modality)
    set_changed = ~same_set
    assert frag[set_changed].all(), np.nonzero(set_changed & ~frag)[0][:10]
    assert ofrag[same_set & ~same_ids].all(), np.nonzero(same_set & ~same_ids & ~ofrag)[0][:10]
    knock_on = same_ids & ~same_drop
    # experts a changed token left (each such move also adds one expert it joined)
    moves = sum(len(set(ids_o[t].tolist()) - set(ids_g[t].tolist()))
                for t in np.nonzero(set_changed)[0])
    allowed = 2 * moves if capacity > 0 else 0
    assert int(knock_on.sum()) <= allowed, (int(knock_on.sum()), moves)
    return same_ids & same_drop, dict(set_changed=int(set_changed.sum()),
                                      order_changed=int((same_set & ~same_ids).sum()),
                                      knock_on=int(knock_on.sum()), fragile=int(frag.sum()))
