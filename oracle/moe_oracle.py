"""CPU oracle for the forward pass of a Mixture-of-Experts FFN layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The
library itself never calls it, and it shares no code with the CUDA path.

It is a plain, slow, float64 restatement of what the pages define, written to be
checked against them by eye.  Library primitives used as single steps: numpy
matmul (fp64), a stable argsort, cumulative sums.

Sources (page title, section):

* [P1] "Le groupe d'experts (MoE)", AI Engineering from Scratch, Phase 07 lesson
  11: "Le swap FFN", "Le problème de l'équilibre de la charge", "Des experts
  partagés", "Étape 1: le routeur".
* [P2] "Mixture-of-Experts : routage et capacité" (Applied AI session 19 slides):
  "L'idée — Routeur", "L'idée — Top-k et mélange", "L'idée — Capacité",
  "Support visuel — Capacité", "Cas guidé — trace complète", and the trainer
  answer notes.
* [P3] "Mixture-of-Experts" (DeepSeek-V4.1-Flash, fondations 03): "Le
  mécanisme", the table "Les chiffres de DeepSeek-V4.1-Flash", "Le compte des
  paramètres", "L'équilibrage de charge", "La nouveauté de V4.1 : l'équilibrage
  par modalité".
* [P4] "Mixture of Experts" (dataistudio): the NumPy listing "couche Mixture of
  Experts en Python".
* [P5] "Основы MoE" (ai.flicky.cc, stage 5.3 lesson 01): "Как устроен MoE-слой"
  (steps 1-4 and the numeric example), "Практика" (the ``topk_route``
  contract), "Эксперимент на PyTorch".

Readings where the pages are silent:

* R1  top-k keys: softmax scoring selects on ``z + b`` (the raw logit, plus the
      selection bias when there is one, as P1's ``route`` does); with no bias
      this is the same set as the top-k of ``softmax(z)`` (P5 step 2).  Sigmoid
      scoring selects on ``fl32(fl32(sigma(z)) + b)``.
* R2  ties go to the lower expert index, and the ids are listed by descending
      key (P5 ``topk_route`` docstring: stable argsort of ``-p``).
* R3  sigma in float32 is evaluated with an exp built from Cody & Waite's range
      reduction (two-part ln 2) and a degree-7 Taylor polynomial, every step a
      correctly rounded float32 operation, arguments clipped to [-80, 80].
      Both sides implement this independently so that selection on sigmoid
      keys is reproducible bit for bit.
* R4  gates: softmax + renorm = softmax over the selected unbiased logits
      (P1 ``route``, P4 listing, equal to P5 step 3); renorm=0 gives the raw
      full-softmax probability (P5: Switch k=1); sigmoid + renorm = s_i / sum
      of the selected unbiased s (P3 "L'équilibrage de charge": gates come from
      the unbiased scores).
* R5  capacity C = ceil(T*k/E*f) (P2 "L'idée — Capacité"); assignments to one
      expert are served in token order (P2 trainer notes: arrival order); the
      first C are kept; a dropped slot contributes 0 and the surviving gates are
      not renormalised (P2 trace: t6 keeps only 0.426).
* R6  SwiGLU expert FFN(x) = (SiLU(x W_gate) * (x W_up)) W_down, three matrices
      (P3 "Le compte des paramètres"; P5 ``w1, w2, w3``); the "clipped at 10" of
      the P3 table is read as clamping both the gate and the up pre-activation
      to [-10, 10] before SiLU(gate) * up.  ReLU expert: max(x W1, 0) W2 (P4).
* R7  the shared expert has weight 1, outside the renormalisation (P2 trainer
      notes; P1 "Des experts partagés"); no residual and no norm inside the layer
      (P5 step 4 defines y without them).
* R8  router logits are float32 (the fp64 dot product rounded once); an
      optional per-expert logit offset is added before that rounding (the skewed
      capacity workload).

* R11 the balance statistic's P_i for sigmoid scoring averages the affinities
      normalised per token to sum 1 (the pages print the formula for softmax only).
* R12 the bias update compares each expert's load with its set's mean load
      (total / E) exactly, in integers; gamma = 0.001 (both pages' update rate).
* R14 overflow policy "report" (P2 table "Politiques de débordement quand E1 reçoit
      6 tokens pour C = 5", row "Report sur E2/E3": the token is handled by its
      third-best score).  After the capacity pass, a token's i-th dropped slot (slot
      order, i = 0, 1, ...) is offered its (k+i)-th best expert by selection key (the
      third best for top-2).  Offers to one expert are served in token order, then
      slot order, while the expert's kept count plus the offers it took stays below
      C; an offer that finds no room leaves the slot dropped.  The gates are those of
      R4 over the token's final slot list (a moved slot takes its new expert's score;
      a slot still dropped stays in the list and contributes 0, as in R5).

Parity unpinned: the clamp (R6) beyond unit values, the whole-layer output beyond
brute force and closed forms -- no page prints a layer output -- the hash
router (a reading of an exercise, pinned only by bijectivity and uniformity), and
the "report" overflow policy (R14) beyond the slides' one-token example.
"""
from __future__ import annotations

import math
from fractions import Fraction
from typing import Optional

import numpy as np

SOFTMAX, SIGMOID = 0, 1
SWIGLU, RELU = 0, 1

# ---------------------------------------------------------------------------
# float32 exp / sigmoid (reading R3)
# ---------------------------------------------------------------------------
_f32 = np.float32
_LN2 = math.log(2.0)
# ln 2 split in two (Cody & Waite): the high part keeps 16 significant bits so
# that n * LN2_HI is exact for |n| < 2^8; the low part is the float32 remainder.
_LN2_HI = _f32(round(_LN2 * 65536.0) / 65536.0)
_LN2_LO = _f32(_LN2 - float(_LN2_HI))
_INV_LN2 = _f32(1.0 / _LN2)
# Taylor coefficients 1/i! for i = 0..7, each rounded to float32.
_TAYLOR = [_f32(1.0 / math.factorial(i)) for i in range(8)]
_SIG_CLIP = _f32(80.0)


def exp_f32(x) -> np.ndarray:
    """float32 e^x by range reduction x = n ln2 + r and a Taylor polynomial in r.

    Valid for |x| <= 80 (the sigmoid clips its argument there).  Every
    operation below is one correctly rounded float32 operation.
    """
    x = np.asarray(x, dtype=_f32)
    n = np.rint(x * _INV_LN2).astype(_f32)
    r = (x - n * _LN2_HI) - n * _LN2_LO
    p = _TAYLOR[7]
    for c in _TAYLOR[6::-1]:
        p = p * r + c
    return np.ldexp(p, n.astype(np.int32)).astype(_f32)


def sigmoid_f32(z) -> np.ndarray:
    """float32 sigma(z) = 1 / (1 + e^-z), with z clipped to [-80, 80] (R3)."""
    z = np.clip(np.asarray(z, dtype=_f32), -_SIG_CLIP, _SIG_CLIP)
    e = exp_f32(-z)
    return (_f32(1.0) / (_f32(1.0) + e)).astype(_f32)


# ---------------------------------------------------------------------------
# step 1: router projection  (P5 "Как устроен MoE-слой", step 1; P1 Étape 1)
# ---------------------------------------------------------------------------
def router_logits(x, W_g, logit_offset=None) -> np.ndarray:
    """z = x . W_g in float64, plus an optional per-expert offset, rounded to float32.

    ``x`` is [N][d]; ``W_g`` is stored [E][d] (so the math ``d x E`` matrix is its
    transpose).  Returns float32 [N][E] (reading R8).
    """
    z = np.asarray(x, np.float64) @ np.asarray(W_g, np.float64).T
    if logit_offset is not None:
        z = z + np.asarray(logit_offset, np.float64)[None, :]
    return z.astype(np.float32)


# ---------------------------------------------------------------------------
# steps 2-3: scores, top-k and gates  (P5 steps 2-3; P1 route(); P3 balancing)
# ---------------------------------------------------------------------------
def softmax64(z) -> np.ndarray:
    """Row softmax in float64: exp(z - max) / sum exp(z - max)."""
    z = np.asarray(z, np.float64)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def selection_keys(logits, score_fn, bias=None, modality=None) -> np.ndarray:
    """float32 selection keys (readings R1, R3).

    bias is [n_sets][E]; a token t uses set ``modality[t]`` (P3: one bias set per
    modality, text = 0, image = 1).  With a single set every token uses set 0.
    """
    z = np.asarray(logits, np.float32)
    base = z if score_fn == SOFTMAX else sigmoid_f32(z)
    if bias is None:
        return base.astype(np.float32)
    bias = np.asarray(bias, np.float32)
    if modality is None:
        per_token = np.broadcast_to(bias[0], z.shape)
    else:
        per_token = bias[np.asarray(modality, np.int64)]
    return (base + per_token).astype(np.float32)


def topk_ids(keys, k) -> np.ndarray:
    """The k largest keys per row, listed by descending key, ties to the lower index (R2)."""
    order = np.argsort(-np.asarray(keys, np.float32), axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gates_for(logits, ids, score_fn, renorm) -> np.ndarray:
    """Gate weights of the selected experts, in float64 from the unbiased scores (R4)."""
    z = np.asarray(logits, np.float64)
    sel = np.take_along_axis(z, ids.astype(np.int64), axis=1)
    if score_fn == SOFTMAX:
        if renorm:
            # softmax over the chosen original logits (P1 route, P4 listing)
            e = np.exp(sel - sel.max(axis=1, keepdims=True))
            return e / e.sum(axis=1, keepdims=True)
        # Switch k=1: the full-softmax probability itself (P5)
        return np.take_along_axis(softmax64(z), ids.astype(np.int64), axis=1)
    s = 1.0 / (1.0 + np.exp(-sel))
    if renorm:
        return s / s.sum(axis=1, keepdims=True)
    return s


def route(logits, k, score_fn=SOFTMAX, renorm=1, bias=None, modality=None):
    """Routing of P5 steps 1-3: returns (ids [N][k] int32, gates [N][k] float64)."""
    keys = selection_keys(logits, score_fn, bias, modality)
    ids = topk_ids(keys, k)
    return ids, gates_for(logits, ids, score_fn, renorm)


# ---------------------------------------------------------------------------
# capacity, dropping and the per-expert permutation  (P2 "Capacité"; R5)
# ---------------------------------------------------------------------------
def capacity(T: int, k: int, E: int, cf) -> int:
    """C = ceil(T * k / E * f) in exact rational arithmetic; cf None means no limit (-> 0)."""
    if cf is None:
        return 0
    q = Fraction(T * k, E) * Fraction(cf)
    return -((-q.numerator) // q.denominator)


def dispatch(ids, E: int, C: int = 0):
    """Capacity check in token order and the contiguous per-expert row layout.

    rank(t, e) = number of earlier tokens t' < t that chose e.  An assignment is
    kept iff C <= 0 or rank < C.  Kept rows are laid out expert by expert, each
    expert's tokens in increasing token order.

    Returns a dict: demand [E], counts [E], offsets [E+1], row_token [M],
    slot_row [N][k] (-1 = dropped), drop_mask [N][k] (uint8).
    """
    ids = np.asarray(ids, np.int64)
    N, k = ids.shape
    chose = np.zeros((N, E), np.int64)
    np.put_along_axis(chose, ids, 1, axis=1)
    rank_all = np.cumsum(chose, axis=0) - chose          # exclusive: earlier tokens only
    rank = np.take_along_axis(rank_all, ids, axis=1)
    demand = chose.sum(axis=0)
    keep = rank < C if C > 0 else np.ones_like(rank, dtype=bool)
    counts = np.minimum(demand, C) if C > 0 else demand.copy()
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    slot_row = np.where(keep, offsets[ids] + rank, -1)
    row_token = np.full(int(offsets[-1]), -1, np.int64)
    t_idx = np.broadcast_to(np.arange(N)[:, None], ids.shape)
    row_token[slot_row[keep]] = t_idx[keep]
    return {
        "demand": demand.astype(np.int32),
        "counts": counts.astype(np.int32),
        "offsets": offsets.astype(np.int32),
        "row_token": row_token.astype(np.int32),
        "slot_row": slot_row.astype(np.int32),
        "drop_mask": (~keep).astype(np.uint8),
    }


def dispatch_masked(ids, E: int, drop_mask):
    """The contiguous per-expert layout of the assignments not marked in ``drop_mask``
    (no capacity of its own): kept rows expert by expert, token order inside an expert.
    Returns the same keys as ``dispatch``; ``demand`` counts the kept assignments."""
    ids = np.asarray(ids, np.int64)
    keep = np.asarray(drop_mask) == 0
    N, k = ids.shape
    counts = np.zeros(E, np.int64)
    np.add.at(counts, ids[keep], 1)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    slot_row = np.full((N, k), -1, np.int64)
    row_token = np.full(int(offsets[-1]), -1, np.int64)
    fill = offsets[:-1].copy()
    for t in range(N):                 # token order, then slot order
        for j in range(k):
            if keep[t, j]:
                e = ids[t, j]
                slot_row[t, j] = fill[e]
                row_token[fill[e]] = t
                fill[e] += 1
    return {"demand": counts.astype(np.int32), "counts": counts.astype(np.int32),
            "offsets": offsets.astype(np.int32), "row_token": row_token.astype(np.int32),
            "slot_row": slot_row.astype(np.int32), "drop_mask": (~keep).astype(np.uint8)}


def route_reroute(logits, k, C, score_fn=SOFTMAX, renorm=1, bias=None, modality=None):
    """Routing under the "report" overflow policy (reading R14).

    Returns (ids [N][k] int32: the final expert of every slot, gates [N][k] float64,
    drop_mask [N][k] uint8: slots still dropped, rerouted [N][k] uint8: slots moved to
    another expert, first: the ``dispatch`` result of the plain capacity pass)."""
    keys = selection_keys(logits, score_fn, bias, modality)
    N, E = keys.shape
    order = topk_ids(keys, min(E, 2 * k))      # descending key, lower index on ties
    ids = order[:, :k].astype(np.int32).copy()
    first = dispatch(ids, E, C)
    drop = first["drop_mask"].astype(bool).copy()
    rerouted = np.zeros((N, k), bool)
    kept = first["counts"].astype(np.int64)
    taken = np.zeros(E, np.int64)
    for t in range(N):                         # token order
        i = 0
        for j in range(k):                     # slot order
            if not drop[t, j]:
                continue
            if k + i < order.shape[1]:
                e = int(order[t, k + i])
                if kept[e] + taken[e] < C:
                    taken[e] += 1
                    ids[t, j] = e
                    drop[t, j] = False
                    rerouted[t, j] = True
            i += 1
    gates = gates_for(logits, ids, score_fn, renorm)
    return ids, gates, drop.astype(np.uint8), rerouted.astype(np.uint8), first


def dispatch_padded(ids, E: int, C: int):
    """The padded dispatch buffer [E, C, d] of the slides ("Support visuel — Capacité"): slot
    c of expert e holds the c-th kept token (token order), empty slots stay empty.
    Returns slot_row [N][k] (e*C + rank, -1 = dropped), row_token [E*C] (-1 = empty slot),
    counts [E], drop_mask [N][k]."""
    if C <= 0:
        raise ValueError("the padded layout needs a capacity")
    d = dispatch(ids, E, C)
    ids = np.asarray(ids, np.int64)
    keep = d["drop_mask"] == 0
    rank = d["slot_row"] - d["offsets"][ids]           # rank inside the expert, for kept ones
    slot = np.where(keep, ids * C + rank, -1)
    row_token = np.full(E * C, -1, np.int64)
    t_idx = np.broadcast_to(np.arange(ids.shape[0])[:, None], ids.shape)
    row_token[slot[keep]] = t_idx[keep]
    return {"slot_row": slot.astype(np.int32), "row_token": row_token.astype(np.int32),
            "counts": d["counts"], "drop_mask": d["drop_mask"]}


def load_fractions(ids, E: int):
    """Per-expert load: bincount/N (P4 listing, sums to k) and count/(T k) (P5, sums to 1)."""
    ids = np.asarray(ids, np.int64)
    cnt = np.bincount(ids.ravel(), minlength=E).astype(np.float64)
    return cnt / ids.shape[0], cnt / ids.size


# ---------------------------------------------------------------------------
# expert FFN  (R6)
# ---------------------------------------------------------------------------
def silu(a):
    return a / (1.0 + np.exp(-a))


def expert_ffn(xr, W_gu_e, W_down_e, act=SWIGLU, clamp=0.0):
    """One expert on rows ``xr`` [m][d], float64.

    SwiGLU: W_gu_e is [2F][d] (gate rows then up rows), W_down_e is [d][F].
    ReLU:   W_gu_e is [F][d] (W1 stored out-major), W_down_e is [d][F].
    """
    xr = np.asarray(xr, np.float64)
    Wgu = np.asarray(W_gu_e, np.float64)
    Wd = np.asarray(W_down_e, np.float64)
    if act == SWIGLU:
        F = Wgu.shape[0] // 2
        g = xr @ Wgu[:F].T
        u = xr @ Wgu[F:].T
        if clamp > 0:
            g = np.clip(g, -clamp, clamp)
            u = np.clip(u, -clamp, clamp)
        h = silu(g) * u
    else:
        h = np.maximum(xr @ Wgu.T, 0.0)
    return h @ Wd.T


# ---------------------------------------------------------------------------
# the whole layer  (P5 step 4; P2 "Top-k et mélange"; R7)
# ---------------------------------------------------------------------------
def forward(x, W_g, W_gu, W_down, *, k, E, score_fn=SOFTMAX, renorm=1, act=SWIGLU,
            clamp=0.0, n_shared=0, bias=None, modality=None, logit_offset=None,
            C=0, logits=None, tokens=None, ids=None, gates=None, overflow="drop"):
    """y[t] = sum_{kept j} g[t,j] FFN_{ids[t,j]}(x_t) + sum_shared FFN_s(x_t), float64.

    ``logits`` (float32 [N][E]) replaces the router projection when given.
    ``ids`` and ``gates`` ([N][k]) replace the whole router when given: forced or
    replayed routing ("Le groupe d'experts (MoE)", exercise "Hard": record the experts
    that fired and force the same routing later); capacity still applies.
    ``tokens`` restricts the expert work and the returned rows to those token
    indices; routing and capacity still see every token.
    ``overflow="reroute"`` applies the "report" overflow policy (reading R14) to the
    router's choice instead of dropping.
    Returns (y [len(tokens) or N][d] float64, route dict).
    """
    x64 = np.asarray(x, np.float64)
    N = x64.shape[0]
    if ids is not None:
        z = None
        ids = np.asarray(ids, np.int32)
        gates = np.asarray(gates, np.float64)
    elif overflow == "reroute":
        z = router_logits(x64, W_g, logit_offset) if logits is None else np.asarray(logits, np.float32)
        ids, gates, drop, rerouted, first = route_reroute(z, k, C, score_fn, renorm, bias,
                                                          modality)
    else:
        z = router_logits(x64, W_g, logit_offset) if logits is None else np.asarray(logits, np.float32)
        ids, gates = route(z, k, score_fn, renorm, bias, modality)
    if overflow == "reroute" and ids is not None and z is not None:
        disp = dispatch_masked(ids, E, drop)
        disp["demand"] = first["demand"]
        disp["rerouted"] = rerouted
    else:
        disp = dispatch(ids, E, C)
    keep = disp["drop_mask"] == 0
    tok = np.arange(N) if tokens is None else np.asarray(tokens, np.int64)
    y = np.zeros((tok.size, x64.shape[1]), np.float64)
    for e in range(E):
        sel_t, sel_j = np.nonzero((ids[tok] == e) & keep[tok])
        if sel_t.size == 0:
            continue
        out = expert_ffn(x64[tok[sel_t]], W_gu[e], W_down[e], act, clamp)
        np.add.at(y, sel_t, gates[tok[sel_t], sel_j][:, None] * out)
    for s in range(n_shared):
        y += expert_ffn(x64[tok], W_gu[E + s], W_down[E + s], act, clamp)
    info = {"logits": z, "ids": ids, "gates": gates, **disp}
    return y, info


# ---------------------------------------------------------------------------
# balancing statistics and the aux-loss-free bias update
# ---------------------------------------------------------------------------
def router_probs(logits, score_fn):
    """Per-token router probabilities over all experts: softmax(z), or for sigmoid scoring
    the affinities s = sigma(z) normalised to sum 1 (reading R11)."""
    z = np.asarray(logits, np.float64)
    if score_fn == SOFTMAX:
        return softmax64(z)
    s = 1.0 / (1.0 + np.exp(-z))
    return s / s.sum(axis=1, keepdims=True)


def balance_stats(logits, ids, E, score_fn=SOFTMAX):
    """Switch balance statistic ("Основы MoE", "Вспомогательный лосс Switch Transformer"):
    f_i = share of the top-k assignments that went to expert i (sums to 1), P_i = mean
    router probability of expert i over the tokens, aux = E * sum_i f_i P_i (the loss is
    alpha * aux).  Returns (f, P, aux) in float64."""
    ids = np.asarray(ids, np.int64)
    f = np.bincount(ids.ravel(), minlength=E) / ids.size
    P = router_probs(logits, score_fn).mean(axis=0)
    return f, P, float(E * np.sum(f * P))


def per_set_load(ids, E, modality=None, n_sets=1):
    """Assignments per (bias set, expert): token t counts in set modality[t] (set 0 without flags)."""
    ids = np.asarray(ids, np.int64)
    sets = np.zeros(ids.shape[0], np.int64) if modality is None else np.asarray(modality, np.int64)
    load = np.zeros((n_sets, E), np.int64)
    for m in range(n_sets):
        load[m] = np.bincount(ids[sets == m].ravel(), minlength=E)
    return load


def bias_update(bias, load, gamma=0.001):
    """Aux-loss-free balancing ("Le groupe d'experts (MoE)", "Le problème de l'équilibre de la
    charge"; DeepSeek-V4.1-Flash page, "L'équilibrage de charge" and "l'équilibrage par
    modalité"): after a step each expert's selection bias moves by -gamma when its load is
    above the set's mean load, +gamma when below, unchanged when equal; each bias set uses
    its own loads.  float32 in, float32 out (reading R12: the comparison is exact in
    integers, load_e * E versus the set's total)."""
    bias = np.asarray(bias, np.float32)
    load = np.asarray(load, np.int64)
    E = load.shape[1]
    total = load.sum(axis=1, keepdims=True)
    step = np.sign(total - load * E).astype(np.float32) * np.float32(gamma)
    return (bias + step).astype(np.float32)


def fmix32(h):
    """The 32-bit finaliser of MurmurHash3 (A. Appleby, public domain): a bijection on
    32-bit integers that mixes every input bit into every output bit."""
    h = np.asarray(h, np.uint64) & 0xFFFFFFFF
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & 0xFFFFFFFF
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & 0xFFFFFFFF
    h ^= h >> 16
    return h.astype(np.uint32)


def hash_route(token_ids, E, k):
    """Hash router ("Le groupe d'experts (MoE)", exercise "Medium": deterministic, not
    learned).  Reading: expert e's key for token id t is fmix32(t * 0x9E3779B1 + e) (32-bit
    wrap-around); the k largest keys are selected, listed by descending key (the keys of one
    token are distinct because fmix32 is a bijection); every selected expert gets the gate 1/k.
    Returns (ids [N][k] int32, gates [N][k] float64)."""
    t = np.asarray(token_ids, np.int64).astype(np.uint64) & 0xFFFFFFFF
    e = np.arange(E, dtype=np.uint64)
    keys = fmix32((t[:, None] * 0x9E3779B1 + e[None, :]) & 0xFFFFFFFF).astype(np.int64)
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    return ids, np.full(ids.shape, 1.0 / k)


def dense_mixture(x, W_g, W_gu, W_down, *, E, act=SWIGLU, clamp=0.0, logit_offset=None):
    """The dense limit k = E with softmax: y = sum_e p_e FFN_e(x) (P5 "Практика")."""
    x64 = np.asarray(x, np.float64)
    p = softmax64(router_logits(x64, W_g, logit_offset))
    y = np.zeros_like(x64)
    for e in range(E):
        y += p[:, e:e + 1] * expert_ffn(x64, W_gu[e], W_down[e], act, clamp)
    return y


__all__ = ["exp_f32", "sigmoid_f32", "router_logits", "softmax64", "selection_keys",
           "topk_ids", "gates_for", "route", "capacity", "dispatch", "dispatch_padded",
           "dispatch_masked", "route_reroute",
           "load_fractions",
           "silu", "expert_ffn", "forward", "dense_mixture", "fmix32", "hash_route",
           "router_probs", "balance_stats", "per_set_load", "bias_update",
           "SOFTMAX", "SIGMOID",
           "SWIGLU", "RELU"]
