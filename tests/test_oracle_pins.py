"""Pins of the CPU oracle against what the pages print and what the mathematics fixes.

Each test names the page and section its numbers come from.  A plausible mistake
in the oracle (a dropped term, a sign, a transposed operand, an off-by-one in the
token-order ranks) fails at least one of them.
"""
import math

import numpy as np
import pytest
from scipy.special import expit, softmax as sp_softmax

from golden.reader import floats, ints, load
import oracle as O


# --------------------------------------------------------------------------
# router scores, top-k and gates: printed worked examples
# --------------------------------------------------------------------------
def test_p2_router_softmax_and_renorm():
    g = load("p2_router_example.txt")
    z = np.array([floats(g["logits"])], np.float32)
    np.testing.assert_allclose(np.round(O.softmax64(z)[0], 3), floats(g["softmax"]))
    # the intermediate exponentials and their sum as printed (3 decimals)
    e = np.exp(np.asarray(z[0], np.float64))
    np.testing.assert_allclose(np.round(e, 3), floats(g["exp"]), atol=1.5e-3)
    assert round(float(e.sum()), 3) == pytest.approx(float(g["exp_sum"]), abs=1.5e-3)
    ids, gates = O.route(z, 2)
    assert ids.tolist() == [ints(g["top2_ids"])]
    np.testing.assert_allclose(np.round(gates[0], 3), floats(g["top2_renorm"]))


def test_p2_router_alternative_logits():
    g = load("p2_router_example.txt")
    z = np.array([floats(g["alt_logits"])], np.float32)
    np.testing.assert_allclose(np.round(O.softmax64(z)[0], 3), floats(g["alt_softmax"]))
    ids, _ = O.route(z, 2)
    assert sorted(ids[0].tolist()) == ints(g["alt_top2_set"])


def test_p5_topk_example_and_switch():
    g = load("p5_topk_example.txt")
    z = np.array([floats(g["logits"])], np.float32)
    np.testing.assert_allclose(np.round(O.softmax64(z)[0], 3), floats(g["softmax"]))
    ids, w = O.route(z, 2)
    assert ids.tolist() == [ints(g["top2_ids"])]
    np.testing.assert_allclose(np.round(w[0], 3), floats(g["top2_weights"]))
    # Switch: k = 1 keeps the raw probability
    ids1, w1 = O.route(z, 1, renorm=0)
    assert ids1[0, 0] == int(g["switch_top1_id"])
    assert round(float(w1[0, 0]), 3) == float(g["switch_top1_weight"])
    # whereas renormalising a single weight would give exactly 1
    _, w1r = O.route(z, 1, renorm=1)
    assert w1r[0, 0] == 1.0


def test_softmax_matches_library_routine():
    z = np.random.default_rng(5).normal(0, 3, (50, 17)).astype(np.float32)
    np.testing.assert_allclose(O.softmax64(z), sp_softmax(z.astype(np.float64), axis=1),
                               rtol=1e-13, atol=0)


def test_ties_go_to_lower_index_and_order_is_descending():
    z = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]], np.float32)
    assert O.route(z, 2)[0].tolist() == [[1, 2]]
    assert O.route(z, 4)[0].tolist() == [[1, 2, 4, 3]]
    # all equal: ids 0..k-1 and equal gates 1/k (softmax and sigmoid alike)
    z = np.zeros((3, 6), np.float32)
    for sf in (O.SOFTMAX, O.SIGMOID):
        ids, w = O.route(z, 3, score_fn=sf)
        assert ids.tolist() == [[0, 1, 2]] * 3
        np.testing.assert_allclose(w, 1.0 / 3.0, rtol=1e-15)


def test_topk_brute_force_small():
    """Against an exhaustive ranking written with Python's sort on (-key, index)."""
    rng = np.random.default_rng(11)
    for E, k in ((4, 1), (5, 3), (8, 8), (13, 6)):
        z = np.round(rng.normal(0, 1, (40, E)) * 4) / 4          # many exact ties
        z = z.astype(np.float32)
        ids = O.topk_ids(z, k)
        for t in range(z.shape[0]):
            want = sorted(range(E), key=lambda e: (-float(z[t, e]), e))[:k]
            assert ids[t].tolist() == want


# --------------------------------------------------------------------------
# sigmoid scoring, selection-only bias, modality bias sets
# --------------------------------------------------------------------------
def test_exp_f32_accuracy_and_exact_points():
    x = np.linspace(-80, 80, 400001).astype(np.float32)
    got = O.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(got - ref) / ulp) <= 2.0
    assert O.exp_f32(np.float32(0.0)) == np.float32(1.0)
    assert float(O.exp_f32(np.float32(math.log(2.0)))) == pytest.approx(2.0, rel=2e-7)
    assert float(O.exp_f32(np.float32(-1.0))) == pytest.approx(math.exp(-1.0), rel=1.2e-7)


def test_sigmoid_f32_against_library():
    z = np.linspace(-30, 30, 200001).astype(np.float32)
    got = O.sigmoid_f32(z).astype(np.float64)
    ref = expit(z.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    assert np.max(np.abs(got - ref) / ulp) <= 3.0
    assert O.sigmoid_f32(np.float32(0)) == np.float32(0.5)
    assert O.sigmoid_f32(np.float32(100)) == np.float32(1.0)        # clipped, saturates
    assert 0 < O.sigmoid_f32(np.float32(-100)) < 1e-30


def test_sigmoid_without_bias_selects_like_softmax():
    z = np.random.default_rng(3).normal(0, 1, (500, 32)).astype(np.float32)
    a, _ = O.route(z, 6, score_fn=O.SOFTMAX)
    b, _ = O.route(z, 6, score_fn=O.SIGMOID)
    # sigma is monotone, so the selected sets agree wherever float32 sigma keeps
    # the values distinct (it does for N(0,1) logits)
    assert (np.sort(a, 1) == np.sort(b, 1)).all()


def test_sigmoid_gates_renormalised_from_unbiased_scores():
    z = np.array([[0.5, -1.0, 2.0, 0.0]], np.float32)
    ids, w = O.route(z, 2, score_fn=O.SIGMOID)
    assert ids.tolist() == [[2, 0]]
    s = expit(np.array([2.0, 0.5]))
    np.testing.assert_allclose(w[0], s / s.sum(), rtol=1e-7)


def test_selection_bias_changes_selection_not_gates():
    """A large bias on expert j forces j into every token's set; its gate still uses s_j."""
    rng = np.random.default_rng(4)
    z = rng.normal(0, 1, (200, 16)).astype(np.float32)
    bias = np.zeros((1, 16), np.float32)
    bias[0, 9] = 5.0
    ids, w = O.route(z, 4, score_fn=O.SIGMOID, bias=bias)
    assert (ids[:, 0] == 9).all()
    s = expit(np.take_along_axis(z.astype(np.float64), ids.astype(np.int64), 1))
    np.testing.assert_allclose(w, s / s.sum(1, keepdims=True), rtol=1e-7)
    # softmax scoring with the same bias: gate = softmax over the chosen raw logits
    ids2, w2 = O.route(z, 2, score_fn=O.SOFTMAX, bias=bias)
    assert (ids2[:, 0] == 9).all()
    sel = np.take_along_axis(z.astype(np.float64), ids2.astype(np.int64), 1)
    np.testing.assert_allclose(w2, sp_softmax(sel, axis=1), rtol=1e-12)


def test_modality_picks_its_bias_set():
    z = np.zeros((4, 8), np.float32)
    bias = np.zeros((2, 8), np.float32)
    bias[0, 3] = 1.0      # text favours expert 3
    bias[1, 6] = 1.0      # image favours expert 6
    mod = np.array([0, 1, 1, 0], np.uint8)
    ids, w = O.route(z, 1, score_fn=O.SIGMOID, bias=bias, modality=mod)
    assert ids[:, 0].tolist() == [3, 6, 6, 3]
    np.testing.assert_allclose(w, 1.0)


# --------------------------------------------------------------------------
# capacity and dropping: the slides' full trace
# --------------------------------------------------------------------------
def _trace_logits(assign, E):
    """Token logits that route each token to its printed pair, first expert first.

    The pair gets 2.1 and 1.8 as on t1; the others 0.2 (any value below 1.8 keeps
    the same top-2 and the same renormalised gates).
    """
    z = np.full((len(assign), E), 0.2, np.float32)
    for t, (a, b) in enumerate(assign):
        z[t, a], z[t, b] = 2.1, 1.8
    return z


def _trace():
    g = load("p2_capacity_trace.txt")
    assign = [tuple(int(v) for v in p.split()) for p in g["assign"].split("|")]
    return g, assign, int(g["T"]), int(g["E"]), int(g["k"])


def test_capacity_formula_printed_values():
    g, _, T, E, k = _trace()
    from fractions import Fraction as Fr
    assert O.capacity(T, k, E, Fr(5, 4)) == int(g["C_1.25"])
    assert O.capacity(T, k, E, 1) == int(g["C_1.0"])
    assert O.capacity(T, k, E, 2) == int(g["C_2.0"])
    assert O.capacity(T, 1, E, Fr(5, 4)) == int(g["C_k1"])
    assert O.capacity(T, k, E, Fr(3, 2)) == int(g["C_1.5"])
    assert O.capacity(T, k, E, None) == 0
    # exact ceiling: 100 tokens, k=2, E=64, f=1 -> 200/64 = 3.125 -> 4
    assert O.capacity(100, 2, 64, 1) == 4
    assert O.capacity(128, 2, 64, 1) == 4


def test_capacity_trace_f125_dispatch_table():
    g, assign, T, E, k = _trace()
    z = _trace_logits(assign, E)
    ids, gates = O.route(z, k)
    assert [tuple(r) for r in ids.tolist()] == assign
    d = O.dispatch(ids, E, int(g["C_1.25"]))
    assert d["demand"].tolist() == ints(g["demand_1.25"])
    t_drop, e_drop = (int(v) for v in g["dropped_1.25"].split(":"))
    dropped = [(t, int(ids[t, j])) for t, j in zip(*np.nonzero(d["drop_mask"]))]
    assert dropped == [(t_drop, e_drop)]
    assert int(d["counts"].sum()) == int(g["filled_1.25"])
    assert E * int(g["C_1.25"]) == int(g["slots_1.25"])
    for e in range(E):
        rows = d["row_token"][d["offsets"][e]:d["offsets"][e + 1]]
        assert rows.tolist() == ints(g[f"table_E{e}"])
    # slot_row and row_token are inverse maps on the kept assignments
    for t in range(T):
        for j in range(k):
            r = d["slot_row"][t, j]
            if d["drop_mask"][t, j]:
                assert r == -1
            else:
                assert d["row_token"][r] == t and d["offsets"][ids[t, j]] <= r < d["offsets"][ids[t, j] + 1]
    # the dropped token keeps only its second gate, not renormalised
    j_kept = int(np.nonzero(d["drop_mask"][t_drop] == 0)[0][0])
    assert round(float(gates[t_drop, j_kept]), 3) == float(g["t6_kept_gate"])


@pytest.mark.parametrize("tag,cf,kk", [("1.0", 1, 2), ("2.0", 2, 2), ("1.5", None, 2), ("k1", None, 1)])
def test_capacity_trace_variants(tag, cf, kk):
    from fractions import Fraction as Fr
    g, assign, T, E, k = _trace()
    cf = {"1.0": 1, "2.0": 2, "1.5": Fr(3, 2), "k1": Fr(5, 4)}[tag]
    z = _trace_logits(assign, E)
    ids, _ = O.route(z, kk)
    C = O.capacity(T, kk, E, cf)
    d = O.dispatch(ids, E, C)
    assert C == int(g[f"C_{tag}"])
    assert int(d["drop_mask"].sum()) == int(g[f"drops_{tag}"])
    if f"filled_{tag}" in g:
        assert int(d["counts"].sum()) == int(g[f"filled_{tag}"])
    if f"slots_{tag}" in g:
        assert E * C == int(g[f"slots_{tag}"])
    if tag == "k1":
        assert d["demand"].tolist() == ints(g["demand_k1"])


def test_dispatch_invariants_random():
    rng = np.random.default_rng(9)
    for N, E, k, C in ((1, 4, 2, 0), (129, 8, 2, 20), (300, 64, 6, 5), (50, 3, 3, 0), (64, 5, 2, 1)):
        z = rng.normal(0, 1, (N, E)).astype(np.float32)
        ids, _ = O.route(z, k)
        d = O.dispatch(ids, E, C)
        assert int(d["demand"].sum()) == N * k
        assert int(d["counts"].sum()) + int(d["drop_mask"].sum()) == N * k
        assert (d["row_token"] >= 0).all()
        # brute force ranks: walk the tokens in order with per-expert counters
        seen = [0] * E
        for t in range(N):
            for j in range(k):
                e = int(ids[t, j])
                kept = C <= 0 or seen[e] < C
                assert bool(d["drop_mask"][t, j]) == (not kept)
                if kept:
                    assert d["slot_row"][t, j] == d["offsets"][e] + seen[e]
                seen[e] += 1


def test_load_fractions_sum():
    z = np.random.default_rng(1).normal(0, 1, (1000, 8)).astype(np.float32)
    ids, _ = O.route(z, 2)
    per_n, per_tk = O.load_fractions(ids, 8)
    assert per_n.sum() == pytest.approx(2.0, abs=1e-12)      # dataistudio "Mixture of Experts": bincount / N sums to k
    assert per_tk.sum() == pytest.approx(1.0, abs=1e-12)     # "Основы MoE": count / (T k) sums to 1


# --------------------------------------------------------------------------
# expert FFN and the whole layer: closed forms and brute force
# --------------------------------------------------------------------------
def test_router_logits_orientation():
    x = np.array([[1.0, 2.0]])
    W_g = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])     # stored [E][d]
    np.testing.assert_array_equal(O.router_logits(x, W_g), [[1.0, 2.0, 3.0]])
    np.testing.assert_array_equal(O.router_logits(x, W_g, [0.5, 0, -1]), [[1.5, 2.0, 2.0]])


def test_swiglu_expert_hand_values():
    x = np.array([[1.0, 2.0]])
    W_gu = np.array([[1.0, 0.0],     # gate row (F = 1)
                     [0.0, 1.0]])    # up row
    W_down = np.array([[1.0], [2.0]])  # [d][F]
    silu1 = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(O.expert_ffn(x, W_gu, W_down), [[2 * silu1, 4 * silu1]], rtol=1e-15)
    # clip at 10 on both pre-activations (unit values only; the layer-level clamp is unpinned)
    x = np.array([[20.0, -30.0]])
    want = (10.0 / (1.0 + math.exp(-10.0))) * -10.0
    np.testing.assert_allclose(O.expert_ffn(x, W_gu, W_down, clamp=10.0), [[want, 2 * want]], rtol=1e-15)
    # below the clip the clamp is the identity
    x = np.array([[3.0, -4.0]])
    np.testing.assert_allclose(O.expert_ffn(x, W_gu, W_down, clamp=10.0), O.expert_ffn(x, W_gu, W_down))


def test_relu_expert_hand_values():
    x = np.array([[1.0, -1.0]])
    W1 = np.array([[2.0, 1.0], [1.0, 3.0]])     # stored [F][d]: h = relu([1, -2]) = [1, 0]
    W2 = np.array([[1.0, 5.0], [-2.0, 7.0]])    # stored [d][F]
    np.testing.assert_allclose(O.expert_ffn(x, W1, W2, act=O.RELU), [[1.0, -2.0]])


def _tiny_layer(rng, N, d, E, F, G, act=O.SWIGLU):
    x = rng.normal(0, 1, (N, d))
    W_g = rng.normal(0, 0.5, (E, d))
    rows = 2 * F if act == O.SWIGLU else F
    W_gu = rng.normal(0, 0.3, (G, rows, d))
    W_down = rng.normal(0, 0.3, (G, d, F))
    return x, W_g, W_gu, W_down


def test_dense_limit_k_equals_E():
    """k = E with softmax turns the layer into the dense mixture of all experts ("Основы MoE", "Практика")."""
    rng = np.random.default_rng(7)
    N, d, E, F = 9, 6, 5, 4
    x, W_g, W_gu, W_down = _tiny_layer(rng, N, d, E, F, E)
    y, _ = O.forward(x, W_g, W_gu, W_down, k=E, E=E)
    p = sp_softmax((x @ W_g.T).astype(np.float32).astype(np.float64), axis=1)   # logits are float32
    want = np.zeros_like(x)
    for t in range(N):
        for e in range(E):
            g = x[t] @ W_gu[e, :F].T
            u = x[t] @ W_gu[e, F:].T
            want[t] += p[t, e] * ((g / (1 + np.exp(-g)) * u) @ W_down[e].T)
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-13)
    # the oracle's own dense mixture is the same hand sum, and equals the routed layer at k = E
    dense = O.dense_mixture(x, W_g, W_gu, W_down, E=E)
    np.testing.assert_allclose(dense, want, rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(dense, y, rtol=1e-10, atol=1e-13)


def test_dense_mixture_reacts_to_every_term():
    """Each expert's term, the router and the SwiGLU clamp move ``dense_mixture``: a version
    that dropped an expert, ignored the logit offset or skipped the clamp would not."""
    rng = np.random.default_rng(17)
    N, d, E, F = 7, 5, 4, 3
    x, W_g, W_gu, W_down = _tiny_layer(rng, N, d, E, F, E)
    base = O.dense_mixture(x, W_g, W_gu, W_down, E=E)
    for e in range(E):
        W_down2 = W_down.copy()
        W_down2[e] = 0.0
        p = sp_softmax((x @ W_g.T).astype(np.float32).astype(np.float64), axis=1)
        g = x @ W_gu[e, :F].T
        u = x @ W_gu[e, F:].T
        term = p[:, e:e + 1] * ((g / (1 + np.exp(-g)) * u) @ W_down[e].T)
        np.testing.assert_allclose(O.dense_mixture(x, W_g, W_gu, W_down2, E=E), base - term,
                                   rtol=1e-9, atol=1e-12)
    # a huge offset on expert 2 makes the mixture that expert alone
    off = np.zeros(E, np.float32)
    off[2] = 1e3
    only2 = O.expert_ffn(x, W_gu[2], W_down[2])
    np.testing.assert_allclose(O.dense_mixture(x, W_g, W_gu, W_down, E=E, logit_offset=off),
                               only2, rtol=1e-12, atol=1e-12)
    # the clamp acts on the pre-activations: a tiny clamp bounds every |h| by c * 1
    big = x * 100
    clamped = O.dense_mixture(big, W_g, W_gu, W_down, E=E, clamp=0.5)
    assert not np.allclose(clamped, O.dense_mixture(big, W_g, W_gu, W_down, E=E))
    bound = 0.5 * 0.5 * np.abs(W_down).sum(axis=2).max()
    assert np.abs(clamped).max() <= bound + 1e-12


def test_forward_equals_dense_evaluation_masked_to_topk():
    """Brute force: evaluate all E experts on every token, keep the top-k by mask, weight by
    the renormalised softmax over the kept ones ("Основы MoE", steps 2-4), plus the shared
    expert with weight 1 ("Le groupe d'experts (MoE)", "Des experts partagés")."""
    rng = np.random.default_rng(19)
    N, d, E, F, k = 11, 6, 6, 4, 3
    x, W_g, W_gu, W_down = _tiny_layer(rng, N, d, E, F, E + 1)
    y, info = O.forward(x, W_g, W_gu, W_down, k=k, E=E, n_shared=1)
    z = (x @ W_g.T).astype(np.float32).astype(np.float64)
    want = np.zeros_like(x)
    for t in range(N):
        order = sorted(range(E), key=lambda e: (-z[t, e], e))[:k]
        w = np.exp(z[t, order] - z[t, order].max())
        w /= w.sum()
        outs = [O.expert_ffn(x[t:t + 1], W_gu[e], W_down[e])[0] for e in range(E + 1)]
        for e in range(E):
            if e in order:
                want[t] += w[order.index(e)] * outs[e]
        want[t] += outs[E]
    np.testing.assert_allclose(y, want, rtol=1e-10, atol=1e-12)


def test_linear_experts_closed_form_with_shared_and_capacity():
    """ReLU experts with positive inputs and weights act linearly: y = sum_kept g x A_e + x A_s."""
    rng = np.random.default_rng(8)
    N, d, E, F, k = 12, 3, 4, 5, 2
    x = rng.uniform(0.1, 1, (N, d))
    W_g = rng.normal(0, 1, (E, d))
    W1 = rng.uniform(0.1, 1, (E + 1, F, d))
    W2 = rng.normal(0, 1, (E + 1, d, F))
    C = 4
    y, info = O.forward(x, W_g, W1, W2, k=k, E=E, act=O.RELU, n_shared=1, C=C)
    A = [W1[e].T @ W2[e].T for e in range(E + 1)]            # d x d linear map of expert e
    z = (x @ W_g.T).astype(np.float32).astype(np.float64)
    seen = [0] * E
    for t in range(N):
        order = sorted(range(E), key=lambda e: (-z[t, e], e))[:k]
        ez = np.exp(z[t, order] - z[t, order].max())
        g = ez / ez.sum()
        want = x[t] @ A[E]
        for j, e in enumerate(order):
            if seen[e] < C:
                want = want + g[j] * (x[t] @ A[e])
            seen[e] += 1
        np.testing.assert_allclose(y[t], want, rtol=1e-12, atol=1e-12)


def test_trace_token6_output_is_second_gate_plus_shared():
    g, assign, T, E, k = _trace()
    rng = np.random.default_rng(12)
    d, F = 4, 3
    x = rng.normal(0, 1, (T, d))
    W_gu = rng.normal(0, 0.5, (E + 1, 2 * F, d))
    W_down = rng.normal(0, 0.5, (E + 1, d, F))
    z = _trace_logits(assign, E)
    y, info = O.forward(x, None, W_gu, W_down, k=k, E=E, n_shared=1, C=int(g["C_1.25"]), logits=z)
    t6 = 5
    g2 = math.exp(1.8) / (math.exp(2.1) + math.exp(1.8))
    assert round(g2, 3) == float(g["t6_kept_gate"])

    def ffn(e, v):
        gg = W_gu[e, :F] @ v
        uu = W_gu[e, F:] @ v
        return W_down[e] @ (gg / (1 + np.exp(-gg)) * uu)
    np.testing.assert_allclose(y[t6], g2 * ffn(1, x[t6]) + ffn(E, x[t6]), rtol=1e-6)
    # a token that kept both experts gets both, with gates 0.574 / 0.426
    g1 = 1 - g2
    np.testing.assert_allclose(y[0], g1 * ffn(0, x[0]) + g2 * ffn(1, x[0]) + ffn(E, x[0]), rtol=1e-6)


def test_forward_token_subset_matches_full():
    rng = np.random.default_rng(10)
    N, d, E, F = 40, 8, 6, 4
    x, W_g, W_gu, W_down = _tiny_layer(rng, N, d, E, F, E + 1)
    full, _ = O.forward(x, W_g, W_gu, W_down, k=2, E=E, n_shared=1, C=9)
    sub = [0, 7, 39, 13]
    part, _ = O.forward(x, W_g, W_gu, W_down, k=2, E=E, n_shared=1, C=9, tokens=sub)
    np.testing.assert_allclose(part, full[sub], rtol=1e-13)


def test_logit_offset_enters_selection_and_gates():
    """An offset added to the logits is not selection-only: it moves the gates too."""
    z = np.array([[1.0, 1.2, 0.0]], np.float32)
    off = np.array([0.5, 0.0, 0.0])
    x = np.ones((1, 3))
    W_g = np.diag(z[0].astype(np.float64))          # stored [E][d]: z = row sums
    zz = O.router_logits(x, W_g, off)
    ids, w = O.route(zz, 2)
    assert ids.tolist() == [[0, 1]]
    np.testing.assert_allclose(w[0], sp_softmax([1.5, 1.2]), rtol=1e-7)


# --------------------------------------------------------------------------
# forced (replayed) routing and the hash router ("Le groupe d'experts (MoE)", exercises)
# --------------------------------------------------------------------------
def test_forced_routing_reproduces_the_routed_layer_and_closed_forms():
    rng = np.random.default_rng(21)
    N, d, E, F = 30, 6, 5, 4
    x, W_g, W_gu, W_down = _tiny_layer(rng, N, d, E, F, E + 1)
    y, info = O.forward(x, W_g, W_gu, W_down, k=2, E=E, n_shared=1, C=11)
    y2, info2 = O.forward(x, None, W_gu, W_down, k=2, E=E, n_shared=1, C=11,
                          ids=info["ids"], gates=info["gates"])
    np.testing.assert_array_equal(y2, y)
    np.testing.assert_array_equal(info2["drop_mask"], info["drop_mask"])
    # every token forced to expert 3 with gate 1 and no capacity: y = FFN_3(x) + FFN_shared(x)
    ids = np.full((N, 1), 3, np.int32)
    y3, _ = O.forward(x, None, W_gu, W_down, k=1, E=E, n_shared=1, ids=ids, gates=np.ones((N, 1)))
    want = O.expert_ffn(x, W_gu[3], W_down[3]) + O.expert_ffn(x, W_gu[E], W_down[E])
    np.testing.assert_allclose(y3, want, rtol=1e-13)
    # and with capacity C the tokens after the C-th keep only the shared expert
    y4, d4 = O.forward(x, None, W_gu, W_down, k=1, E=E, n_shared=1, ids=ids,
                       gates=np.ones((N, 1)), C=7)
    np.testing.assert_allclose(y4[:7], want[:7], rtol=1e-13)
    np.testing.assert_allclose(y4[7:], O.expert_ffn(x[7:], W_gu[E], W_down[E]), rtol=1e-13)
    assert d4["drop_mask"][:, 0].tolist() == [0] * 7 + [1] * (N - 7)


def test_fmix32_is_a_bijection_with_fixed_points_of_the_definition():
    v = np.arange(1 << 16, dtype=np.uint64) * 65537          # 65536 distinct 32-bit inputs
    h = O.fmix32(v)
    assert np.unique(h).size == v.size
    assert int(O.fmix32(0)) == 0                             # every step maps 0 to 0
    # one step written out with Python integers (shift-xor, multiply mod 2^32, ...)
    a = 0xDEADBEEF
    a ^= a >> 16
    a = (a * 0x85EBCA6B) % 2**32
    a ^= a >> 13
    a = (a * 0xC2B2AE35) % 2**32
    a ^= a >> 16
    assert int(O.fmix32(0xDEADBEEF)) == a


def test_hash_route_is_deterministic_distinct_uniform():
    tok = np.arange(20000, dtype=np.int32) * 7 + 3
    ids, g = O.hash_route(tok, 64, 2)
    assert ids.shape == (20000, 2) and (ids[:, 0] != ids[:, 1]).all()
    np.testing.assert_array_equal(g, 0.5)
    ids2, _ = O.hash_route(tok, 64, 2)
    np.testing.assert_array_equal(ids, ids2)
    counts = np.bincount(ids.ravel(), minlength=64)
    # uniform load: chi-square with 63 degrees of freedom stays far below 130
    chi2 = ((counts - counts.mean()) ** 2 / counts.mean()).sum()
    assert chi2 < 130, chi2
    # the same token id always lands on the same experts, wherever it sits in the batch
    ids3, _ = O.hash_route(tok[::-1], 64, 2)
    np.testing.assert_array_equal(ids3[::-1], ids)


# --------------------------------------------------------------------------
# balancing statistics and the bias update
# --------------------------------------------------------------------------
def test_switch_balance_statistic_printed_example():
    g = load("p5_aux_loss.txt")
    E = int(g["N"])
    f, P = np.array(floats(g["load"])), np.array(floats(g["probs"]))
    # the statistic as defined: E * sum f_i P_i, here through balance_stats' own arithmetic
    # by building ids and logits whose f and P are exactly the printed ones
    ids = np.repeat(np.arange(E), (f * 10).astype(int))[:, None]          # 10 assignments
    z = np.log(np.tile(P, (len(ids), 1)))                                 # softmax(z) = P
    f_o, P_o, aux = O.balance_stats(z, ids, E)
    np.testing.assert_allclose(f_o, f, rtol=1e-12)
    np.testing.assert_allclose(P_o, P, rtol=1e-12)
    assert round(aux, 2) == float(g["value"])
    # uniform router and uniform load give 1; collapse onto one expert gives about E
    zu = np.zeros((8, E))
    idu = np.arange(8)[:, None] % E
    assert O.balance_stats(zu, idu, E)[2] == pytest.approx(float(g["uniform_value"]))
    zc = np.zeros((8, E)); zc[:, 0] = 50.0
    assert O.balance_stats(zc, np.zeros((8, 1), int), E)[2] == pytest.approx(E, rel=1e-12)


def test_bias_update_on_the_slides_trace_loads():
    # the slides' trace ("Cas guidé"): demand 6/4/3/3 (mean 4): E1 overloaded, E2 on target, E3 and E4 underloaded
    gt, assign, T, E, k = _trace()
    ids = np.array(assign, np.int32)
    load = O.per_set_load(ids, E)
    assert load.tolist() == [[6, 4, 3, 3]]
    b = O.bias_update(np.zeros((1, E), np.float32), load, 0.001)
    np.testing.assert_array_equal(b, np.float32([[-0.001, 0.0, 0.001, 0.001]]))
    # two modality sets are balanced separately
    mod = np.array([0, 0, 0, 0, 1, 1, 1, 1], np.uint8)
    load2 = O.per_set_load(ids, E, mod, 2)
    assert load2.tolist() == [[4, 2, 1, 1], [2, 2, 2, 2]]
    b2 = O.bias_update(np.zeros((2, E), np.float32), load2, 0.001)
    np.testing.assert_array_equal(b2[1], 0.0)
    np.testing.assert_array_equal(b2[0], np.float32([-0.001, 0.0, 0.001, 0.001]))   # mean 2


def test_sigmoid_probs_sum_to_one_and_follow_the_affinities():
    z = np.random.default_rng(2).normal(0, 1, (50, 9))
    P = O.router_probs(z, O.SIGMOID)
    np.testing.assert_allclose(P.sum(1), 1.0, rtol=1e-14)
    s = expit(z)
    np.testing.assert_allclose(P, s / s.sum(1, keepdims=True), rtol=1e-14)


def test_padded_dispatch_buffer_is_the_slides_table():
    """[E, C, d] buffer with C = 5: rows as printed, '.' = empty slot, t6 rejected."""
    g, assign, T, E, k = _trace()
    C = int(g["C_1.25"])
    ids = np.array(assign, np.int32)
    p = O.dispatch_padded(ids, E, C)
    for e in range(E):
        row = p["row_token"][e * C:(e + 1) * C]
        printed = ints(g[f"table_E{e}"])
        assert row[:len(printed)].tolist() == printed
        assert (row[len(printed):] == -1).all()
    assert int((p["row_token"] >= 0).sum()) == int(g["filled_1.25"])
    assert p["row_token"].size == int(g["slots_1.25"])
    # kept slots point back to their token; t6's first choice is the rejected one
    for t in range(T):
        for j in range(k):
            r = p["slot_row"][t, j]
            assert (r == -1) == bool(p["drop_mask"][t, j])
            if r >= 0:
                assert p["row_token"][r] == t and r // C == ids[t, j]
    assert p["slot_row"][5, 0] == -1


# --------------------------------------------------------------------------
# overflow policy "report" (slides, "Politiques de débordement"; reading R14)
# --------------------------------------------------------------------------
def test_report_policy_on_the_slides_trace():
    g, assign, T, E, k = _trace()
    C = int(g["C_1.25"])
    z = _trace_logits(assign, E)
    z[5, 3] = -1.0          # t6 = t1's logits on E1..E3; E4 below them
    ids, gates, drop, rerouted, first = O.route_reroute(z, k, C)
    assert first["drop_mask"].sum() == 1 and first["drop_mask"][5, 0] == 1
    t6_new = int(g["report_t6_expert"])
    assert ids[5].tolist() == [t6_new, 1]          # slot 0 (E1) moved to E3, E2 kept
    assert drop.sum() == 0 and rerouted.sum() == 1 and rerouted[5, 0] == 1
    assert (np.delete(ids, 5, axis=0) == np.delete(np.array(assign), 5, axis=0)).all()
    layout = O.dispatch_masked(ids, E, drop)
    assert layout["counts"].tolist() == [5, 4, 4, 3]
    # gates over t6's final list {E3, E2} from the printed exponentials 1.221 and 6.050
    e = floats(load("p2_router_example.txt")["exp"])
    np.testing.assert_allclose(gates[5], [e[2] / (e[1] + e[2]), e[1] / (e[1] + e[2])], atol=1e-3)
    # the other tokens keep their 0.574 / 0.426
    np.testing.assert_allclose(np.round(gates[0], 3), [0.574, 0.426])


def test_report_policy_without_overflow_is_plain_routing():
    rng = np.random.default_rng(21)
    z = rng.normal(0, 1.5, (300, 16)).astype(np.float32)
    for C in (0, 1000):
        ids, gates, drop, rerouted, _ = O.route_reroute(z, 3, C)
        ids_r, gates_r = O.route(z, 3)
        assert (ids == ids_r).all() and not drop.any() and not rerouted.any()
        np.testing.assert_array_equal(gates, gates_r)


def test_report_policy_closed_form_one_hot_expert():
    # every token ranks the experts 0 > 1 > 2 > 3; k = 1, C = 3: tokens 0-2 keep expert 0,
    # tokens 3-5 are moved to expert 1 (their second best), tokens 6-9 find it full: dropped
    z = np.tile(np.array([[3.0, 2.0, 1.0, 0.0]], np.float32), (10, 1))
    ids, gates, drop, rerouted, _ = O.route_reroute(z, 1, 3)
    assert ids[:, 0].tolist() == [0, 0, 0, 1, 1, 1, 0, 0, 0, 0]   # a refused slot keeps its id
    assert drop[:, 0].tolist() == [0] * 6 + [1] * 4
    assert rerouted[:, 0].tolist() == [0, 0, 0, 1, 1, 1, 0, 0, 0, 0]
    # renorm over a single slot: the gate is 1 whether the slot moved or not
    np.testing.assert_allclose(gates[:, 0], 1.0)
    # Switch gate (renorm = 0): the moved slot takes expert 1's own probability
    _, g0, _, _, _ = O.route_reroute(z, 1, 3, renorm=0)
    p = sp_softmax(z[0].astype(np.float64))
    np.testing.assert_allclose(g0[:3, 0], p[0])
    np.testing.assert_allclose(g0[3:6, 0], p[1])
    np.testing.assert_allclose(g0[6:, 0], p[0])     # refused: still expert 0's slot, output 0


def test_report_policy_invariants_random():
    rng = np.random.default_rng(22)
    N, E, k = 400, 12, 3
    z = (rng.normal(0, 1, (N, E)) + np.linspace(2, -2, E)[None, :]).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, (1, E)).astype(np.float32)
    for sf in (O.SOFTMAX, O.SIGMOID):
        C = O.capacity(N, k, E, 1)
        ids, gates, drop, rerouted, first = O.route_reroute(z, k, C, sf, 1, bias if sf else None)
        keys = O.selection_keys(z, sf, bias if sf else None)
        order = O.topk_ids(keys, 2 * k)
        lay = O.dispatch_masked(ids, E, drop)
        assert (lay["counts"] <= C).all()
        assert lay["counts"].sum() >= first["counts"].sum()
        for t in range(N):
            assert len(set(ids[t].tolist())) == k          # experts stay distinct per token
            i = 0
            for j in range(k):
                if first["drop_mask"][t, j]:
                    if rerouted[t, j]:
                        assert ids[t, j] == order[t, k + i]
                    else:
                        assert drop[t, j] and ids[t, j] == order[t, j]
                    i += 1
                else:
                    assert ids[t, j] == order[t, j] and not drop[t, j]
        # every expert that refused an offer is full
        for t in range(N):
            for j in range(k):
                if drop[t, j]:
                    i = int(first["drop_mask"][t, :j].sum())
                    if k + i < E:
                        assert lay["counts"][order[t, k + i]] == C


def test_forward_with_report_policy_matches_hand_sum():
    g, assign, T, E, k = _trace()
    rng = np.random.default_rng(23)
    d, F = 4, 3
    x = rng.normal(0, 1, (T, d))
    W_gu = rng.normal(0, 0.5, (E + 1, 2 * F, d))
    W_down = rng.normal(0, 0.5, (E + 1, d, F))
    z = _trace_logits(assign, E)
    z[5, 3] = -1.0
    y, info = O.forward(x, None, W_gu, W_down, k=k, E=E, n_shared=1, C=int(g["C_1.25"]),
                        logits=z, overflow="reroute")

    def ffn(e, v):
        gg = W_gu[e, :F] @ v
        uu = W_gu[e, F:] @ v
        return W_down[e] @ (gg / (1 + np.exp(-gg)) * uu)
    e3 = math.exp(0.2) / (math.exp(0.2) + math.exp(1.8))
    np.testing.assert_allclose(y[5], e3 * ffn(2, x[5]) + (1 - e3) * ffn(1, x[5]) + ffn(E, x[5]),
                               rtol=1e-6)
    assert info["drop_mask"].sum() == 0 and info["rerouted"].sum() == 1
    assert info["demand"].tolist() == [6, 4, 3, 3]
